"""GPU parity of gdn_backward (through the C ABI) against the oracle's reverse recurrence.

Bar: every gradient tensor within max|g - g_ref| / max|g_ref| <= 1e-2; dS0 also in relative
Frobenius norm <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import make_inputs
from tests._metrics import G_TOL, S_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu

NAMES = ["dq", "dk", "dv", "dalpha", "dbeta", "ds0"]


def _run(inp, ds_final=None, scale=1.0, l2norm=True):
    g = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    out = api.gdn_backward(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["dy"], s0=g["s0"],
                           ds_final=None if ds_final is None else ds_final.cuda(), scale=scale,
                           l2norm_qk=l2norm)
    torch.cuda.synchronize()
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], s0=inp["s0"],
                          dy=inp["dy"], ds_final=ds_final, scale=scale, l2norm=l2norm)
    return out, ref


def _check(out, ref):
    for n in NAMES:
        assert max_rel(out[n], ref[n]) <= G_TOL, n
    assert frob_rel(out["ds0"], ref["ds0"]) <= S_TOL


@pytest.mark.parametrize("B,T,H,d,dtype", [
    (1, 64, 1, 128, "bf16"),
    (2, 150, 2, 128, "bf16"),   # ragged final chunk
    (1, 70, 3, 64, "bf16"),
    (2, 33, 2, 64, "fp32"),
    (1, 130, 2, 128, "fp32"),
])
def test_backward_small(B, T, H, d, dtype):
    inp = make_inputs(B, T, H, d, d, dtype=dtype, seed=T + d, with_s0=True, with_dy=True)
    out, ref = _run(inp)
    _check(out, ref)


def test_backward_with_state_gradient_scale_and_no_norm():
    B, T, H, d = 1, 100, 2, 128
    inp = make_inputs(B, T, H, d, d, seed=9, with_s0=True, with_dy=True)
    for n in ("q", "k"):
        x = inp[n].double()
        inp[n] = (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    rng = np.random.default_rng(4)
    dsf = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32))
    out, ref = _run(inp, ds_final=dsf, scale=0.5, l2norm=False)
    _check(out, ref)


@pytest.mark.parametrize("d", [64, 128])
def test_backward_long_with_states(d):
    """13 chunks (ragged last) through both chunk chains, with a nonzero S0, dS_final and scale."""
    B, T, H = 1, 777, 2
    inp = make_inputs(B, T, H, d, d, seed=31 + d, with_s0=True, with_dy=True)
    rng = np.random.default_rng(d)
    dsf = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32))
    out, ref = _run(inp, ds_final=dsf, scale=0.9)
    _check(out, ref)


def test_backward_training_config_full():
    """Training shape B=8, T=4096, H=32, dk=dv=128, bf16, dy ~ N(0,1), S0 = 0, dS_final = 0.
    Every (sequence, head) chain against the oracle's reverse recurrence, one sequence at a
    time to bound host memory; the bars hold per sequence and for dS0 per chain."""
    B, T, H, d = 8, 4096, 32, 128
    inp = make_inputs(B, T, H, d, d, seed=0, with_dy=True)
    g = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    out = api.gdn_backward(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["dy"])
    torch.cuda.synchronize()
    out = {n: out[n].cpu() for n in NAMES}
    del g
    for b in range(B):
        sub = {n: inp[n][b:b + 1].contiguous() for n in ("q", "k", "v", "alpha", "beta", "dy")}
        ref = oracle.backward(sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"],
                              dy=sub["dy"])
        for n in ("dq", "dk", "dv", "dalpha", "dbeta"):
            assert max_rel(out[n][b:b + 1], ref[n]) <= G_TOL, (n, b)
        for h in range(H):
            assert frob_rel(out["ds0"][b, h], ref["ds0"][0, h]) <= S_TOL, (b, h)


def test_backward_workspace_is_caller_owned():
    """The caller can hand in its own workspace of exactly gdn_workspace_bytes()."""
    from gated_deltanet_linear_eqs_b200._abi import GDN_OP_BACKWARD
    B, T, H, d = 1, 80, 2, 64
    inp = make_inputs(B, T, H, d, d, seed=2, with_dy=True)
    n = api.gdn_workspace_bytes(GDN_OP_BACKWARD, B, T, H, d, d)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    g = {k: (t.cuda() if isinstance(t, torch.Tensor) else t) for k, t in inp.items()}
    out = api.gdn_backward(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["dy"], ws=ws)
    torch.cuda.synchronize()
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], dy=inp["dy"])
    for k in ("dq", "dk", "dv", "dalpha", "dbeta"):
        assert max_rel(out[k], ref[k]) <= G_TOL, k


def test_backward_slow_decay():
    """Slow decays (alpha uniform in [0.97, 0.9995]) carry state and its gradient across many
    chunks; every gradient and dS0 stay within their bars."""
    B, T, H, d = 1, 1000, 2, 128
    inp = make_inputs(B, T, H, d, d, seed=17, with_s0=True, with_dy=True)
    rng = np.random.default_rng(18)
    inp["alpha"] = torch.from_numpy(rng.uniform(0.97, 0.9995, (B, T, H)).astype(np.float32))
    out, ref = _run(inp)
    print("slow decays: " + ", ".join(f"{n} {max_rel(out[n], ref[n]):.2e}" for n in NAMES)
          + f", dS0 frob {frob_rel(out['ds0'], ref['ds0']):.2e}")
    _check(out, ref)

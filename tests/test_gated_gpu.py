"""GPU parity of the gated form (eqs. (9)-(10) feeding the recurrence) and of the gated RMSNorm
(eq. (11)), through the C ABI, against the fp64 oracle (``oracle/gates.py`` around the token
loop).

Bars as for the plain calls: y max|dy|/max|y_ref| <= 1e-2, states relative Frobenius <= 1e-3,
every gradient tensor max-normalised <= 1e-2 and dS0 in Frobenius norm <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
import oracle.gates as og
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import (cu_seqlens_from, make_gate_inputs,
                                                   make_inputs, make_norm_inputs)
from tests._metrics import G_TOL, S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


def _cuda(d):
    return {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in d.items()}


def _gates(gi):
    """alpha, beta of eqs. (9)-(10) in fp64 from the same fp32 logits."""
    _, alpha, beta = og.gates(gi["a"], gi["b"], gi["A_log"], gi["b_alpha"])
    return alpha, beta


@pytest.mark.parametrize("B,T,H,d,dtype", [
    (1, 64, 2, 128, "bf16"),
    (2, 200, 3, 128, "bf16"),   # ragged tail
    (1, 130, 2, 64, "bf16"),
    (2, 77, 2, 64, "fp32"),     # the token-loop path
])
def test_gated_prefill_dense(B, T, H, d, dtype):
    inp = make_inputs(B, T, H, d, d, dtype=dtype, seed=T + d, with_s0=True)
    gi = make_gate_inputs((B, T, H), H, seed=T)
    g, gg = _cuda(inp), _cuda(gi)
    y, sf = api.gdn_prefill_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                  gg["b_alpha"], g["s0"], scale=0.8)
    torch.cuda.synchronize()
    alpha, beta = _gates(gi)
    yr, sr = oracle.forward(inp["q"], inp["k"], inp["v"], alpha, beta, inp["s0"], scale=0.8)
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(sf, sr) <= S_TOL


@pytest.mark.parametrize("d", [64, 128])
def test_gated_prefill_varlen(d):
    lengths = [100, 0, 257, 64, 3]
    T, H = sum(lengths), 2
    inp = make_inputs(1, T, H, d, d, seed=d, with_s0=True, num_states=len(lengths))
    gi = make_gate_inputs((1, T, H), H, seed=d + 1)
    cu = cu_seqlens_from(lengths)
    g, gg = _cuda(inp), _cuda(gi)
    y, sf = api.gdn_prefill_varlen_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                         gg["b_alpha"], cu.cuda(), g["s0"])
    torch.cuda.synchronize()
    alpha, beta = _gates(gi)
    yr, sr = oracle.forward_varlen(inp["q"], inp["k"], inp["v"], alpha, beta, cu.numpy(),
                                   inp["s0"])
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(sf, sr) <= S_TOL


def test_gated_prefill_strong_decay_in_log_space():
    """Logits whose decay underflows fp32 (ln alpha near -220): the gated path keeps ln alpha
    and resets the state there, as the fp64 oracle does."""
    B, T, H, d = 1, 192, 2, 128
    inp = make_inputs(B, T, H, d, d, seed=5, with_s0=True)
    gi = make_gate_inputs((B, T, H), H, seed=6)
    gi["a"][0, 70] = 30.0
    gi["a"][0, 150:153] = 25.0
    gi["A_log"][:] = 2.0
    g, gg = _cuda(inp), _cuda(gi)
    y, sf = api.gdn_prefill_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                  gg["b_alpha"], g["s0"])
    torch.cuda.synchronize()
    alpha, beta = _gates(gi)
    assert alpha.min() < 1e-60
    yr, sr = oracle.forward(inp["q"], inp["k"], inp["v"], alpha, beta, inp["s0"])
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(sf, sr) <= S_TOL


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_gated_decode_steps(dtype, d):
    N, H, steps = 6, 2, 5
    S0 = make_inputs(N, 1, H, d, d, seed=11, with_s0=True)["s0"]
    per_head = make_gate_inputs((1, H), H, seed=7)
    Sg = S0.cuda()
    Sr = S0.double().numpy()
    for t in range(steps):
        inp = make_inputs(N, 1, H, d, d, dtype=dtype, seed=20 + t)
        tok = {n: inp[n][:, 0] for n in ("q", "k", "v")}
        gi = make_gate_inputs((N, H), H, seed=40 + t)
        gi["A_log"], gi["b_alpha"] = per_head["A_log"], per_head["b_alpha"]  # fixed parameters
        g, gg = _cuda(tok), _cuda(gi)
        y = api.gdn_decode_step_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                      gg["b_alpha"], Sg, scale=0.5)
        torch.cuda.synchronize()
        alpha, beta = _gates(gi)
        yr, Sr = oracle.decode_step(tok["q"], tok["k"], tok["v"], alpha, beta, Sr, scale=0.5)
        assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(Sg, Sr) <= S_TOL


@pytest.mark.parametrize("B,T,H,d,dtype", [
    (1, 64, 2, 128, "bf16"),
    (2, 150, 2, 128, "bf16"),   # ragged final chunk
    (1, 70, 3, 64, "fp32"),
])
def test_gated_backward(B, T, H, d, dtype):
    inp = make_inputs(B, T, H, d, d, dtype=dtype, seed=T + 3, with_s0=True, with_dy=True)
    gi = make_gate_inputs((B, T, H), H, seed=T + 4)
    rng = np.random.default_rng(T)
    dsf = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32))
    g, gg = _cuda(inp), _cuda(gi)
    out = api.gdn_backward_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                 gg["b_alpha"], g["dy"], s0=g["s0"], ds_final=dsf.cuda(),
                                 scale=0.9)
    torch.cuda.synchronize()
    alpha, beta = _gates(gi)
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], alpha, beta, s0=inp["s0"], dy=inp["dy"],
                          ds_final=dsf, scale=0.9)
    gref = og.gates_backward(gi["a"], gi["b"], gi["A_log"], gi["b_alpha"],
                             dalpha=ref["dalpha"], dbeta=ref["dbeta"])
    for n in ("dq", "dk", "dv", "ds0"):
        assert max_rel(out[n], ref[n]) <= G_TOL, n
    for n, r in (("da", "da"), ("db", "db"), ("dA_log", "dA_log"), ("db_alpha", "db_alpha")):
        assert max_rel(out[n], gref[r]) <= G_TOL, n
    assert frob_rel(out["ds0"], ref["ds0"]) <= S_TOL


@pytest.mark.parametrize("rows,dv,dtype", [
    (1000, 128, "bf16"), (333, 64, "bf16"), (517, 128, "fp32"), (3, 64, "fp32"), (0, 128, "bf16"),
])
def test_gated_rmsnorm(rows, dv, dtype):
    inp = make_norm_inputs(rows, dv, dtype=dtype, seed=rows + dv)
    g = _cuda(inp)
    o = api.gdn_gated_rmsnorm(g["y"], g["z"], g["w"])
    torch.cuda.synchronize()
    assert o.shape == (rows, dv) and o.dtype == inp["y"].dtype
    if rows == 0:
        return
    ref = og.gated_output(inp["y"].double().numpy(), inp["z"].double().numpy(),
                          inp["w"].double().numpy())
    tol = Y_TOL if dtype == "bf16" else 1e-5
    assert max_rel(o, ref) <= tol


@pytest.mark.parametrize("rows,dv,dtype", [(1000, 128, "bf16"), (333, 64, "fp32"), (0, 64, "fp32")])
def test_gated_rmsnorm_backward(rows, dv, dtype):
    inp = make_norm_inputs(rows, dv, dtype=dtype, seed=rows + 2 * dv, with_do=True)
    g = _cuda(inp)
    out = api.gdn_gated_rmsnorm_backward(g["y"], g["z"], g["w"], g["d_o"])
    torch.cuda.synchronize()
    if rows == 0:
        assert torch.count_nonzero(out["dw"]).item() == 0
        return
    ref = og.gated_output_backward(inp["y"].double().numpy(), inp["z"].double().numpy(),
                                   inp["w"].double().numpy(), inp["d_o"].double().numpy())
    for n in ("dy", "dz", "dw"):
        assert max_rel(out[n], ref[n]) <= G_TOL, n


def test_gated_layer_core_end_to_end():
    """Gates -> recurrence -> gated RMSNorm on the GPU equals the oracle's layer_core."""
    B, T, H, d = 1, 300, 4, 128
    inp = make_inputs(B, T, H, d, d, seed=77, with_s0=True)
    gi = make_gate_inputs((B, T, H), H, seed=78)
    ni = make_norm_inputs(B * T * H, d, seed=79)
    z = ni["z"].reshape(B, T, H, d)
    g, gg = _cuda(inp), _cuda(gi)
    y, sf = api.gdn_prefill_gated(g["q"], g["k"], g["v"], gg["a"], gg["b"], gg["A_log"],
                                  gg["b_alpha"], g["s0"])
    o = api.gdn_gated_rmsnorm(y, z.cuda(), ni["w"].cuda())
    torch.cuda.synchronize()
    o_ref, _, s_ref = og.layer_core(inp["q"], inp["k"], inp["v"], gi["a"], gi["b"],
                                    z.double().numpy(), gi["A_log"], gi["b_alpha"],
                                    ni["w"].double().numpy(), s0=inp["s0"])
    assert max_rel(o, o_ref) <= Y_TOL
    assert frob_rel(sf, s_ref) <= S_TOL

"""gdn_backward_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (a plugin whose device memory belongs to its host framework's pool, a server
that reserves all memory at start-up) cannot hand the backward pass a workspace from
cudaMalloc.  This entry point runs the token-loop form of the backward on a fixed scratch
array built into the library (gdn_backward runs the chunked form).  The GPU test calls it
through the C ABI twice in a row, on different inputs, and compares each result with the fp64
oracle's reverse recurrence and with gdn_backward's on the same inputs.  The second call checks
that the contents the first call leaves in the shared array cannot leak into the next result.
This file is collected last; it passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import _abi, api
from gated_deltanet_linear_eqs_b200.build import build
from gated_deltanet_linear_eqs_b200.inputs import make_inputs
from tests._metrics import G_TOL, S_TOL, frob_rel, max_rel

NAMES = ["dq", "dk", "dv", "dalpha", "dbeta", "ds0"]


def _cuda(inp):
    return {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,H,d,dtype", [(2, 200, 2, 128, "bf16"), (1, 130, 3, 64, "fp32")])
def test_noalloc_matches_backward_on_two_calls(B, T, H, d, dtype):
    need = ((T + 63) // 64 + 64) * B * H * d * d * 4  # the token-loop scratch
    assert need <= api.gdn_backward_noalloc_max_workspace()
    rng = np.random.default_rng(7)
    for call in range(2):
        inp = make_inputs(B, T, H, d, d, dtype=dtype, seed=100 + call, with_s0=True, with_dy=True)
        g = _cuda(inp)
        dsf_h = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32))
        dsf = dsf_h.cuda()
        exact = oracle.backward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                s0=inp["s0"], dy=inp["dy"], ds_final=dsf_h, scale=0.8)
        ref = api.gdn_backward(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["dy"],
                               s0=g["s0"], ds_final=dsf, scale=0.8)
        out = api.gdn_backward_noalloc(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["dy"],
                                       s0=g["s0"], ds_final=dsf, scale=0.8)
        torch.cuda.synchronize()
        for n in NAMES:
            assert torch.isfinite(out[n]).all(), (call, n)
            assert max_rel(out[n], exact[n]) <= G_TOL, (call, n)
            assert max_rel(out[n], ref[n]) <= G_TOL, (call, n)
        assert frob_rel(out["ds0"], exact["ds0"]) <= S_TOL, call
        assert frob_rel(out["ds0"], ref["ds0"]) <= S_TOL, call


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A workspace larger than the fixed scratch is refused before anything is launched."""
    build()
    lib = _abi.load()
    cap = lib.gdn_backward_noalloc_max_workspace()
    assert cap == 32 << 20
    A = 0x10000  # aligned placeholder addresses: the size check rejects before any access
    args = [A] * 6 + [A, 0] + [A] * 6
    # B*H*(ceil(T/64) + 64) * 128*128*4 bytes: 8*32*(64+64) states of 64 KiB each >> 32 MiB
    assert lib.gdn_backward_noalloc(*args, 8, 4096, 32, 128, 128, 0, 1.0, 1, None) == \
        _abi.GDN_ERR_WORKSPACE
    # one state over the limit: (ceil(T/64) + 64) = 513 states at d = 128, B = H = 1
    assert lib.gdn_backward_noalloc(*args, 1, 449 * 64, 1, 128, 128, 0, 1.0, 1, None) == \
        _abi.GDN_ERR_WORKSPACE

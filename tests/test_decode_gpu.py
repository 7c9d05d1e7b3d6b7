"""GPU parity of gdn_decode_step (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import (make_decode_state, make_decode_step_inputs,
                                                   make_inputs)
from tests._metrics import S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


def _dev(d):
    return {n: (t.cuda() if t is not None else None) for n, t in d.items()}


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 64), ("fp32", 128)])
@pytest.mark.parametrize("l2norm", [True, False])
def test_decode_one_step(dtype, d, l2norm):
    N, H = 5, 3
    inp = make_decode_step_inputs(N, H, d, d, step=0, dtype=dtype)
    if not l2norm:  # feed unit-norm keys/queries when the kernel does not normalise
        for n in ("q", "k"):
            x = inp[n].double()
            inp[n] = (x / x.norm(dim=-1, keepdim=True)).to(inp[n].dtype)
    S = make_decode_state(N, H, d, d, seed=3)
    g = _dev(inp)
    Sg = S.cuda()
    y = api.gdn_decode_step(g["q"], g["k"], g["v"], g["alpha"], g["beta"], Sg, scale=0.75,
                            l2norm_qk=l2norm)
    torch.cuda.synchronize()
    yr, Sr = oracle.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], S,
                                scale=0.75, l2norm=l2norm)
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(Sg, Sr) <= S_TOL
    # fp32 state arithmetic: far inside the bar
    assert frob_rel(Sg, Sr) <= 1e-5


def test_decode_many_steps_small():
    N, H, d, steps = 3, 2, 128, 40
    S = make_decode_state(N, H, d, d, seed=5)
    Sg = S.cuda()
    Sr = S.double().numpy()
    for t in range(steps):
        inp = make_decode_step_inputs(N, H, d, d, step=t)
        g = _dev(inp)
        y = api.gdn_decode_step(g["q"], g["k"], g["v"], g["alpha"], g["beta"], Sg)
        yr, Sr = oracle.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], Sr)
        assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(Sg, Sr) <= 1e-5


def test_decode_full_size_1000_steps_full():
    """Full decode workload (256 sequences x 16 heads x 128 x 128 fp32 state, 1000 steps with
    fresh seeded tokens); the oracle follows every (sequence, head) pair all the way: y of
    every step within the y bar, and the final state within the state bar per pair."""
    N, H, d, steps = 256, 16, 128, 1000
    S = make_decode_state(N, H, d, d, seed=0)
    Sg = S.cuda()
    Sr = S.double().numpy()
    worst_y = 0.0
    for t in range(steps):
        inp = make_decode_step_inputs(N, H, d, d, step=t)
        g = _dev(inp)
        y = api.gdn_decode_step(g["q"], g["k"], g["v"], g["alpha"], g["beta"], Sg)
        yr, Sr = oracle.decode_step(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], Sr)
        worst_y = max(worst_y, max_rel(y, yr))
    assert worst_y <= Y_TOL
    Sg = Sg.cpu()
    assert frob_rel(Sg, Sr) <= S_TOL
    for n in range(N):
        assert frob_rel(Sg[n], Sr[n]) <= S_TOL, n


def test_decode_equals_oracle_prefill_of_same_tokens():
    """T decode steps equal one prefill of T tokens (oracle prefill as the reference)."""
    N, H, d, T = 2, 2, 64, 9
    inp = make_inputs(N, T, H, d, d, seed=11, with_s0=True)
    Sg = inp["s0"].clone().cuda()
    ys = []
    for t in range(T):
        g = {n: inp[n][:, t].contiguous().cuda() for n in ("q", "k", "v", "alpha", "beta")}
        ys.append(api.gdn_decode_step(g["q"], g["k"], g["v"], g["alpha"], g["beta"], Sg))
    y = torch.stack(ys, 1)
    yr, Sr = oracle.forward(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["s0"])
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(Sg, Sr) <= 1e-5

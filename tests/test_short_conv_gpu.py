"""GPU parity of the short causal convolution (gdn_short_conv_varlen / gdn_short_conv_step,
through the C ABI) against the fp64 oracle (oracle/short_conv.py).

Bars: outputs max|dy|/max|y_ref| <= 1e-2 for bf16 (rounding of the output), <= 1e-5 for fp32;
the conv states are copies of inputs, so they must match exactly."""
import numpy as np
import pytest
import torch

import oracle
import oracle.short_conv as oconv
from gated_deltanet_linear_eqs_b200 import api
from gated_deltanet_linear_eqs_b200.inputs import (make_conv_inputs, make_varlen_inputs,
                                                   varlen_lengths)
from tests._metrics import S_TOL, Y_TOL, frob_rel, max_rel

pytestmark = pytest.mark.gpu


def _run(inp, activation):
    g = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in inp.items()}
    y, sf = api.gdn_short_conv_varlen(g["x"], g["w"], g["cu_seqlens"], g["conv_state"],
                                      activation=activation)
    torch.cuda.synchronize()
    yr, sr = oconv.short_conv_varlen(inp["x"], inp["w"], inp["cu_seqlens"].numpy(),
                                     inp["conv_state"], activation=activation)
    return y, sf, yr, sr


def _tol(dtype):
    return Y_TOL if dtype == "bf16" else 1e-5


@pytest.mark.parametrize("lengths", [[1, 2, 3, 40], [0, 17, 0, 5, 16, 33], [300], [3, 0]])
@pytest.mark.parametrize("W", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype,act", [("bf16", "silu"), ("bf16", "none"), ("fp32", "silu")])
def test_short_conv_varlen_small(lengths, W, dtype, act):
    C = 2048 + 64  # two channel blocks, the second partly filled
    inp = make_conv_inputs(lengths, C, W, dtype=dtype, seed=W + sum(lengths))
    y, sf, yr, sr = _run(inp, act)
    if sum(lengths):
        assert max_rel(y, yr) <= _tol(dtype)
    np.testing.assert_array_equal(sf.double().cpu().numpy(), sr)


def test_short_conv_without_state():
    inp = make_conv_inputs([5, 70, 1], 256, 4, seed=9, with_state=False)
    y, sf, yr, sr = _run(inp, "silu")
    assert max_rel(y, yr) <= Y_TOL
    np.testing.assert_array_equal(sf.double().cpu().numpy(), sr)


def test_short_conv_long_varlen_fused_qkv():
    """The long varlen workload's q, k, v as one fused [32768, 3 * 16 * 128] tensor, 4 seeded
    documents, W = 4, SiLU, seeded conv states (whole tensors)."""
    lengths = varlen_lengths(32768, 4, seed=0)
    inp = make_conv_inputs(lengths, 3 * 16 * 128, 4, seed=0)
    y, sf, yr, sr = _run(inp, "silu")
    assert max_rel(y, yr) <= Y_TOL
    np.testing.assert_array_equal(sf.double().cpu().numpy(), sr)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_short_conv_decode_steps(dtype):
    """50 decode steps (state updated in place) against the oracle's steps, then against one
    packed call over the same tokens."""
    N, C, W, steps = 37, 384, 4, 50
    inp = make_conv_inputs([steps] * N, C, W, dtype=dtype, seed=3)
    x = inp["x"].view(N, steps, C)
    st = inp["conv_state"].cuda().clone()
    sr = inp["conv_state"].double().numpy()
    w = inp["w"].cuda()
    ys = []
    for t in range(steps):
        xt = x[:, t].contiguous()
        y = api.gdn_short_conv_step(xt.cuda(), w, st, activation="silu")
        yr, sr = oconv.short_conv_step(xt, inp["w"], sr, activation="silu")
        assert max_rel(y, yr) <= _tol(dtype)
        ys.append(y)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(st.double().cpu().numpy(), sr)
    yall, sall = api.gdn_short_conv_varlen(inp["x"].cuda(), w, inp["cu_seqlens"].cuda(),
                                           inp["conv_state"].cuda(), activation="silu")
    assert torch.equal(torch.stack(ys, 1).reshape(N * steps, C), yall)
    assert torch.equal(sall, st)


def test_short_conv_then_prefill():
    """The convolution ahead of the recurrence: conv(q), conv(k), conv(v) on the GPU, then the
    varlen prefill (L2 norm fused), against the oracle's convolution and token loop."""
    lengths, H, d, W = [100, 37, 200], 2, 128, 4
    inp = make_varlen_inputs(lengths, H, d, d, seed=41)
    cu = inp["cu_seqlens"]
    T = int(cu[-1])
    taps = make_conv_inputs(lengths, H * d, W, seed=42)
    conv = {}
    ref = {}
    for i, n in enumerate(("q", "k", "v")):
        x = inp[n].reshape(T, H * d)
        w = taps["w"] * (1.0 + 0.25 * i)
        yg, _ = api.gdn_short_conv_varlen(x.cuda(), w.cuda(), cu.cuda(), None, activation="silu",
                                          return_state=False)
        conv[n] = yg.view(1, T, H, d)
        ref[n] = oconv.short_conv_varlen(x, w, cu.numpy(), None, activation="silu")[0]
    g = {n: inp[n].cuda() for n in ("alpha", "beta", "s0")}
    y, sf = api.gdn_prefill_varlen(conv["q"], conv["k"], conv["v"], g["alpha"], g["beta"],
                                   cu.cuda(), g["s0"])
    torch.cuda.synchronize()
    # the oracle recurrence sees the convolution's outputs as the kernel stored them (bf16)
    for n in ("q", "k", "v"):
        assert max_rel(conv[n].reshape(T, H * d), ref[n]) <= Y_TOL
    yr, sr = oracle.forward_varlen(conv["q"].cpu(), conv["k"].cpu(), conv["v"].cpu(),
                                   inp["alpha"], inp["beta"], cu.numpy(), inp["s0"])
    assert max_rel(y, yr) <= Y_TOL
    assert frob_rel(sf, sr) <= S_TOL

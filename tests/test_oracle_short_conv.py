"""Pins for the fp64 oracle of the short causal convolution (``oracle/short_conv.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "1. GDN Hybrid Token Mixing":
"short causal convolutions" ahead of the recurrence, in the depthwise reading the
oracle states.  Each check takes the module under test, so that the mutation tests can
run the same checks against a copy with a planted mistake.
"""
import math
import os

import numpy as np
import pytest

import oracle.short_conv as conv_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            d[key] = np.array([float(x) for x in vals])
    return d


def _rand(seed, T, C, W, N=1):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, C)), rng.standard_normal((C, W)),
            rng.standard_normal((N, W - 1, C)))


# --------------------------------------------------------------------------- checks


def check_hand_example(M):
    """Three documents worked by hand (tests/golden/short_conv_hand.txt): a full one, one
    shorter than W - 1 and an empty one."""
    g = _load_golden("short_conv_hand.txt")
    C, W = int(g["C"][0]), int(g["W"][0])
    cu = g["cu"].astype(int)
    N = len(cu) - 1
    y, fin = M.short_conv_varlen(g["x"].reshape(-1, C), g["w"].reshape(C, W), cu,
                                 g["state"].reshape(N, W - 1, C))
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(fin.ravel(), g["final"], rtol=0, atol=1e-15)


def check_identity_and_delay_taps(M):
    """Taps (0, .., 0, 1) give y = x and keep the last W - 1 inputs as the state; taps with
    the one at position W - 1 - s delay the input by s tokens, reading the state where the
    delay reaches before the document."""
    T, C, W = 9, 5, 4
    x, _, st = _rand(1, T, C, W)
    eye = np.zeros((C, W))
    eye[:, -1] = 1.0
    y, fin = M.short_conv_varlen(x, eye, [0, T], st)
    np.testing.assert_array_equal(y, x)
    np.testing.assert_array_equal(fin[0], x[T - (W - 1):])
    for s in range(1, W):
        w = np.zeros((C, W))
        w[:, W - 1 - s] = 1.0
        y, _ = M.short_conv_varlen(x, w, [0, T], st)
        np.testing.assert_array_equal(y[s:], x[:T - s])
        np.testing.assert_array_equal(y[:s], st[0, W - 1 - s:])


def check_matches_numpy_convolve(M):
    """Per channel, one document with a zero state is numpy's full discrete convolution with
    the taps reversed, truncated to the first T outputs."""
    T, C, W = 17, 3, 4
    x, w, _ = _rand(2, T, C, W)
    y, _ = M.short_conv_varlen(x, w, [0, T], None)
    for c in range(C):
        ref = np.convolve(x[:, c], w[c, ::-1])[:T]
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-13, atol=1e-13)


def check_resume_and_varlen(M):
    """Splitting a document and passing the state on gives the same outputs and state; packed
    documents equal separate calls."""
    T, C, W = 23, 4, 4
    x, w, st = _rand(3, T, C, W)
    y, fin = M.short_conv_varlen(x, w, [0, T], st)
    for cut in (1, 2, 3, 11, 22):
        y1, f1 = M.short_conv_varlen(x[:cut], w, [0, cut], st)
        y2, f2 = M.short_conv_varlen(x[cut:], w, [0, T - cut], f1)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(f2, fin, rtol=1e-13, atol=1e-14)
    lens = [5, 0, 1, 2, 15]
    cu = np.concatenate([[0], np.cumsum(lens)])
    stN = np.random.default_rng(4).standard_normal((len(lens), W - 1, C))
    yp, fp = M.short_conv_varlen(x, w, cu, stN, activation="silu")
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        yn, fn = M.short_conv_varlen(x[a:b], w, [0, b - a], stN[n:n + 1], activation="silu")
        np.testing.assert_allclose(yp[a:b], yn, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(fp[n], fn[0], rtol=1e-13, atol=1e-14)


def check_decode_steps(M):
    """T decode steps equal one document of T tokens (outputs and state)."""
    T, C, W = 7, 6, 3
    x, w, st = _rand(5, T, C, W)
    y, fin = M.short_conv_varlen(x, w, [0, T], st, activation="silu")
    s = st.copy()
    for t in range(T):
        yt, s = M.short_conv_step(x[t:t + 1], w, s, activation="silu")
        np.testing.assert_allclose(yt[0], y[t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s, fin, rtol=1e-13, atol=1e-14)


def check_silu_closed_forms(M):
    """SiLU(x) = x sigmoid(x): 0 at 0, (3/4) ln 3 at ln 3, -(1/4) ln 3 at -ln 3; through the
    convolution with the identity taps."""
    x = np.array([[0.0], [math.log(3.0)], [-math.log(3.0)]])
    w = np.array([[0.0, 1.0]])
    y, _ = M.short_conv_varlen(x, w, [0, 3], None, activation="silu")
    np.testing.assert_allclose(y[:, 0], [0.0, 0.75 * math.log(3.0), -0.25 * math.log(3.0)],
                               rtol=1e-15, atol=1e-16)


CHECKS = [check_hand_example, check_identity_and_delay_taps, check_matches_numpy_convolve,
          check_resume_and_varlen, check_decode_steps, check_silu_closed_forms]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_short_conv_oracle(check):
    check(conv_mod)

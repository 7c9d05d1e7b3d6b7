"""Pins for the fp64 oracle of the gates and the gated output (``oracle/gates.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "1. GDN Hybrid Token Mixing",
eqs. (9)-(11).  Each check takes the module under test as its argument, so that
``test_oracle_mutants`` can run the same checks against a copy with a planted mistake.
"""
import math
import os

import numpy as np
import pytest

import oracle
import oracle.gates as gates_mod

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


# --------------------------------------------------------------------------- checks


def check_decay_closed_forms(G):
    """Eq. (10) with A = 0 is exp(-softplus(x)) = 1/(1 + e^x); with A = ln 2 it is the
    square of that; exact values at ln 3: softplus(ln 3) = ln 4, softplus(-ln 3) = ln(4/3)."""
    x = np.linspace(-20.0, 20.0, 81).reshape(1, 81, 1)
    zero = np.zeros(1)
    _, alpha0, _ = G.gates(x, np.zeros_like(x), zero, zero)
    np.testing.assert_allclose(alpha0, 1.0 / (1.0 + np.exp(x)), rtol=1e-13)
    _, alpha2, _ = G.gates(x, np.zeros_like(x), np.full(1, math.log(2.0)), zero)
    np.testing.assert_allclose(alpha2, (1.0 / (1.0 + np.exp(x))) ** 2, rtol=1e-13)
    # bias enters inside the softplus: a = 0, b_alpha = ln 3, A = ln 2 -> alpha = 1/16
    g, alpha, _ = G.gates(np.zeros((1, 1, 1)), np.zeros((1, 1, 1)), np.full(1, math.log(2.0)),
                          np.full(1, math.log(3.0)))
    np.testing.assert_allclose(alpha, 1.0 / 16.0, rtol=1e-14)
    np.testing.assert_allclose(g, -math.log(16.0), rtol=1e-14)
    _, alpha, _ = G.gates(np.full((1, 1, 1), -math.log(3.0)), np.zeros((1, 1, 1)), zero, zero)
    np.testing.assert_allclose(alpha, 0.75, rtol=1e-14)


def check_log_decay_asymptotes(G):
    """softplus(x) -> x for large x and -> e^x for very negative x, so
    g = -e^A softplus(x) is -e^A x and -e^A e^x there (relative error below e^-40)."""
    A = np.array([0.3, -1.2])
    x = np.array([40.0, -40.0]).reshape(1, 2, 1) * np.ones((1, 1, 2))
    g, _, _ = G.gates(x, np.zeros_like(x), A, np.zeros(2))
    np.testing.assert_allclose(g[0, 0], -np.exp(A) * 40.0, rtol=1e-15)
    np.testing.assert_allclose(g[0, 1], -np.exp(A) * np.exp(-40.0), rtol=1e-15)


def check_beta_values(G):
    """Eq. (9): sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(x) + sigmoid(-x) = 1."""
    b = np.array([0.0, math.log(3.0), -math.log(3.0)]).reshape(1, 3, 1)
    _, _, beta = G.gates(np.zeros_like(b), b, np.zeros(1), np.zeros(1))
    np.testing.assert_allclose(beta.reshape(-1), [0.5, 0.75, 0.25], rtol=1e-15)
    x = np.linspace(-30.0, 30.0, 61).reshape(1, 61, 1)
    _, _, bp = G.gates(np.zeros_like(x), x, np.zeros(1), np.zeros(1))
    _, _, bm = G.gates(np.zeros_like(x), -x, np.zeros(1), np.zeros(1))
    np.testing.assert_allclose(bp + bm, 1.0, rtol=1e-15)


def check_gated_output_hand(G):
    """Hand-worked values of sigmoid(z) * RMSNorm(y) (derivation in the fixture)."""
    g = _load_golden("gated_output_hand.txt")
    dv = int(g["dv"][0])
    o = G.gated_output(g["y"].reshape(-1, dv), g["z"].reshape(-1, dv), g["w"],
                       eps=float(g["eps"][0]))
    np.testing.assert_allclose(o.reshape(-1), g["o"], rtol=0, atol=1e-15)


def check_rmsnorm_invariants(G):
    """With eps = 0 and w = 0: the output has unit root mean square and does not change
    when y is scaled by c > 0; the gain (1 + w) multiplies column by column."""
    rng = np.random.default_rng(11)
    y = rng.standard_normal((5, 3, 16))
    w = np.zeros(16)
    n = G.rmsnorm(y, w, eps=0.0)
    np.testing.assert_allclose(np.mean(n * n, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(G.rmsnorm(7.5 * y, w, eps=0.0), n, rtol=1e-14)
    w2 = rng.standard_normal(16)
    np.testing.assert_allclose(G.rmsnorm(y, w2, eps=0.0), n * (1.0 + w2), rtol=1e-14)


def _central(f, x, h=1e-6):
    """Central differences of the scalar function f at every element of x (in place)."""
    out = np.zeros_like(x)
    for i in np.ndindex(x.shape):
        old = x[i]
        x[i] = old + h
        fp = f()
        x[i] = old - h
        fm = f()
        x[i] = old
        out[i] = (fp - fm) / (2 * h)
    return out


def check_gates_backward_differences(G):
    """Reverse mode of eqs. (9)-(10) against central differences, with the upstream given
    both as d alpha and as d ln alpha."""
    rng = np.random.default_rng(12)
    a, b = rng.standard_normal((2, 3, 2)), rng.standard_normal((2, 3, 2))
    A, ba = rng.standard_normal(2) * 0.5, rng.standard_normal(2)
    da_up, dg_up, db_up = (rng.standard_normal((2, 3, 2)) for _ in range(3))

    def loss():
        g, alpha, beta = G.gates(a, b, A, ba)
        return np.sum(da_up * alpha) + np.sum(dg_up * g) + np.sum(db_up * beta)

    got = G.gates_backward(a, b, A, ba, dalpha=da_up, dbeta=db_up, dg=dg_up)
    for name, x in (("da", a), ("db", b), ("dA_log", A), ("db_alpha", ba)):
        np.testing.assert_allclose(got[name], _central(loss, x), rtol=1e-6, atol=1e-9,
                                   err_msg=name)


def check_gated_output_backward_differences(G):
    """Reverse mode of sigmoid(z) * RMSNorm(y) against central differences."""
    rng = np.random.default_rng(13)
    y, z, do = (rng.standard_normal((2, 3, 5)) for _ in range(3))
    w = rng.standard_normal(5) * 0.5

    def loss():
        return np.sum(do * G.gated_output(y, z, w))

    got = G.gated_output_backward(y, z, w, do)
    for name, x in (("dy", y), ("dz", z), ("dw", w)):
        np.testing.assert_allclose(got[name], _central(loss, x), rtol=1e-6, atol=1e-9,
                                   err_msg=name)


def check_layer_core_backward_differences(G):
    """The whole chain eqs. (9)-(10) -> (1)-(4) -> (11) against central differences, for
    every input and parameter, with a nonzero initial state and final-state gradient."""
    rng = np.random.default_rng(14)
    B, T, H, dk, dv = 1, 4, 2, 3, 3
    q, k = rng.standard_normal((B, T, H, dk)), rng.standard_normal((B, T, H, dk))
    v, z = rng.standard_normal((B, T, H, dv)), rng.standard_normal((B, T, H, dv))
    a, b = rng.standard_normal((B, T, H)), rng.standard_normal((B, T, H))
    A, ba = rng.standard_normal(H) * 0.5, rng.standard_normal(H)
    w = rng.standard_normal(dv) * 0.3
    s0 = rng.standard_normal((B, H, dk, dv)) * 0.5
    do = rng.standard_normal((B, T, H, dv))
    dsf = rng.standard_normal((B, H, dk, dv))

    def loss():
        o, _, sf = G.layer_core(q, k, v, a, b, z, A, ba, w, s0)
        return np.sum(do * o) + np.sum(dsf * sf)

    got = G.layer_core_backward(q, k, v, a, b, z, A, ba, w, do, s0, ds_final=dsf)
    for name, x in (("dq", q), ("dk", k), ("dv", v), ("dz", z), ("da", a), ("db", b),
                    ("dA_log", A), ("db_alpha", ba), ("dw", w), ("ds0", s0)):
        np.testing.assert_allclose(got[name], _central(loss, x), rtol=1e-6, atol=1e-8,
                                   err_msg=name)


CHECKS = [check_decay_closed_forms, check_log_decay_asymptotes, check_beta_values,
          check_gated_output_hand, check_rmsnorm_invariants, check_gates_backward_differences,
          check_gated_output_backward_differences, check_layer_core_backward_differences]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_gates_oracle(check):
    check(gates_mod)


def test_layer_core_uses_the_recurrence_oracle():
    """layer_core's y is the token-loop oracle's y for the alpha, beta of eqs. (9)-(10)."""
    rng = np.random.default_rng(15)
    q, k, v, z = (rng.standard_normal((2, 9, 2, 4)) for _ in range(4))
    a, b = rng.standard_normal((2, 9, 2)), rng.standard_normal((2, 9, 2))
    A, ba, w = rng.standard_normal(2), rng.standard_normal(2), rng.standard_normal(4)
    _, y, sf = gates_mod.layer_core(q, k, v, a, b, z, A, ba, w)
    alpha = 1.0 / (1.0 + np.exp(a + ba)) ** np.exp(A)      # exp(-e^A softplus(x))
    beta = 1.0 / (1.0 + np.exp(-b))
    y_ref, sf_ref = oracle.forward(q, k, v, alpha, beta)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sf, sf_ref, rtol=1e-12, atol=1e-14)

"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics, not by the
oracle itself.

Equations referenced: Qwen3.8-Flash-Next summary (picx.dev), "Theoretical foundations",
eqs. (1)-(4) (the gated delta rule) and "Methodology" / "1. GDN Hybrid Token Mixing"
(L2-normalised q and k).  Each test names the fact it checks.
"""
import os

import numpy as np
import pytest

import oracle
import oracle.chunked as oracle_chunked

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


def _run_golden(name):
    g = _load_golden(name)
    dk, dv, T = int(g["dk"][0]), int(g["dv"][0]), int(g["T"][0])
    eps = float(g["eps"][0]) if "eps" in g else oracle.EPS
    l2 = "eps" in g
    s0 = g["s0"].reshape(1, 1, dk, dv) if "s0" in g else None
    y, sf = oracle.forward(g["q"].reshape(1, T, 1, dk), g["k"].reshape(1, T, 1, dk),
                           g["v"].reshape(1, T, 1, dv), g["alpha"].reshape(1, T, 1),
                           g["beta"].reshape(1, T, 1), s0, l2norm=l2, eps=eps)
    return g, y.reshape(-1), sf.reshape(-1)


@pytest.mark.parametrize("name", ["scalar_three_tokens.txt", "two_by_three.txt",
                                  "l2norm_one_token.txt"])
def test_hand_worked_examples(name):
    """Hand-computed values of eqs. (1)-(4) (derivations in the fixture files)."""
    g, y, sf = _run_golden(name)
    np.testing.assert_allclose(y, g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(sf, g["s_final"], rtol=0, atol=1e-14)



def test_hand_worked_backward():
    """Hand-computed gradients of eqs. (1)-(4) for dk = dv = 1 (scalar chain rule; the
    derivation is in the fixture), compared with the oracle's reverse recurrence."""
    g = _load_golden("scalar_three_tokens_backward.txt")
    T = int(g["T"][0])
    sh = (1, T, 1, 1)
    args = (g["q"].reshape(sh), g["k"].reshape(sh), g["v"].reshape(sh),
            g["alpha"].reshape(1, T, 1), g["beta"].reshape(1, T, 1))
    s0 = g["s0"].reshape(1, 1, 1, 1)
    y, sf = oracle.forward(*args, s0, l2norm=False)
    np.testing.assert_allclose(y.reshape(-1), g["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(sf.reshape(-1), g["s_final"], rtol=0, atol=1e-14)
    out = oracle.backward(*args, s0, dy=g["dy"].reshape(sh),
                          ds_final=g["ds_final"].reshape(1, 1, 1, 1), l2norm=False)
    for name, key in (("dq", "dq"), ("dk", "dk_grad"), ("dv", "dv_grad"),
                      ("dalpha", "dalpha"), ("dbeta", "dbeta"), ("ds0", "ds0")):
        np.testing.assert_allclose(out[name].reshape(-1), g[key], rtol=0, atol=1e-14,
                                   err_msg=name)

def _rand(rng, B, T, H, dk, dv, s0=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.05, 0.999, (B, T, H))
    beta = rng.uniform(0.01, 0.99, (B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3 if s0 else None
    return q, k, v, alpha, beta, S0


def _l2n(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + oracle.EPS)


def test_l2norm_unit_rows():
    """With eps -> 0 the normalised key has unit length: with beta=1, S0=0, one token,
    S = k_hat v^T, so |S[:, j]| = |v_j| for every column."""
    rng = np.random.default_rng(1)
    q, k, v, _, _, _ = _rand(rng, 1, 1, 1, 8, 5)
    _, sf = oracle.forward(q, k, v, np.ones((1, 1, 1)), np.ones((1, 1, 1)), eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(sf[0, 0], axis=0), np.abs(v[0, 0, 0]),
                               rtol=1e-14)


def test_alpha1_beta0_is_identity():
    """alpha=1, beta=0 leaves S unchanged and y_t = S0^T q_hat_t."""
    rng = np.random.default_rng(2)
    q, k, v, _, _, S0 = _rand(rng, 2, 7, 3, 6, 5)
    ones, zeros = np.ones((2, 7, 3)), np.zeros((2, 7, 3))
    y, sf = oracle.forward(q, k, v, ones, zeros, S0)
    np.testing.assert_allclose(sf, S0, rtol=0, atol=1e-15)
    expect = np.einsum("bhkv,bthk->bthv", S0, _l2n(q))
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-14)


def test_one_token_outer_product():
    """alpha=1, beta=1, S0=0, one token: S = k_hat v^T and y = (k_hat . q_hat) v."""
    rng = np.random.default_rng(3)
    q, k, v, _, _, _ = _rand(rng, 1, 1, 2, 7, 4)
    y, sf = oracle.forward(q, k, v, np.ones((1, 1, 2)), np.ones((1, 1, 2)))
    kh, qh = _l2n(k)[0, 0], _l2n(q)[0, 0]
    for h in range(2):
        np.testing.assert_allclose(sf[0, h], np.outer(kh[h], v[0, 0, h]), rtol=1e-13)
        np.testing.assert_allclose(y[0, 0, h], (kh[h] @ qh[h]) * v[0, 0, h], rtol=1e-13)


def test_beta1_unit_key_writes_exactly():
    """beta=1 with a unit key: after token t, S_t^T k_hat_t = v_t exactly (any alpha, S0)."""
    rng = np.random.default_rng(4)
    T, dk, dv = 6, 5, 3
    q, k, v, alpha, _, S0 = _rand(rng, 1, T, 1, dk, dv)
    beta = np.ones((1, T, 1))
    kh = _l2n(k) if False else k / np.linalg.norm(k, axis=-1, keepdims=True)
    for t in range(1, T + 1):
        _, sf = oracle.forward(q[:, :t], k[:, :t], v[:, :t], alpha[:, :t], beta[:, :t], S0,
                               eps=0.0)
        np.testing.assert_allclose(sf[0, 0].T @ kh[0, t - 1, 0], v[0, t - 1, 0], rtol=1e-12,
                                   atol=1e-13)


def test_beta0_closed_form():
    """beta=0: S_t = (prod_{s<=t} alpha_s) S0 and y_t = prod(alpha) S0^T q_hat_t."""
    rng = np.random.default_rng(5)
    q, k, v, alpha, _, S0 = _rand(rng, 1, 9, 2, 4, 6)
    y, sf = oracle.forward(q, k, v, alpha, np.zeros_like(alpha), S0)
    cum = np.cumprod(alpha, axis=1)  # [1,T,H]
    np.testing.assert_allclose(sf[0], cum[0, -1][:, None, None] * S0[0], rtol=1e-12)
    expect = cum[..., None] * np.einsum("bhkv,bthk->bthv", S0, _l2n(q))
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-15)


def test_orthonormal_keys_exact_retrieval():
    """alpha=beta=1, S0=0, orthonormal keys k_1..k_n (n <= dk): S_n^T k_j = v_j for all j."""
    rng = np.random.default_rng(6)
    dk, dv, n = 8, 5, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T.reshape(1, n, 1, dk)
    v = rng.standard_normal((1, n, 1, dv))
    q = rng.standard_normal((1, n, 1, dk))
    _, sf = oracle.forward(q, keys, v, np.ones((1, n, 1)), np.ones((1, n, 1)), eps=0.0)
    np.testing.assert_allclose(keys[0, :, 0] @ sf[0, 0], v[0, :, 0], rtol=1e-12, atol=1e-13)


def test_homogeneity_in_v_and_s0():
    """The recurrence is linear in (v, S0) jointly: scaling both by c scales y and S by c."""
    rng = np.random.default_rng(7)
    q, k, v, alpha, beta, S0 = _rand(rng, 1, 12, 2, 5, 4)
    y1, s1 = oracle.forward(q, k, v, alpha, beta, S0)
    y2, s2 = oracle.forward(q, k, -2.5 * v, alpha, beta, -2.5 * S0)
    np.testing.assert_allclose(y2, -2.5 * y1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(s2, -2.5 * s1, rtol=1e-12, atol=1e-14)


def test_columns_of_state_are_independent():
    """Column j of S only sees column j of v and S0: splitting dv in two halves reproduces
    the full result."""
    rng = np.random.default_rng(8)
    q, k, v, alpha, beta, S0 = _rand(rng, 2, 10, 2, 6, 8)
    y, sf = oracle.forward(q, k, v, alpha, beta, S0)
    ya, sa = oracle.forward(q, k, v[..., :3], alpha, beta, S0[..., :3])
    yb, sb = oracle.forward(q, k, v[..., 3:], alpha, beta, S0[..., 3:])
    np.testing.assert_allclose(np.concatenate([ya, yb], -1), y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(np.concatenate([sa, sb], -1), sf, rtol=1e-13, atol=1e-15)


def test_resume_from_final_state():
    """prefill(T1) then prefill(T2, S0 = S_T1) equals prefill(T1 + T2)."""
    rng = np.random.default_rng(9)
    q, k, v, alpha, beta, S0 = _rand(rng, 1, 20, 2, 5, 4)
    y, sf = oracle.forward(q, k, v, alpha, beta, S0)
    y1, s1 = oracle.forward(q[:, :7], k[:, :7], v[:, :7], alpha[:, :7], beta[:, :7], S0)
    y2, s2 = oracle.forward(q[:, 7:], k[:, 7:], v[:, 7:], alpha[:, 7:], beta[:, 7:], s1)
    np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s2, sf, rtol=1e-13, atol=1e-15)


def test_decode_steps_equal_prefill():
    """T one-token decode steps equal one prefill of T tokens."""
    rng = np.random.default_rng(10)
    q, k, v, alpha, beta, S0 = _rand(rng, 3, 5, 2, 4, 6)
    y, sf = oracle.forward(q, k, v, alpha, beta, S0)
    st = S0
    for t in range(5):
        yt, st = oracle.decode_step(q[:, t], k[:, t], v[:, t], alpha[:, t], beta[:, t], st)
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(st, sf, rtol=1e-13, atol=1e-15)


def test_varlen_equals_separate_calls():
    """Packed documents restart from their own S0 at each cu_seqlens boundary."""
    rng = np.random.default_rng(11)
    lens = [5, 1, 9, 4]
    T = sum(lens)
    q, k, v, alpha, beta, _ = _rand(rng, 1, T, 2, 4, 3, s0=False)
    S0 = rng.standard_normal((4, 2, 4, 3))
    cu = np.concatenate([[0], np.cumsum(lens)])
    y, sf = oracle.forward_varlen(q, k, v, alpha, beta, cu, S0)
    for n in range(4):
        a, b = cu[n], cu[n + 1]
        yn, sn = oracle.forward(q[:, a:b], k[:, a:b], v[:, a:b], alpha[:, a:b], beta[:, a:b],
                                S0[n:n + 1])
        np.testing.assert_allclose(y[:, a:b], yn, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(sf[n:n + 1], sn, rtol=1e-14, atol=1e-15)


def test_frobenius_norm_bound():
    """|I - beta k k^T|_2 <= 1 for unit k and beta in [0,1], so
    |S_t|_F <= alpha_t |S_{t-1}|_F + beta_t |v_t|."""
    rng = np.random.default_rng(12)
    T = 12
    q, k, v, alpha, beta, S0 = _rand(rng, 1, T, 1, 6, 4)
    prev = S0[0, 0]
    for t in range(1, T + 1):
        _, sf = oracle.forward(q[:, :t], k[:, :t], v[:, :t], alpha[:, :t], beta[:, :t], S0,
                               eps=0.0)
        cur = sf[0, 0]
        bound = alpha[0, t - 1, 0] * np.linalg.norm(prev) + beta[0, t - 1, 0] * np.linalg.norm(
            v[0, t - 1, 0])
        assert np.linalg.norm(cur) <= bound * (1 + 1e-12)
        prev = cur


def test_scale_multiplies_y_only():
    rng = np.random.default_rng(13)
    q, k, v, alpha, beta, S0 = _rand(rng, 1, 6, 1, 4, 4)
    y1, s1 = oracle.forward(q, k, v, alpha, beta, S0)
    y2, s2 = oracle.forward(q, k, v, alpha, beta, S0, scale=0.125)
    np.testing.assert_allclose(y2, 0.125 * y1, rtol=1e-14)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=0)


@pytest.mark.parametrize("C", [1, 16, 64])
@pytest.mark.parametrize("l2norm", [True, False])
def test_chunked_form_matches_token_loop(C, l2norm, chunked=None):
    """The chunked WY/UT form and the token-by-token form agree (T not a multiple of C).
    ``chunked`` replaces ``oracle.chunked`` (the mutation check passes a planted copy)."""
    forward_chunked = (chunked or oracle_chunked).forward_chunked
    rng = np.random.default_rng(14)
    q, k, v, alpha, beta, S0 = _rand(rng, 2, 150, 2, 16, 24)
    if not l2norm:
        q, k = _l2n(q), _l2n(k)
    y, sf = oracle.forward(q, k, v, alpha, beta, S0, l2norm=l2norm)
    yc, sc = forward_chunked(q, k, v, alpha, beta, S0, C=C, l2norm=l2norm)
    np.testing.assert_allclose(yc, y, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sc, sf, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("n", [64, 50, 16, 1])
def test_blocked_inverse_matches_dense_inverse(n, chunked=None):
    """The 16 x 16 blocked inversion of the unit lower-triangular I + A that the kernels use
    (diagonal blocks by substitution, off-diagonal blocks by distance) equals the dense inverse,
    for A of the method's form strictLower(diag(beta) (K K^T * Gam))."""
    inv = (chunked or oracle_chunked).blocked_unit_lower_inverse
    rng = np.random.default_rng(19 + n)
    K = _l2n(rng.standard_normal((n, 8)))
    beta = rng.uniform(0.05, 0.95, n)
    G = np.cumsum(np.log(rng.uniform(0.5, 0.999, n)))
    Gam = np.exp(np.minimum(G[:, None] - G[None, :], 0.0))
    A = np.tril(beta[:, None] * (K @ K.T) * Gam, k=-1)
    ref = np.linalg.inv(np.eye(n) + A)
    np.testing.assert_allclose(inv(A), ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("unroll", [False, True])
def test_coupled_chunk_form_matches_token_loop(unroll, chunked=None):
    """The coupled form the CUDA prefill's sequential kernel runs (U_c from U_{c-1} and a state
    one chunk back through X_c = -W_c K_{c-1}^T), and its two-chunk unrolling, agree with the
    token-by-token form (T not a multiple of C, nonzero S0, a scale)."""
    fc = (chunked or oracle_chunked).forward_chunked_coupled
    rng = np.random.default_rng(17)
    q, k, v, alpha, beta, S0 = _rand(rng, 2, 330, 2, 16, 12)
    slow = rng.uniform(0.9, 0.999, alpha.shape)  # chunk decays near 1: every coupling term counts
    for a in (alpha, slow):
        y, sf = oracle.forward(q, k, v, a, beta, S0, scale=0.8)
        yc, sc = fc(q, k, v, a, beta, S0, C=32, scale=0.8, unroll=unroll)
        np.testing.assert_allclose(yc, y, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(sc, sf, rtol=1e-9, atol=1e-11)


def test_lag2_coupled_chunk_form_matches_token_loop(chunked=None):
    """The coupled form with the state product two chunks behind (the extra coupling X2_c =
    -W_c K_{c-2}^T) agrees with the token-by-token form, at the benchmark's decays and at decays
    near 1 where every coupling term counts."""
    fc = (chunked or oracle_chunked).forward_chunked_coupled
    rng = np.random.default_rng(19)
    q, k, v, alpha, beta, S0 = _rand(rng, 2, 330, 2, 16, 12)
    slow = rng.uniform(0.9, 0.999, alpha.shape)
    for a in (alpha, slow):
        y, sf = oracle.forward(q, k, v, a, beta, S0, scale=0.8)
        yc, sc = fc(q, k, v, a, beta, S0, C=32, scale=0.8, lag2=True)
        np.testing.assert_allclose(yc, y, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(sc, sf, rtol=1e-9, atol=1e-11)


def test_chunked_form_small_alpha_no_overflow(chunked=None):
    """Cumulative log-decay far below -88 within a chunk (exp(-G) alone would overflow
    fp64 only much later, but the relative form must stay finite and exact)."""
    forward_chunked = (chunked or oracle_chunked).forward_chunked
    rng = np.random.default_rng(15)
    q, k, v, _, beta, S0 = _rand(rng, 1, 70, 1, 8, 8)
    alpha = np.full((1, 70, 1), 1e-8)
    y, sf = oracle.forward(q, k, v, alpha, beta, S0)
    yc, sc = forward_chunked(q, k, v, alpha, beta, S0, C=64)
    assert np.all(np.isfinite(yc)) and np.all(np.isfinite(sc))
    np.testing.assert_allclose(yc, y, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("C", [16, 64])
@pytest.mark.parametrize("l2norm", [True, False])
def test_chunked_backward_matches_reverse_recurrence(C, l2norm, chunked=None):
    """The chunked backward (the forward chain transposed plus chunk-local gradients, the form the
    CUDA backward runs) agrees with the token-by-token reverse recurrence: dk != dv, T not a
    multiple of C, a nonzero dS_final and a scale."""
    backward_chunked = (chunked or oracle_chunked).backward_chunked
    rng = np.random.default_rng(16)
    q, k, v, alpha, beta, S0 = _rand(rng, 2, 150, 2, 16, 24)
    if not l2norm:
        q, k = _l2n(q), _l2n(k)
    dy = rng.standard_normal((2, 150, 2, 24))
    dsf = rng.standard_normal((2, 2, 16, 24))
    ref = oracle.backward(q, k, v, alpha, beta, s0=S0, dy=dy, ds_final=dsf, scale=0.7, l2norm=l2norm)
    got = backward_chunked(q, k, v, alpha, beta, s0=S0, dy=dy, ds_final=dsf, C=C, scale=0.7,
                           l2norm=l2norm)
    for name in ("dq", "dk", "dv", "dalpha", "dbeta", "ds0"):
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-11, err_msg=name)


# ------------------------------------------------------------------ backward pins

def _loss(inputs, dy, dsf, l2norm, scale):
    q, k, v, alpha, beta, S0 = inputs
    y, sf = oracle.forward(q, k, v, alpha, beta, S0, l2norm=l2norm, scale=scale)
    return float(np.sum(y * dy) + np.sum(sf * dsf))


@pytest.mark.parametrize("l2norm", [True, False])
def test_backward_matches_central_differences(l2norm):
    """Every gradient of L = <dy, y> + <dS_final, S_T> against central differences
    (step 1e-6, fp64) at B=1, H=1, T=8, dk=4, dv=3."""
    rng = np.random.default_rng(16)
    B, T, H, dk, dv = 1, 8, 1, 4, 3
    inputs = list(_rand(rng, B, T, H, dk, dv))
    dy = rng.standard_normal((B, T, H, dv))
    dsf = rng.standard_normal((B, H, dk, dv))
    scale = 0.7
    g = oracle.backward(*inputs, dy=dy, ds_final=dsf, l2norm=l2norm, scale=scale)
    names = ["dq", "dk", "dv", "dalpha", "dbeta", "ds0"]
    h = 1e-6
    for idx, name in enumerate(names):
        x = inputs[idx]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            old = x[mi]
            x[mi] = old + h
            lp = _loss(inputs, dy, dsf, l2norm, scale)
            x[mi] = old - h
            lm = _loss(inputs, dy, dsf, l2norm, scale)
            x[mi] = old
            num[mi] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_adjoint_identity():
    """<grad, delta> equals the directional derivative for a random delta over all inputs
    at once (larger size than the per-element check)."""
    rng = np.random.default_rng(17)
    B, T, H, dk, dv = 2, 70, 2, 6, 5
    inputs = list(_rand(rng, B, T, H, dk, dv))
    dy = rng.standard_normal((B, T, H, dv))
    dsf = rng.standard_normal((B, H, dk, dv))
    g = oracle.backward(*inputs, dy=dy, ds_final=dsf)
    deltas = [rng.standard_normal(x.shape) for x in inputs]
    deltas[3] *= 0.01  # keep alpha, beta inside (0, 1)
    deltas[4] *= 0.01
    h = 1e-5
    plus = [x + h * d for x, d in zip(inputs, deltas)]
    minus = [x - h * d for x, d in zip(inputs, deltas)]
    num = (_loss(plus, dy, dsf, True, 1.0) - _loss(minus, dy, dsf, True, 1.0)) / (2 * h)
    ana = sum(float(np.sum(g[n] * d)) for n, d in
              zip(["dq", "dk", "dv", "dalpha", "dbeta", "ds0"], deltas))
    assert abs(ana - num) <= 1e-7 * max(1.0, abs(num))


def test_backward_without_upstream_state_grad():
    """ds_final = None is the same as ds_final = 0; dy = 0 with ds_final = 0 gives zeros."""
    rng = np.random.default_rng(18)
    inputs = list(_rand(rng, 1, 9, 1, 4, 4))
    dy = rng.standard_normal((1, 9, 1, 4))
    g1 = oracle.backward(*inputs, dy=dy)
    g2 = oracle.backward(*inputs, dy=dy, ds_final=np.zeros((1, 1, 4, 4)))
    for n in g1:
        np.testing.assert_array_equal(g1[n], g2[n])
    g0 = oracle.backward(*inputs, dy=np.zeros_like(dy))
    for n in g0:
        assert not np.any(g0[n])

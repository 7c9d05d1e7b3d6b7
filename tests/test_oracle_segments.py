"""Pins for the segment form of the recurrence (``oracle/segments.py``): affine maps of runs of
tokens, their composition and scan.  Facts fixed by eqs. (1)-(4) of the Qwen3.8-Flash-Next
summary (picx.dev, "Theoretical foundations"); each check takes the module under test so that
``test_oracle_mutants`` can run it against a copy with a planted mistake.
"""
import numpy as np
import pytest

import oracle
import oracle.segments as seg_mod


def _rand(rng, B, T, H, dk, dv):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(0.05, 0.999, (B, T, H))
    beta = rng.uniform(0.01, 0.99, (B, T, H))
    s0 = rng.standard_normal((B, H, dk, dv)) * 0.3
    return q, k, v, alpha, beta, s0


def check_segmented_equals_token_loop(S):
    """Cutting a sequence into segments (maps, scan, then each segment from its start state)
    gives the token loop's outputs and final state, for any cut, empty segments included."""
    rng = np.random.default_rng(21)
    q, k, v, alpha, beta, s0 = _rand(rng, 2, 37, 2, 5, 4)
    yr, sr = oracle.forward(q, k, v, alpha, beta, s0, scale=0.7)
    for bounds in ([0, 37], [0, 18, 37], [0, 1, 2, 20, 36, 37], [0, 0, 10, 10, 37, 37]):
        y, sf = S.forward_segmented(q, k, v, alpha, beta, bounds, s0=s0, scale=0.7)
        np.testing.assert_allclose(y, yr, rtol=1e-10, atol=1e-12, err_msg=str(bounds))
        np.testing.assert_allclose(sf, sr, rtol=1e-10, atol=1e-12, err_msg=str(bounds))


def check_map_is_the_affine_action(S):
    """A segment's map applied to any start state equals the token loop run from that state:
    S_end = M S0 + N (the map does not depend on S0)."""
    rng = np.random.default_rng(22)
    _, k, v, alpha, beta, _ = _rand(rng, 1, 29, 1, 6, 3)
    m = S.segment_map(k[0, :, 0], v[0, :, 0], alpha[0, :, 0], beta[0, :, 0])
    for trial in range(3):
        S0 = rng.standard_normal((1, 1, 6, 3))
        _, sf = oracle.forward(k, k, v, alpha, beta, S0)  # q is irrelevant to the state
        np.testing.assert_allclose(S.apply(m, S0[0, 0]), sf[0, 0], rtol=1e-11, atol=1e-12)


def check_closed_forms(S):
    """beta = 0: M = (prod alpha) I, N = 0.  alpha = beta = 1 with orthonormal keys (eqs.
    (1)-(3) with unit keys): M = I - sum kh kh^T and N = sum kh v^T."""
    rng = np.random.default_rng(23)
    k = rng.standard_normal((9, 4))
    v = rng.standard_normal((9, 3))
    a = rng.uniform(0.3, 0.99, 9)
    M, N = S.segment_map(k, v, a, np.zeros(9))
    np.testing.assert_allclose(M, np.prod(a) * np.eye(4), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(N, 0.0, atol=1e-15)
    Qm, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    ko = Qm[:, :4].T                                    # 4 orthonormal keys in R^6
    vo = rng.standard_normal((4, 5))
    M, N = S.segment_map(ko, vo, np.ones(4), np.ones(4), l2norm=False)
    np.testing.assert_allclose(M, np.eye(6) - ko.T @ ko, atol=1e-13)
    np.testing.assert_allclose(N, ko.T @ vo, atol=1e-13)


def check_single_token_spectrum(S):
    """One token's M = alpha (I - beta kh kh^T): kh is an eigenvector with eigenvalue
    alpha (1 - beta); every vector orthogonal to kh is scaled by alpha."""
    rng = np.random.default_rng(24)
    k = rng.standard_normal(5)
    kh = k / np.linalg.norm(k)
    M, N = S.token_map(k, rng.standard_normal(2), 0.8, 0.3, eps=0.0)
    np.testing.assert_allclose(M @ kh, 0.8 * 0.7 * kh, atol=1e-14)
    u = rng.standard_normal(5)
    u -= kh * (kh @ u)
    np.testing.assert_allclose(M @ u, 0.8 * u, atol=1e-14)
    # N writes only along kh: its columns lie in span(kh)
    np.testing.assert_allclose(N - np.outer(kh, kh @ N), 0.0, atol=1e-14)
    assert np.linalg.matrix_rank(N) == 1


def check_composition_is_associative(S):
    rng = np.random.default_rng(25)
    maps = [(rng.standard_normal((4, 4)), rng.standard_normal((4, 3))) for _ in range(3)]
    left = S.compose(maps[2], S.compose(maps[1], maps[0]))
    right = S.compose(S.compose(maps[2], maps[1]), maps[0])
    for x, y in zip(left, right):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-12)
    # composition order: applying the composite equals applying earlier, then later
    S0 = rng.standard_normal((4, 3))
    np.testing.assert_allclose(S.apply(S.compose(maps[1], maps[0]), S0),
                               S.apply(maps[1], S.apply(maps[0], S0)), rtol=1e-12, atol=1e-12)


def check_chunked_map_matches_token_product(S):
    """The map from the chunked WY quantities equals the product of the token maps, for chunk
    lengths that divide the run and ones that leave a ragged last chunk."""
    rng = np.random.default_rng(26)
    _, k, v, alpha, beta, _ = _rand(rng, 1, 70, 1, 8, 5)
    ref = S.segment_map(k[0, :, 0], v[0, :, 0], alpha[0, :, 0], beta[0, :, 0])
    for C in (1, 16, 64, 70):
        got = S.segment_map_chunked(k[0, :, 0], v[0, :, 0], alpha[0, :, 0], beta[0, :, 0], C=C)
        for x, y in zip(got, ref):
            np.testing.assert_allclose(x, y, rtol=1e-10, atol=1e-12, err_msg=f"C={C}")


CHECKS = [check_segmented_equals_token_loop, check_map_is_the_affine_action, check_closed_forms,
          check_single_token_spectrum, check_composition_is_associative,
          check_chunked_map_matches_token_product]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_segments_oracle(check):
    check(seg_mod)

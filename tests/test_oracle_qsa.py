"""Pins for the fp64 oracle of the QSA block indexer (``oracle/qsa_indexer.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "2. Qwen Sparse Attention (QSA)",
eq. (13).  Each check takes the module under test, so that the mutation tests can run the
same checks against a copy with a planted mistake.
"""
import os

import numpy as np
import pytest

import oracle.qsa_indexer as qsa_mod

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


def _rand(seed, lengths, d=16, hq=4):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    return (rng.standard_normal((T, hq, d)), rng.standard_normal((T, d)),
            1.0 + 0.1 * rng.standard_normal(d), np.concatenate([[0], np.cumsum(lengths)]))


# --------------------------------------------------------------------------- checks


def check_hand_example(M):
    """One document worked by hand (tests/golden/qsa_indexer_hand.txt): pooled keys, the
    block-causal visibility, ReLU, the head sum, the budget and the tie-break."""
    g = _load_golden("qsa_indexer_hand.txt")
    d, r, budget = int(g["d"][0]), int(g["r"][0]), int(g["budget"][0])
    k = g["k"].reshape(-1, d)
    T = k.shape[0]
    q = g["q"].reshape(T, 2, d)
    kh, base, sc, sel = M.indexer(q, k, g["g"], [0, T], budget=budget, r=r, eps=0.0)
    np.testing.assert_array_equal(kh, g["khat"].reshape(-1, d))
    np.testing.assert_array_equal(base, [0, 3])
    assert [len(s) for s in sc] == list(g["nvis"].astype(int))
    np.testing.assert_array_equal(np.concatenate(sc), g["scores"])
    np.testing.assert_array_equal(sel, g["sel"].reshape(T, budget).astype(int))


def check_varlen_equals_separate(M):
    """Packed documents equal separate calls: blocks restart at every document."""
    lengths = [9, 0, 4, 3, 17]
    q, k, g, cu = _rand(1, lengths)
    kh, base, sc, sel = M.indexer(q, k, g, cu, budget=3)
    assert list(np.diff(base)) == [n // 4 for n in lengths]
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        khn, _, scn, seln = M.indexer(q[a:b], k[a:b], g, [0, b - a], budget=3)
        np.testing.assert_allclose(kh[base[n]:base[n + 1]], khn, rtol=1e-14)
        for s1, s2 in zip(sc[a:b], scn):
            np.testing.assert_allclose(s1, s2, rtol=1e-14)
        np.testing.assert_array_equal(sel[a:b], seln)


def check_pooled_keys_unit_rms(M):
    """Every pooled key, divided by the gain, has unit RMS (eps = 0), and is the normalised
    mean of its r rows."""
    q, k, g, cu = _rand(2, [50])
    kh, base, _, _ = M.indexer(q, k, g, cu, eps=0.0)
    x = kh / g
    np.testing.assert_allclose(np.sqrt(np.mean(x * x, axis=1)), 1.0, rtol=1e-13)
    m = k[:48].reshape(12, 4, -1).mean(axis=1)
    np.testing.assert_allclose(x, m / np.sqrt(np.mean(m * m, axis=1, keepdims=True)), rtol=1e-13)


def check_selection_is_top_set(M):
    """The selection holds min(budget, visible) blocks, sorted and padded with -1, and every
    selected block scores at least as high as every unselected visible one (lexsort as the
    independent ranking)."""
    q, k, g, cu = _rand(3, [203])
    for budget in (1, 5, 50, 60):
        _, _, sc, sel = M.indexer(q, k, g, cu, budget=budget)
        for s, row in zip(sc, sel):
            n = min(budget, len(s))
            chosen = row[:n]
            assert np.all(row[n:] == -1) and np.all(np.diff(chosen) > 0)
            ref = np.sort(np.lexsort((np.arange(len(s)), -s))[:n])
            np.testing.assert_array_equal(chosen, ref)


def check_positive_scaling(M):
    """ReLU is positively homogeneous: scaling every query by c > 0 scales the scores by c and
    keeps the selection."""
    q, k, g, cu = _rand(4, [77, 40])
    _, _, sc, sel = M.indexer(q, k, g, cu, budget=4)
    _, _, sc2, sel2 = M.indexer(3.0 * q, k, g, cu, budget=4)
    for a, b in zip(sc, sc2):
        np.testing.assert_allclose(b, 3.0 * a, rtol=1e-13)
    np.testing.assert_array_equal(sel, sel2)


def check_scores_against_einsum(M):
    """Scores of one document against numpy's einsum over all (token, head, block) triples, the
    causal mask applied afterwards."""
    q, k, g, cu = _rand(5, [33])
    kh, _, sc, _ = M.indexer(q, k, g, cu)
    full = np.maximum(np.einsum("thd,bd->tbh", q, kh), 0.0).sum(axis=2)
    for i, s in enumerate(sc):
        nv = (i + 1) // 4
        np.testing.assert_allclose(s, full[i, :nv], rtol=1e-13, atol=1e-13)


CHECKS = [check_hand_example, check_varlen_equals_separate, check_pooled_keys_unit_rms,
          check_selection_is_top_set, check_positive_scaling, check_scores_against_einsum]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_qsa_oracle(check):
    check(qsa_mod)

"""fp64 oracle of the QSA block indexer.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "2. Qwen Sparse Attention
(QSA)", eq. (13), and the bud-325 wiki entry ("Key claims": 4 indexer query heads,
1 shared key head, head dim 128; a budget of 512 blocks or 2048 tokens):

* keys are cut into blocks of r = 4 tokens and each block is compressed to
      k^_b = RMSNorm(AvgPool(k_{p_b .. p_b + r - 1})),  0 <= b < floor(n / r);
* a query scores every block by the ReLU of its query-key similarity, summed over
  the indexer's query heads:  I[t, b] = sum_h ReLU(q[t, h] . k^_b);
* block-causal masking, and up to 512 complete blocks are selected per query.

Readings where the pages are silent:

* RMSNorm(x) = g * x / sqrt(mean(x^2) + eps) with a per-channel gain g, eps = 1e-6;
* packed documents are independent: a document's blocks start at its first token,
  and a trailing partial block (fewer than r tokens) is never scored;
* block b of a document is visible to the query at position i of that document iff
  the block is complete at or before it: r (b + 1) - 1 <= i (the block holding i is
  visible only once i is its last token);
* the selection is the min(budget, visible) blocks of highest score, ties broken
  towards the lower block index; it is returned sorted by block index and padded
  with -1 to the budget.

Everything is evaluated in float64, as written above.
"""
from __future__ import annotations

import numpy as np

R_BLOCK = 4
EPS_NORM = 1e-6


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rmsnorm(x, g, eps=EPS_NORM):
    x = _f64(x)
    return _f64(g) * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def pooled_keys(k, g, cu_seqlens, r=R_BLOCK, eps=EPS_NORM):
    """k [T, d] -> (k_hat [NB, d], block_base [N+1]): the compressed blocks of every document,
    packed document after document (document n owns rows block_base[n] .. block_base[n+1]-1)."""
    k = _f64(k)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    rows, base = [], [0]
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        nb = (b - a) // r
        for j in range(nb):
            rows.append(np.mean(k[a + r * j:a + r * (j + 1)], axis=0))
        base.append(base[-1] + nb)
    kh = rmsnorm(np.array(rows).reshape(-1, k.shape[1]), g, eps) if rows else np.zeros((0, k.shape[1]))
    return kh, np.array(base)


def block_scores(q, k_hat, block_base, cu_seqlens, r=R_BLOCK):
    """q [T, Hq, d].  Returns a list over tokens of the visible blocks' scores (document-local
    block order): I[t, b] = sum_h ReLU(q[t, h] . k_hat[b])."""
    q = _f64(q)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    out = []
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        kd = k_hat[block_base[n]:block_base[n + 1]]
        for i in range(b - a):
            nvis = (i + 1) // r
            sim = q[a + i] @ kd[:nvis].T          # [Hq, nvis]
            out.append(np.maximum(sim, 0.0).sum(axis=0))
    return out


def select_blocks(scores, budget=512):
    """Indices of the min(budget, len) highest scores, ties to the lower index, sorted
    ascending and padded with -1 to ``budget``."""
    s = np.asarray(scores, dtype=np.float64)
    order = sorted(range(len(s)), key=lambda b: (-s[b], b))[:budget]
    sel = sorted(order)
    return np.array(sel + [-1] * (budget - len(sel)), dtype=np.int64)


def indexer(q, k, g, cu_seqlens, budget=512, r=R_BLOCK, eps=EPS_NORM):
    """The whole indexer: returns (k_hat, block_base, scores per token, selection [T, budget])."""
    kh, base = pooled_keys(k, g, cu_seqlens, r, eps)
    sc = block_scores(q, kh, base, cu_seqlens, r)
    sel = np.stack([select_blocks(s, budget) for s in sc]) if sc else np.zeros((0, budget), np.int64)
    return kh, base, sc, sel

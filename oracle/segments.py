"""fp64 oracle of the segment form of the recurrence: affine maps of runs of tokens.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

From eqs. (1)-(3) of the Qwen3.8-Flash-Next summary (picx.dev, "Theoretical foundations"), one
token acts on the state as an affine map (kh the L2-normalised key):

    S_t = alpha_t (I - beta_t kh_t kh_t^T) S_{t-1} + beta_t kh_t v_t^T  =  M_t S_{t-1} + N_t.

A run of tokens therefore acts as the composition of its tokens' maps,

    (M2, N2) o (M1, N1) = (M2 M1, M2 N1 + N2),

and a sequence cut into segments can be run in three steps: the map of every segment from its
own tokens alone (no state needed), an exclusive scan of the maps from S0 that gives every
segment's start state, and every segment's outputs (eq. (4)) from its start state, again
independently of the other segments.  The pages do not describe this; it follows from eqs.
(1)-(4) and is exact up to rounding.  It is the one exchange that splitting a single sequence
across processors needs: a dk x (dk + dv) map per segment.

Two routes to a segment's map live here: ``segment_map`` composes the token maps one by one
(the definition), and ``segment_map_chunked`` builds each chunk's map from the chunked WY
quantities of ``oracle/chunked.py``'s derivation,

    M_c = gamma_n I - (diag(gamma_n / gamma) Kh)^T W,   N_c = (diag(gamma_n / gamma) Kh)^T Ut,

then composes the chunks; the tests hold the two to each other.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

EPS = 1e-6


def _l2n(x, eps, on):
    if not on:
        return x
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def identity_map(dk, dv):
    return np.eye(dk), np.zeros((dk, dv))


def token_map(k_t, v_t, alpha_t, beta_t, l2norm=True, eps=EPS):
    """(M_t, N_t) of one token: M = alpha (I - beta kh kh^T), N = beta kh v^T."""
    kh = _l2n(np.asarray(k_t, dtype=np.float64), eps, l2norm)
    v_t = np.asarray(v_t, dtype=np.float64)
    M = alpha_t * (np.eye(kh.shape[0]) - beta_t * np.outer(kh, kh))
    N = beta_t * np.outer(kh, v_t)
    return M, N


def compose(later, earlier):
    """The map of `earlier` followed by `later`."""
    M2, N2 = later
    M1, N1 = earlier
    return M2 @ M1, M2 @ N1 + N2


def apply(m, S):
    M, N = m
    return M @ S + N


def segment_map(k, v, alpha, beta, l2norm=True, eps=EPS):
    """Map of one (sequence, head) run: k [n,dk], v [n,dv], alpha, beta [n]; composes the token
    maps in order (n = 0 gives the identity)."""
    k, v = np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64)
    m = identity_map(k.shape[1], v.shape[1])
    for t in range(k.shape[0]):
        m = compose(token_map(k[t], v[t], float(alpha[t]), float(beta[t]), l2norm, eps), m)
    return m


def segment_map_chunked(k, v, alpha, beta, C=64, l2norm=True, eps=EPS):
    """The same map built chunk by chunk from the WY form (see the module docstring)."""
    k, v = np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64)
    alpha, beta = np.asarray(alpha, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    dk, dv = k.shape[1], v.shape[1]
    m = identity_map(dk, dv)
    for t0 in range(0, k.shape[0], C):
        t1 = min(k.shape[0], t0 + C)
        n = t1 - t0
        K = _l2n(k[t0:t1], eps, l2norm)
        be = beta[t0:t1]
        G = np.cumsum(np.log(alpha[t0:t1]))
        lower_incl = np.tril(np.ones((n, n), dtype=bool))
        Gam = np.where(lower_incl, np.exp(np.where(lower_incl, G[:, None] - G[None, :], 0.0)), 0.0)
        gam = np.exp(G)
        IA = np.eye(n) + np.tril(be[:, None] * (K @ K.T) * Gam, k=-1)
        W = solve_triangular(IA, (be * gam)[:, None] * K, lower=True, unit_diagonal=True)
        Ut = solve_triangular(IA, be[:, None] * v[t0:t1], lower=True, unit_diagonal=True)
        Kd = Gam[-1][:, None] * K                    # diag(gamma_n / gamma) Kh
        mc = (gam[-1] * np.eye(dk) - Kd.T @ W, Kd.T @ Ut)
        m = compose(mc, m)
    return m


def exclusive_scan(maps, S0):
    """Start state of every segment: S^(0) = S0, S^(p+1) = M_p S^(p) + N_p.  Returns the start
    states (one per map) and the state after the last segment."""
    starts = []
    S = np.asarray(S0, dtype=np.float64)
    for m in maps:
        starts.append(S)
        S = apply(m, S)
    return starts, S


def forward_segmented(q, k, v, alpha, beta, bounds, s0=None, scale=1.0, l2norm=True, eps=EPS):
    """Same contract as ``oracle.forward`` (shapes [B,T,H,*]), evaluated segment-parallel: the
    tokens are cut at ``bounds`` (0 = b_0 <= b_1 <= ... <= b_P = T), every segment's map is
    formed from its own tokens, the maps are scanned from S0, and every segment runs from its
    start state with the token loop."""
    from . import forward
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    bounds = list(bounds)
    assert bounds[0] == 0 and bounds[-1] == T and all(a <= b for a, b in zip(bounds, bounds[1:]))
    y = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            segs = list(zip(bounds[:-1], bounds[1:]))
            maps = [segment_map(k[b, t0:t1, h], v[b, t0:t1, h], alpha[b, t0:t1, h],
                                beta[b, t0:t1, h], l2norm, eps) for t0, t1 in segs]
            S0 = np.zeros((dk, dv)) if s0 is None else np.asarray(s0[b, h], dtype=np.float64)
            starts, S_end = exclusive_scan(maps, S0)
            for (t0, t1), Ss in zip(segs, starts):
                if t1 == t0:
                    continue
                ys, _ = forward(q[b:b + 1, t0:t1, h:h + 1], k[b:b + 1, t0:t1, h:h + 1],
                                v[b:b + 1, t0:t1, h:h + 1], alpha[b:b + 1, t0:t1, h:h + 1],
                                beta[b:b + 1, t0:t1, h:h + 1], Ss[None, None], scale=scale,
                                l2norm=l2norm, eps=eps)
                y[b, t0:t1, h] = ys[0, :, 0]
            sf[b, h] = S_end
    return y, sf

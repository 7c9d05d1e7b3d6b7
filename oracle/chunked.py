"""Second, independent fp64 form of the gated delta rule: the chunked WY/UT form.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It exists to check the
chunk algebra that the CUDA prefill is built on against the token-by-token
definition; it is never the reference for GPU parity.

Derivation (from eqs. (1)-(4) of the Qwen3.8-Flash-Next summary, picx.dev,
"Theoretical foundations"; the chunkwise delta-rule algebra itself is the
published one of Yang et al. 2024, "Parallelizing Linear Transformers with the
Delta Rule over Sequence Length", and Yang, Kautz & Hatamizadeh 2024, "Gated
Delta Networks").  Inside a chunk that starts from state S0, write
u_t = beta_t e_t, g_t = ln alpha_t, G_t = sum_{s<=t} g_s, gamma_t = exp(G_t) and
Gam_tj = exp(G_t - G_j).  Then S_t = gamma_t S0 + sum_{j<=t} Gam_tj k_j u_j^T and

    (I + A) U = diag(beta) V - diag(beta gamma) K S0,
    A = strictly-lower( diag(beta) (K K^T * Gam) ),
    U = T diag(beta) V - T diag(beta gamma) K S0,        T = (I + A)^{-1},
    Y = diag(gamma) Q S0 + ((Q K^T) * Gam * lower-incl-diag) U,
    S_end = gamma_n S0 + (diag(Gam_{n,.}) K)^T U.

Every exponent formed is G_i - G_j with i >= j (never exp(-G_j) alone).
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

EPS = 1e-6


def _l2n(x, eps, on):
    if not on:
        return x
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def forward_chunked(q, k, v, alpha, beta, s0=None, C=64, scale=1.0, l2norm=True, eps=EPS):
    """Same contract as ``oracle.forward`` (shapes [B,T,H,*]); chunk length C."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    y = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for t0 in range(0, T, C):
                t1 = min(T, t0 + C)
                n = t1 - t0
                K = _l2n(k[b, t0:t1, h], eps, l2norm)
                Q = _l2n(q[b, t0:t1, h], eps, l2norm)
                V = v[b, t0:t1, h]
                be = beta[b, t0:t1, h]
                G = np.cumsum(np.log(alpha[b, t0:t1, h]))
                diff = G[:, None] - G[None, :]
                lower_incl = np.tril(np.ones((n, n), dtype=bool))
                Gam = np.where(lower_incl, np.exp(np.where(lower_incl, diff, 0.0)), 0.0)
                gam = np.exp(G)
                A = np.tril(be[:, None] * (K @ K.T) * Gam, k=-1)
                IA = np.eye(n) + A
                W = solve_triangular(IA, (be * gam)[:, None] * K, lower=True, unit_diagonal=True)
                Ut = solve_triangular(IA, be[:, None] * V, lower=True, unit_diagonal=True)
                U = Ut - W @ S
                Y = gam[:, None] * (Q @ S) + ((Q @ K.T) * Gam) @ U
                y[b, t0:t1, h] = scale * Y
                S = gam[-1] * S + (Gam[-1][:, None] * K).T @ U
            sf[b, h] = S
    return y, sf

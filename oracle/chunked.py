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


def blocked_unit_lower_inverse(A, bs=16):
    """T = (I + A)^-1 for strictly lower-triangular A (n x n), in the blocked order the CUDA
    kernels use: the diagonal bs x bs blocks by forward substitution, then the off-diagonal
    blocks by increasing block distance, T_ij = -T_ii sum_{j <= m < i} A_im T_mj (blocks)."""
    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    nb = (n + bs - 1) // bs
    T = np.zeros((n, n))
    blk = lambda i: slice(i * bs, min(n, (i + 1) * bs))
    for b in range(nb):                       # diagonal blocks: (I + A_bb) T_bb = I
        s = blk(b)
        m = s.stop - s.start
        Ab = A[s, s]
        Tb = np.zeros((m, m))
        for col in range(m):
            x = np.zeros(m)
            for r in range(m):
                x[r] = (1.0 if r == col else 0.0) - Ab[r, :r] @ x[:r]
            Tb[:, col] = x
        T[s, s] = Tb
    for dist in range(1, nb):                  # off-diagonal blocks, nearest first
        for bj in range(nb - dist):
            bi = bj + dist
            acc = sum(A[blk(bi), blk(mb)] @ T[blk(mb), blk(bj)] for mb in range(bj, bi))
            T[blk(bi), blk(bj)] = -T[blk(bi), blk(bi)] @ acc
    return T


def forward_chunked_coupled(q, k, v, alpha, beta, s0=None, C=64, scale=1.0, l2norm=True,
                            eps=EPS, unroll=False, lag2=False):
    """The chunked forward in the coupled form the CUDA prefill's sequential kernel runs, same
    contract as ``forward_chunked``.  With S^c the state at the start of chunk c, gamma_c the
    chunk's total decay, D_c = diag(Gam_{n,.}) (so that S^{c+1} = gamma_c S^c + K_c^T D_c U_c) and
    X_c = -W_c K_{c-1}^T:

        U_c = Ut_c + gamma_{c-1} (-W_c S^{c-1}) + X_c D_{c-1} U_{c-1}      (c >= 1)

    so the only chunk-to-chunk dependence is through U and a state one chunk back.  With
    ``unroll`` the recurrence is also stepped two chunks at a time:

        U_{c+1} = Ut_{c+1} + X_{c+1} D_c Ut_c + A1 S^{c-1} + A2 D_{c-1} U_{c-1},
        A1 = -gamma_c gamma_{c-1} W_{c+1} - gamma_{c-1} X_{c+1} D_c W_c,
        A2 = X_{c+1} D_c X_c - gamma_c W_{c+1} K_{c-1}^T,

    which depends on chunk c only through chunk-local quantities.  With ``lag2`` the state is
    taken two chunks back instead (substituting S^{c-1} = gamma_{c-2} S^{c-2} + K_{c-2}^T D U_{c-2}),

        U_c = Ut_c + gamma_{c-1} gamma_{c-2} (-W_c S^{c-2}) + gamma_{c-1} X2_c D_{c-2} U_{c-2}
              + X_c D_{c-1} U_{c-1},   X2_c = -W_c K_{c-2}^T      (c >= 2),

    so that the product with the state may lag the pseudo-value recursion by two chunks."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    y = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            ch = []
            for t0 in range(0, T, C):
                t1 = min(T, t0 + C)
                n = t1 - t0
                K = _l2n(k[b, t0:t1, h], eps, l2norm)
                Q = _l2n(q[b, t0:t1, h], eps, l2norm)
                be = beta[b, t0:t1, h]
                G = np.cumsum(np.log(alpha[b, t0:t1, h]))
                lower = np.tril(np.ones((n, n), dtype=bool))
                Gam = np.where(lower, np.exp(np.where(lower, G[:, None] - G[None, :], 0.0)), 0.0)
                gam = np.exp(G)
                IA = np.eye(n) + np.tril(be[:, None] * (K @ K.T) * Gam, k=-1)
                W = solve_triangular(IA, (be * gam)[:, None] * K, lower=True, unit_diagonal=True)
                Ut = solve_triangular(IA, be[:, None] * v[b, t0:t1, h], lower=True,
                                      unit_diagonal=True)
                ch.append(dict(t0=t0, t1=t1, K=K, Q=Q, W=W, Ut=Ut, gam=gam, g=gam[-1],
                               D=Gam[-1][:, None], P=(Q @ K.T) * Gam))
            for c in range(1, len(ch)):
                ch[c]["X"] = -ch[c]["W"] @ ch[c - 1]["K"].T
            S = [np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)]
            U = []
            c = 0
            while c < len(ch):
                d = ch[c]
                if c == 0:
                    U.append(d["Ut"] - d["W"] @ S[0])
                elif lag2 and c >= 2:
                    m, mm = ch[c - 1], ch[c - 2]
                    X2 = -d["W"] @ mm["K"].T
                    U.append(d["Ut"] + m["g"] * mm["g"] * (-d["W"] @ S[c - 2])
                             + m["g"] * (X2 @ (mm["D"] * U[c - 2])) + d["X"] @ (m["D"] * U[c - 1]))
                elif unroll and c >= 2 and c % 2 == 0:
                    # U_c from (S^{c-2}, U_{c-2}) through the unrolled pair coefficients
                    m, mm = ch[c - 1], ch[c - 2]
                    A1 = -m["g"] * mm["g"] * d["W"] - mm["g"] * d["X"] @ (m["D"] * m["W"])
                    A2 = d["X"] @ (m["D"] * m["X"]) - m["g"] * d["W"] @ mm["K"].T
                    U.append(d["Ut"] + d["X"] @ (m["D"] * m["Ut"]) + A1 @ S[c - 2]
                             + A2 @ (mm["D"] * U[c - 2]))
                else:
                    m = ch[c - 1]
                    U.append(d["Ut"] + m["g"] * (-d["W"] @ S[c - 1]) + d["X"] @ (m["D"] * U[c - 1]))
                S.append(d["g"] * S[c] + d["K"].T @ (d["D"] * U[c]))
                c += 1
            for c, d in enumerate(ch):
                y[b, d["t0"]:d["t1"], h] = scale * (d["gam"][:, None] * (d["Q"] @ S[c])
                                                    + d["P"] @ U[c])
            sf[b, h] = S[-1]
    return y, sf


def backward_chunked(q, k, v, alpha, beta, s0=None, dy=None, ds_final=None, C=64, scale=1.0,
                     l2norm=True, eps=EPS):
    """Gradients of L = <dy, y> + <ds_final, S_T> in the chunked form; same contract as
    ``oracle.backward`` (dict of dq, dk, dv, dalpha, dbeta, ds0).

    Per chunk, with the forward above written as U = Ut - W S,
    Y = scale (diag(gamma) Qh S + P U) (P = Qh Kh^T * Gam, lower incl.) and
    S' = gamma_n S + Kh^T diag(gamma_n / gamma) U, the reverse pass is:
      - a chain over the chunks in reverse (the forward chain transposed):
            dU = diag(gamma_n / gamma) Kh dS' + scale P^T dY
            dS = gamma_n dS' + scale Qh^T diag(gamma) dY - W^T dU
      - then, per chunk, from S, dS', U and dU alone:
            dV = diag(beta) T^T dU,  dW = -dU S^T,
            dT = dU (diag(beta) V)^T + dW (diag(beta gamma) Kh)^T,
            dA = -T^T dT T^T restricted to A's strictly lower support,
            dP = scale dY U^T on the lower triangle (diagonal included),
            dQh = scale diag(gamma) dY S^T + (dP * Gam) Kh,
            dKh = diag(beta gamma) T^T dW + diag(gamma_n / gamma) U dS'^T + E Kh + E^T Kh
                  + (dP * Gam)^T Qh,   E = dA * beta_i Gam_ij,
            dbeta and d ln(alpha) through gamma, gamma_n and Gam (d G_i collects row i minus
            column i of dA * A + dP * (Qh Kh^T * Gam), and d ln(alpha) is the reverse cumsum
            of d G), and the L2-norm backward dx = (dxh - xh <xh, dxh>) / sqrt(|x|^2 + eps).
    """
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dy = np.zeros((B, T, H, dv)) if dy is None else np.asarray(dy, dtype=np.float64)
    dsf = np.zeros((B, H, dk, dv)) if ds_final is None else np.asarray(ds_final, dtype=np.float64)
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dalpha=np.zeros_like(alpha), dbeta=np.zeros_like(beta), ds0=np.zeros((B, H, dk, dv)))
    for b in range(B):
        for h in range(H):
            chunks = []
            for t0 in range(0, T, C):
                t1 = min(T, t0 + C)
                n = t1 - t0
                qr, kr = q[b, t0:t1, h], k[b, t0:t1, h]
                rq = 1 / np.sqrt(np.sum(qr * qr, axis=-1) + eps) if l2norm else np.ones(n)
                rk = 1 / np.sqrt(np.sum(kr * kr, axis=-1) + eps) if l2norm else np.ones(n)
                Qh, Kh = rq[:, None] * qr, rk[:, None] * kr
                G = np.cumsum(np.log(alpha[b, t0:t1, h]))
                diff = G[:, None] - G[None, :]
                lower_incl = np.tril(np.ones((n, n), dtype=bool))
                Gam = np.where(lower_incl, np.exp(np.where(lower_incl, diff, 0.0)), 0.0)
                gam = np.exp(G)
                be = beta[b, t0:t1, h]
                At = np.tril((Kh @ Kh.T) * Gam, k=-1)          # A / beta_i
                A = be[:, None] * At
                Tm = solve_triangular(np.eye(n) + A, np.eye(n), lower=True, unit_diagonal=True)
                W = Tm @ ((be * gam)[:, None] * Kh)
                Ut = Tm @ (be[:, None] * v[b, t0:t1, h])
                QK = (Qh @ Kh.T) * Gam                          # P / scale
                dec = np.exp(G[-1] - G)                         # gamma_n / gamma
                chunks.append(dict(t0=t0, t1=t1, Qh=Qh, Kh=Kh, rq=rq, rk=rk, qr=qr, kr=kr, V=v[b, t0:t1, h],
                                   be=be, gam=gam, gn=gam[-1], dec=dec, Gam=Gam, At=At, A=A, Tm=Tm, W=W,
                                   Ut=Ut, QK=QK, dY=dy[b, t0:t1, h]))
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for c in chunks:                                   # forward chain
                c["S"] = S
                c["U"] = c["Ut"] - c["W"] @ S
                S = c["gn"] * S + c["Kh"].T @ (c["dec"][:, None] * c["U"])
            dS = dsf[b, h].copy()
            for c in reversed(chunks):                         # reverse chain
                c["dSp"] = dS
                c["dU"] = c["dec"][:, None] * (c["Kh"] @ dS) + scale * c["QK"].T @ c["dY"]
                dS = c["gn"] * dS + scale * c["Qh"].T @ (c["gam"][:, None] * c["dY"]) - c["W"].T @ c["dU"]
            out["ds0"][b, h] = dS
            for c in chunks:                                   # chunk-local gradients
                S, dSp, U, dU, dY = c["S"], c["dSp"], c["U"], c["dU"], c["dY"]
                Tm, Kh, Qh, be, gam, Gam = c["Tm"], c["Kh"], c["Qh"], c["be"], c["gam"], c["Gam"]
                n = len(be)
                Z1 = Tm.T @ dU
                dV = be[:, None] * Z1
                dbe = np.sum(c["V"] * Z1, axis=1)
                dW = -dU @ S.T
                Z2 = Tm.T @ dW
                dKh = (be * gam)[:, None] * Z2
                dbg = np.sum(Kh * Z2, axis=1)                   # d (beta gamma)
                dbe += dbg * gam
                dgam = dbg * be
                dT = dU @ (be[:, None] * c["V"]).T + dW @ ((be * gam)[:, None] * Kh).T
                dA = np.tril(-(Tm.T @ dT @ Tm.T), k=-1)
                G1 = dY @ S.T
                dQh = scale * gam[:, None] * G1
                dgam += scale * np.sum(Qh * G1, axis=1)
                G2 = U @ dSp.T
                dKh += c["dec"][:, None] * G2
                ddec = np.sum(Kh * G2, axis=1)                  # d (gamma_n / gamma_i)
                dgn = np.sum(S * dSp) + np.sum(ddec / gam)
                dgam -= ddec * c["gn"] / gam ** 2
                dP = np.tril(scale * (dY @ U.T))
                E = dA * be[:, None] * Gam
                F = dP * Gam
                dKh += E @ Kh + E.T @ Kh + F.T @ Qh
                dQh += F @ Kh
                dbe += np.sum(dA * c["At"], axis=1)
                M = dA * c["A"] + dP * c["QK"]
                dG = dgam * gam + M.sum(axis=1) - M.sum(axis=0)
                dG[-1] += dgn * c["gn"]
                dlna = np.cumsum(dG[::-1])[::-1]
                t0, t1 = c["t0"], c["t1"]
                if l2norm:
                    dq = c["rq"][:, None] * (dQh - Qh * np.sum(Qh * dQh, axis=1, keepdims=True))
                    dkk = c["rk"][:, None] * (dKh - Kh * np.sum(Kh * dKh, axis=1, keepdims=True))
                else:
                    dq, dkk = dQh, dKh
                out["dq"][b, t0:t1, h] = dq
                out["dk"][b, t0:t1, h] = dkk
                out["dv"][b, t0:t1, h] = dV
                out["dalpha"][b, t0:t1, h] = dlna / alpha[b, t0:t1, h]
                out["dbeta"][b, t0:t1, h] = dbe
    return out

"""Seeded synthetic inputs for the gated delta rule (shared by tests, bench and smoke).

This module holds no arithmetic of the method itself: it only draws random
numbers and rounds them to the storage dtypes.  Both the CUDA library and the
fp64 oracle receive exactly the tensors produced here.

Recipe (per call, ``numpy.random.default_rng(seed)``, drawn in this order):
  q, k, v  ~ N(0, 1)            float32 draws, then rounded to bf16 (RNE) unless
                                 dtype == "fp32"
  a, b     ~ N(0, 1)            float64;  alpha = exp(-softplus(a)), beta = sigmoid(b),
                                 stored as float32 (alpha, beta in (0, 1))
  S0       ~ N(0, 0.02^2)       float32, only if requested
  dy       ~ N(0, 1)            float32 draws rounded like q, only if requested

Gated form (``make_gate_inputs``, its own generator): the logits a, b ~ N(0, 1) per
(token, head), A_log ~ U(-1, 1) and b_alpha ~ N(0, 0.5^2) per head, all float32.
Gated output (``make_norm_inputs``): y, z ~ N(0, 1) rounded like q, w ~ N(0, 0.1^2) float32.
QSA indexer (``make_qsa_inputs``): q ~ N(0, 1) [T, 4, 128] and k ~ N(0, 1) [T, 128] rounded to
bf16, gain g ~ 1 + N(0, 0.1^2) [128] float32.
Short convolution (``make_conv_inputs``): x ~ N(0, 1) [T, C] rounded like q, taps
w ~ N(0, 1/W) [C, W] float32, conv states ~ N(0, 1) [N, W-1, C] rounded like x.
"""
from __future__ import annotations

import numpy as np
import torch

S0_STD = 0.02


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "fp32":
        return t
    raise ValueError(f"unknown dtype {dtype!r}")


def _alpha_beta(rng, shape):
    a = rng.standard_normal(shape)
    b = rng.standard_normal(shape)
    alpha = np.exp(-np.logaddexp(0.0, a))          # exp(-softplus(a))
    beta = 1.0 / (1.0 + np.exp(-b))                # sigmoid(b)
    return (torch.from_numpy(alpha.astype(np.float32)),
            torch.from_numpy(beta.astype(np.float32)))


def make_inputs(B, T, H, dk, dv, dtype="bf16", seed=0, with_s0=False, with_dy=False,
                s0_std=S0_STD, num_states=None):
    """Dense inputs q,k [B,T,H,dk], v [B,T,H,dv], alpha,beta [B,T,H] (CPU tensors).

    ``num_states`` sets the leading size of S0 (defaults to B; the varlen layout
    uses the number of documents)."""
    rng = np.random.default_rng(seed)
    q = _round(rng.standard_normal((B, T, H, dk), dtype=np.float32), dtype)
    k = _round(rng.standard_normal((B, T, H, dk), dtype=np.float32), dtype)
    v = _round(rng.standard_normal((B, T, H, dv), dtype=np.float32), dtype)
    alpha, beta = _alpha_beta(rng, (B, T, H))
    out = dict(q=q, k=k, v=v, alpha=alpha, beta=beta, s0=None, dy=None)
    if with_s0:
        ns = B if num_states is None else num_states
        out["s0"] = torch.from_numpy(
            (rng.standard_normal((ns, H, dk, dv)) * s0_std).astype(np.float32))
    if with_dy:
        out["dy"] = _round(rng.standard_normal((B, T, H, dv), dtype=np.float32), dtype)
    return out


def varlen_lengths(total=32768, num_docs=4, seed=0):
    """Seeded document lengths summing to ``total``: num_docs-1 distinct cut points drawn
    uniformly from [1, total-1], sorted; lengths are their differences."""
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.choice(np.arange(1, total), size=num_docs - 1, replace=False))
    edges = np.concatenate([[0], cuts, [total]])
    return [int(x) for x in np.diff(edges)]


def cu_seqlens_from(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))


def make_varlen_inputs(lengths, H, dk, dv, dtype="bf16", seed=0, with_s0=True):
    """Packed documents as one [1, sum(lengths), H, *] stream plus cu_seqlens [N+1] int32;
    S0 [N,H,dk,dv] ~ N(0, 0.02^2) per document when ``with_s0``."""
    T = int(sum(lengths))
    d = make_inputs(1, T, H, dk, dv, dtype=dtype, seed=seed, with_s0=with_s0,
                    num_states=len(lengths))
    d["cu_seqlens"] = cu_seqlens_from(lengths)
    return d


def make_decode_step_inputs(N, H, dk, dv, step, dtype="bf16"):
    """Fresh tokens for decode step ``step`` (seed = 1 + step): q,k [N,H,dk], v [N,H,dv],
    alpha,beta [N,H]."""
    d = make_inputs(N, 1, H, dk, dv, dtype=dtype, seed=1 + step)
    return {n: (t[:, 0] if t is not None else None) for n, t in d.items()}


def make_decode_state(N, H, dk, dv, seed=0, std=S0_STD):
    """Initial decode state S ~ N(0, 0.02^2), fp32 [N,H,dk,dv]."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy((rng.standard_normal((N, H, dk, dv)) * std).astype(np.float32))


def make_gate_inputs(shape, H, seed=0):
    """Logits of the gated form: a, b fp32 of ``shape`` (last axis H) and the per-head
    parameters A_log, b_alpha [H] fp32."""
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(shape, dtype=np.float32)
    b = rng.standard_normal(shape, dtype=np.float32)
    A_log = rng.uniform(-1.0, 1.0, H).astype(np.float32)
    b_alpha = (rng.standard_normal(H) * 0.5).astype(np.float32)
    return dict(a=torch.from_numpy(a), b=torch.from_numpy(b), A_log=torch.from_numpy(A_log),
                b_alpha=torch.from_numpy(b_alpha))


def make_norm_inputs(rows, dv, dtype="bf16", seed=0, with_do=False):
    """Inputs of the gated RMSNorm: y, z [rows, dv] in ``dtype``, w [dv] fp32, and the
    upstream gradient d_o [rows, dv] when ``with_do``."""
    rng = np.random.default_rng(seed)
    out = dict(y=_round(rng.standard_normal((rows, dv), dtype=np.float32), dtype),
               z=_round(rng.standard_normal((rows, dv), dtype=np.float32), dtype),
               w=torch.from_numpy((rng.standard_normal(dv) * 0.1).astype(np.float32)), d_o=None)
    if with_do:
        out["d_o"] = _round(rng.standard_normal((rows, dv), dtype=np.float32), dtype)
    return out


def make_conv_inputs(lengths, C, W, dtype="bf16", seed=0, with_state=True):
    """Inputs of the short causal convolution over packed documents of the given lengths:
    x [T, C], w [C, W] fp32, conv_state [N, W-1, C] (or None) and cu_seqlens [N+1] int32."""
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    out = dict(x=_round(rng.standard_normal((T, C), dtype=np.float32), dtype),
               w=torch.from_numpy((rng.standard_normal((C, W)) / np.sqrt(W)).astype(np.float32)),
               conv_state=None, cu_seqlens=cu_seqlens_from(lengths))
    if with_state:
        out["conv_state"] = _round(
            rng.standard_normal((len(lengths), W - 1, C), dtype=np.float32), dtype)
    return out


def make_qsa_inputs(lengths, seed=0, hq=4, d=128):
    """Inputs of the QSA block indexer over packed documents: q [T, hq, d], k [T, d] bf16,
    g [d] fp32 and cu_seqlens [N+1] int32."""
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    return dict(q=_round(rng.standard_normal((T, hq, d), dtype=np.float32), "bf16"),
                k=_round(rng.standard_normal((T, d), dtype=np.float32), "bf16"),
                g=torch.from_numpy((1.0 + 0.1 * rng.standard_normal(d)).astype(np.float32)),
                cu_seqlens=cu_seqlens_from(lengths))

"""fp64 oracle of the gates and the gated output around the GDN recurrence.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Qwen3.8-Flash-Next summary (picx.dev), "Methodology", "1. GDN Hybrid Token Mixing":

* eq. (9)   beta_t  = sigmoid(W_beta x_t)
* eq. (10)  alpha_t = exp[-exp(A) softplus(W_alpha x_t + b_alpha)]
* eq. (11)  o_t = W_o [sigmoid(W_z x_t) * RMSNorm(y_t)], with the RMSNorm
  "zero-centered" and the output gate a sigmoid.

The projections W_beta x_t, W_alpha x_t, W_z x_t and W_o(.) are dense products
with learned weights and are not part of this module: its inputs are their
outputs, per (token, head),

* ``a``  = W_alpha x_t  [B,T,H]   (before the bias b_alpha)
* ``b``  = W_beta x_t   [B,T,H]
* ``z``  = W_z x_t      [B,T,H,dv]

and its parameters are ``A_log`` = A and ``b_alpha``, one scalar each per head, and
``w`` [dv], the zero-centred RMSNorm weight.  Readings where the pages are silent:

* A and b_alpha are per head, like alpha_t itself (one decay per token and head).
* RMSNorm acts on one head's y_t (dv values), the vector eq. (4) defines.
* "zero-centered": the gain is (1 + w), so that w = 0 is the identity gain;
  RMSNorm(y) = (1 + w) * y / sqrt(mean(y^2) + eps), eps = 1e-6.
* The decay is also returned in log space, g_t = ln alpha_t = -exp(A) softplus(.),
  which is what the chunked recurrence consumes.
"""
from __future__ import annotations

import numpy as np

EPS_NORM = 1e-6


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def softplus(x):
    """ln(1 + e^x), evaluated as ln(e^0 + e^x) by numpy's logaddexp."""
    return np.logaddexp(0.0, _f64(x))


def sigmoid(x):
    """1 / (1 + e^-x)."""
    x = _f64(x)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def gates(a, b, A_log, b_alpha):
    """Eqs. (9)-(10): returns (g, alpha, beta) with g = ln alpha.

    a, b: [B,T,H]; A_log, b_alpha: [H]."""
    a, b, A_log, b_alpha = map(_f64, (a, b, A_log, b_alpha))
    g = -np.exp(A_log) * softplus(a + b_alpha)
    return g, np.exp(g), sigmoid(b)


def gates_backward(a, b, A_log, b_alpha, dalpha=None, dbeta=None, dg=None):
    """Reverse mode of ``gates``.  The upstream may arrive as dalpha (gradient with
    respect to alpha), as dg (with respect to g = ln alpha), or both; dbeta with
    respect to beta.  Returns dict with da, db [B,T,H] and dA_log, db_alpha [H]."""
    a, b, A_log, b_alpha = map(_f64, (a, b, A_log, b_alpha))
    g, alpha, beta = gates(a, b, A_log, b_alpha)
    dg_tot = np.zeros_like(g)
    if dalpha is not None:
        dg_tot += _f64(dalpha) * alpha          # d alpha / d g = alpha
    if dg is not None:
        dg_tot += _f64(dg)
    # g = -exp(A) softplus(x), x = a + b_alpha; softplus'(x) = sigmoid(x)
    da = dg_tot * (-np.exp(A_log)) * sigmoid(a + b_alpha)
    dA_log = np.sum(dg_tot * g, axis=(0, 1))  # d g / d A = g
    db_alpha = np.sum(da, axis=(0, 1))
    db = (np.zeros_like(b) if dbeta is None else _f64(dbeta)) * beta * (1.0 - beta)
    return dict(da=da, db=db, dA_log=dA_log, db_alpha=db_alpha)


def rmsnorm(y, w, eps=EPS_NORM):
    """Zero-centred RMSNorm over the last axis: (1 + w) * y / sqrt(mean(y^2) + eps)."""
    y, w = _f64(y), _f64(w)
    r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)
    return (1.0 + w) * y * r


def gated_output(y, z, w, eps=EPS_NORM):
    """The bracket of eq. (11): sigmoid(z) * RMSNorm(y), per head (y, z: [..., dv])."""
    return sigmoid(z) * rmsnorm(y, w, eps)


def gated_output_backward(y, z, w, do, eps=EPS_NORM):
    """Reverse mode of ``gated_output``.  Returns dict with dy, dz (shape of y) and
    dw [dv] (summed over every leading axis)."""
    y, z, w, do = map(_f64, (y, z, w, do))
    r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)
    n = y * r                                  # unit-RMS y
    s = sigmoid(z)
    dz = do * (1.0 + w) * n * s * (1.0 - s)
    dw = np.sum(do * s * n, axis=tuple(range(y.ndim - 1)))
    dn = do * s * (1.0 + w)
    # n_i = y_i r, r = (mean(y^2) + eps)^(-1/2): dy = r (dn - n mean(dn * n))
    dy = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    return dict(dy=dy, dz=dz, dw=dw)


def layer_core(q, k, v, a, b, z, A_log, b_alpha, w, s0=None, scale=1.0, eps=EPS_NORM):
    """Eqs. (9)-(10), then the recurrence of eqs. (1)-(4) (token loop, L2-normalised q and
    k), then the bracket of eq. (11).  Returns (o, y, s_final); o and y are [B,T,H,dv]."""
    from . import forward
    _, alpha, beta = gates(a, b, A_log, b_alpha)
    y, sf = forward(q, k, v, alpha, beta, s0, scale=scale)
    return gated_output(y, z, w, eps), y, sf


def layer_core_backward(q, k, v, a, b, z, A_log, b_alpha, w, do, s0=None, ds_final=None,
                        scale=1.0, eps=EPS_NORM):
    """Reverse mode of ``layer_core`` for the upstream gradients do (of o) and ds_final.
    Returns dict with dq, dk, dv, dz, da, db, ds0, dA_log, db_alpha and dw."""
    from . import backward, forward
    _, alpha, beta = gates(a, b, A_log, b_alpha)
    y, _ = forward(q, k, v, alpha, beta, s0, scale=scale)
    go = gated_output_backward(y, z, w, do, eps)
    gr = backward(q, k, v, alpha, beta, s0, dy=go["dy"], ds_final=ds_final, scale=scale)
    gg = gates_backward(a, b, A_log, b_alpha, dalpha=gr["dalpha"], dbeta=gr["dbeta"])
    return dict(dq=gr["dq"], dk=gr["dk"], dv=gr["dv"], dz=go["dz"], da=gg["da"], db=gg["db"],
                ds0=gr["ds0"], dA_log=gg["dA_log"], db_alpha=gg["db_alpha"], dw=go["dw"])

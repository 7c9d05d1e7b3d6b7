"""fp64 CPU oracle for the Gated DeltaNet recurrence.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product library never
does.  It shares no code with ``gated_deltanet_linear_eqs_b200``.

Two independent fp64 forms of the same recurrence live here:

* ``forward`` / ``forward_varlen`` / ``backward`` / ``decode_step``: ctypes
  wrappers around ``gdn_oracle.c`` -- the token-by-token definition of the
  gated delta rule (Qwen3.8-Flash-Next summary, picx.dev, "Theoretical
  foundations", eqs. (1)-(4)) with L2-normalised q and k ("Methodology",
  "1. GDN Hybrid Token Mixing") and its reverse-mode derivative.
* ``chunked.forward_chunked`` / ``chunked.backward_chunked``: numpy form of
  the same recurrence in chunks (the WY/UT representation), used only to
  check that derivation against the token loop.
* ``gates``: numpy fp64 form of the gates of eqs. (9)-(10) and the gated
  RMSNorm of eq. (11) ("Methodology", "1. GDN Hybrid Token Mixing"), with
  their reverse modes, chained around the token loop by ``layer_core``.
* ``segments``: the recurrence as affine maps of runs of tokens (S -> M S + N),
  their composition and scan, and a segment-parallel forward built on them
  (the exchange that splitting one sequence across processors needs).

Every array crosses the boundary as a C-contiguous float64 numpy array; the
caller upcasts bf16/fp32 inputs (exactly) before calling.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None

EPS = 1e-6  # reading of "L2 normalization" adopted here: x / sqrt(|x|^2 + eps)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdn_oracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    """Load a compiled oracle library and declare its argument types."""
    lib = ctypes.CDLL(path)
    D = ctypes.POINTER(ctypes.c_double)
    I = ctypes.c_int
    lib.gdn_oracle_forward.argtypes = [D] * 8 + [I] * 5 + [ctypes.c_double, I,
                                                            ctypes.c_double, I]
    lib.gdn_oracle_forward_varlen.argtypes = (
        [D] * 5 + [ctypes.POINTER(ctypes.c_int), I] + [D] * 3 + [I] * 3
        + [ctypes.c_double, I, ctypes.c_double, I])
    lib.gdn_oracle_backward.argtypes = [D] * 14 + [I] * 5 + [ctypes.c_double, I,
                                                             ctypes.c_double, I]
    for f in (lib.gdn_oracle_forward, lib.gdn_oracle_forward_varlen, lib.gdn_oracle_backward):
        f.restype = ctypes.c_int
    return lib


_override = None


class use_library:
    """Context manager that routes the wrappers below to another build of the oracle
    source (the mutation tests compile deliberately broken copies)."""

    def __init__(self, path):
        self.lib = _bind(path)

    def __enter__(self):
        global _override
        self._prev, _override = _override, self.lib
        return self.lib

    def __exit__(self, *exc):
        global _override
        _override = self._prev
        return False


def _load():
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> exact fp64 copy on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def forward(q, k, v, alpha, beta, s0=None, scale=1.0, l2norm=True, eps=EPS, nthreads=0):
    """Token-by-token gated delta rule, eqs. (1)-(4), per (sequence, head).

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; alpha, beta: [B,T,H]; s0: [B,H,dk,dv] or None (zero).
    Returns (y [B,T,H,dv], s_final [B,H,dk,dv]) in float64.
    """
    q, k, v, alpha, beta, s0 = map(_f64, (q, k, v, alpha, beta, s0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape[:3] == (B, T, H)
    assert alpha.shape == (B, T, H) and beta.shape == (B, T, H)
    if s0 is not None:
        assert s0.shape == (B, H, dk, dv)
    y = np.zeros((B, T, H, dv))
    sf = np.zeros((B, H, dk, dv))
    rc = _load().gdn_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(s0),
                                    _ptr(y), _ptr(sf), B, T, H, dk, dv, float(scale),
                                    int(bool(l2norm)), float(eps), int(nthreads))
    _check(rc, "forward")
    return y, sf


def forward_varlen(q, k, v, alpha, beta, cu_seqlens, s0=None, scale=1.0, l2norm=True, eps=EPS,
                   nthreads=0):
    """Packed documents: q,k [1,Ttot,H,dk] (or [Ttot,H,dk]); the state restarts from
    s0[n] (zero if None) at every cu_seqlens boundary.  Returns (y, s_final [N,H,dk,dv])."""
    q, k, v, alpha, beta, s0 = map(_f64, (q, k, v, alpha, beta, s0))
    if q.ndim == 4:
        q, k, v, alpha, beta = q[0], k[0], v[0], alpha[0], beta[0]
    Ttot, H, dk = q.shape
    dv = v.shape[-1]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    N = int(cu.shape[0]) - 1
    assert cu[0] == 0 and cu[-1] == Ttot
    if s0 is not None:
        assert s0.shape == (N, H, dk, dv)
    y = np.zeros((1, Ttot, H, dv))
    sf = np.zeros((N, H, dk, dv))
    rc = _load().gdn_oracle_forward_varlen(
        _ptr(np.ascontiguousarray(q)), _ptr(np.ascontiguousarray(k)),
        _ptr(np.ascontiguousarray(v)), _ptr(np.ascontiguousarray(alpha)),
        _ptr(np.ascontiguousarray(beta)), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), N,
        _ptr(s0), _ptr(y), _ptr(sf), H, dk, dv, float(scale), int(bool(l2norm)), float(eps),
        int(nthreads))
    _check(rc, "forward_varlen")
    return y, sf


def decode_step(q, k, v, alpha, beta, state, scale=1.0, l2norm=True, eps=EPS, nthreads=0):
    """One token per sequence: q,k [N,H,dk], v [N,H,dv], alpha,beta [N,H], state [N,H,dk,dv].
    Returns (y [N,H,dv], new_state) -- eqs. (1)-(4) with T = 1."""
    q, k, v, alpha, beta, state = map(_f64, (q, k, v, alpha, beta, state))
    y, sf = forward(q[:, None], k[:, None], v[:, None], alpha[:, None], beta[:, None], state,
                    scale=scale, l2norm=l2norm, eps=eps, nthreads=nthreads)
    return y[:, 0], sf


def backward(q, k, v, alpha, beta, s0=None, dy=None, ds_final=None, scale=1.0, l2norm=True,
             eps=EPS, nthreads=0):
    """Reverse-mode gradients of (y, s_final) w.r.t. (q, k, v, alpha, beta, s0), given the
    upstream dy [B,T,H,dv] and ds_final [B,H,dk,dv] (None means zero for either).

    Returns dict with dq, dk, dv, dalpha, dbeta, ds0 (float64, shapes of the inputs)."""
    q, k, v, alpha, beta, dy, s0, ds_final = map(_f64, (q, k, v, alpha, beta, dy, s0, ds_final))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dalpha=np.zeros_like(alpha), dbeta=np.zeros_like(beta),
               ds0=np.zeros((B, H, dk, dv)))
    rc = _load().gdn_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(s0), _ptr(dy), _ptr(ds_final),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dalpha"]),
        _ptr(out["dbeta"]), _ptr(out["ds0"]), B, T, H, dk, dv, float(scale),
        int(bool(l2norm)), float(eps), int(nthreads))
    _check(rc, "backward")
    return out

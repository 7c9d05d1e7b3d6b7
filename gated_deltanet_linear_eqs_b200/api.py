"""Python binding of libgdn.so with the C ABI's names.

Argument marshalling only: every function checks that the torch tensors are CUDA,
contiguous and of the expected dtype, allocates the outputs (and workspace) it is not
given, and calls the C entry point on the current CUDA stream.  Every arithmetic step
runs in the library's kernels; a non-OK status raises ``GdnError``.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import GdnError

_DT = {torch.bfloat16: _abi.GDN_BF16, torch.float32: _abi.GDN_FP32}


def _lib():
    return _abi.load()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t, name, dtype=None, shape=None, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check(rc, what):
    if rc != _abi.GDN_OK:
        raise GdnError(rc, what)


def gdn_workspace_bytes(op, B, T, H, dk, dv, num_seqs=0):
    n = ctypes.c_size_t(0)
    _check(_lib().gdn_workspace_bytes(int(op), B, T, H, dk, dv, num_seqs, ctypes.byref(n)),
           "gdn_workspace_bytes")
    return int(n.value)


def _workspace(op, device, B, T, H, dk, dv, num_seqs=0, ws=None):
    n = gdn_workspace_bytes(op, B, T, H, dk, dv, num_seqs)
    if n == 0:
        return None, 0
    if ws is None:
        ws = torch.empty(n, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def gdn_prefill(q, k, v, alpha, beta, s0=None, scale=1.0, l2norm_qk=True, y=None,
                s_final=None, want_final=True, ws=None, stream=None):
    """q,k [B,T,H,dk], v [B,T,H,dv] (bf16 or fp32), alpha,beta [B,T,H] fp32,
    s0 [B,H,dk,dv] fp32 or None.  Returns (y, s_final)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need(alpha, "alpha", torch.float32, (B, T, H))
    _need(beta, "beta", torch.float32, (B, T, H))
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (B, T, H, dv))
    if s_final is None and want_final:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv), optional=True)
    ws, wsb = _workspace(_abi.GDN_OP_PREFILL, q.device, B, T, H, dk, dv, ws=ws)
    rc = _lib().gdn_prefill(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s0), _p(y),
                            _p(s_final), B, T, H, dk, dv, _DT[dt], float(scale),
                            int(bool(l2norm_qk)), _p(ws), wsb, _stream(stream))
    _check(rc, "gdn_prefill")
    return y, s_final


def gdn_prefill_segmented(q, k, v, alpha, beta, s0=None, num_segments=1, scale=1.0,
                          l2norm_qk=True, y=None, s_final=None, want_final=True, ws=None,
                          stream=None):
    """gdn_prefill with every sequence cut into ``num_segments`` segments that run side by side
    (affine state maps, a scan, and a pass from every segment's start state).  Same tensors as
    gdn_prefill.  Returns (y, s_final)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need(alpha, "alpha", torch.float32, (B, T, H))
    _need(beta, "beta", torch.float32, (B, T, H))
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (B, T, H, dv))
    if s_final is None and want_final:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv), optional=True)
    ws, wsb = _workspace(_abi.GDN_OP_PREFILL_SEGMENTED, q.device, B, T, H, dk, dv,
                         int(num_segments), ws=ws)
    rc = _lib().gdn_prefill_segmented(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s0), _p(y),
                                      _p(s_final), B, T, H, dk, dv, _DT[dt], float(scale),
                                      int(bool(l2norm_qk)), int(num_segments), _p(ws), wsb,
                                      _stream(stream))
    _check(rc, "gdn_prefill_segmented")
    return y, s_final


def gdn_prefill_varlen(q, k, v, alpha, beta, cu_seqlens, s0=None, scale=1.0, l2norm_qk=True,
                       y=None, s_final=None, ws=None, stream=None):
    """Packed documents: q,k [1,T,H,dk] (or [T,H,dk]), v likewise, alpha,beta [1,T,H],
    cu_seqlens int32 [N+1] on the device, s0 [N,H,dk,dv] or None.  Returns (y, s_final)."""
    if q.dim() == 3:
        q, k, v, alpha, beta = (x.unsqueeze(0) for x in (q, k, v, alpha, beta))
    _, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    N = cu_seqlens.numel() - 1
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (1, T, H, dv))
    _need(alpha, "alpha", torch.float32, (1, T, H))
    _need(beta, "beta", torch.float32, (1, T, H))
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    _need(s0, "s0", torch.float32, (N, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((1, T, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (1, T, H, dv))
    if s_final is None:
        s_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (N, H, dk, dv))
    ws, wsb = _workspace(_abi.GDN_OP_PREFILL_VARLEN, q.device, 1, T, H, dk, dv, N, ws=ws)
    rc = _lib().gdn_prefill_varlen(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(cu_seqlens), N,
                                   _p(s0), _p(y), _p(s_final), T, H, dk, dv, _DT[dt],
                                   float(scale), int(bool(l2norm_qk)), _p(ws), wsb,
                                   _stream(stream))
    _check(rc, "gdn_prefill_varlen")
    return y, s_final


def gdn_prefill_varlen_prepare(q, k, v, alpha, beta, cu_seqlens, ws, scale=1.0,
                               l2norm_qk=True, stream=None):
    """First phase of gdn_prefill_varlen (bf16): the state-independent chunk work, into ``ws``
    (a uint8 device tensor of gdn_workspace_bytes(GDN_OP_PREFILL_VARLEN, ...) bytes)."""
    if q.dim() == 3:
        q, k, v, alpha, beta = (x.unsqueeze(0) for x in (q, k, v, alpha, beta))
    _, T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.numel() - 1
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16, q.shape)
    _need(v, "v", torch.bfloat16, (1, T, H, dv))
    _need(alpha, "alpha", torch.float32, (1, T, H))
    _need(beta, "beta", torch.float32, (1, T, H))
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    rc = _lib().gdn_prefill_varlen_prepare(_p(q), _p(k), _p(v), _p(alpha), _p(beta),
                                           _p(cu_seqlens), N, T, H, dk, dv, _DT[torch.bfloat16],
                                           float(scale), int(bool(l2norm_qk)), _p(ws),
                                           ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "gdn_prefill_varlen_prepare")


def gdn_prefill_varlen_finish(q, k, cu_seqlens, ws, s0=None, y=None, s_final=None, dv=None,
                              stream=None):
    """Second phase of gdn_prefill_varlen (bf16): the sequential chunk pass from s0 over the
    records gdn_prefill_varlen_prepare wrote into ``ws``.  Returns (y, s_final)."""
    if q.dim() == 3:
        q, k = q.unsqueeze(0), k.unsqueeze(0)
    _, T, H, dk = q.shape
    dv = dk if dv is None else dv
    N = cu_seqlens.numel() - 1
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16, q.shape)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    _need(s0, "s0", torch.float32, (N, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((1, T, H, dv), dtype=torch.bfloat16, device=q.device)
    _need(y, "y", torch.bfloat16, (1, T, H, dv))
    if s_final is None:
        s_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (N, H, dk, dv))
    rc = _lib().gdn_prefill_varlen_finish(_p(q), _p(k), _p(cu_seqlens), N, _p(s0), _p(y),
                                          _p(s_final), T, H, dk, dv, _DT[torch.bfloat16], _p(ws),
                                          ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "gdn_prefill_varlen_finish")
    return y, s_final


def gdn_decode_step(q, k, v, alpha, beta, state, scale=1.0, l2norm_qk=True, y=None,
                    stream=None):
    """q,k [N,H,dk], v [N,H,dv], alpha,beta [N,H], state [N,H,dk,dv] fp32 (updated in
    place).  Returns y [N,H,dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (N, H, dv))
    _need(alpha, "alpha", torch.float32, (N, H))
    _need(beta, "beta", torch.float32, (N, H))
    _need(state, "state", torch.float32, (N, H, dk, dv))
    if y is None:
        y = torch.empty((N, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (N, H, dv))
    rc = _lib().gdn_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(state), _p(y), N, H,
                                dk, dv, _DT[dt], float(scale), int(bool(l2norm_qk)),
                                _stream(stream))
    _check(rc, "gdn_decode_step")
    return y


def gdn_backward(q, k, v, alpha, beta, dy, s0=None, ds_final=None, scale=1.0, l2norm_qk=True,
                 want_ds0=True, ws=None, stream=None):
    """Gradients of (y, s_final) w.r.t. (q, k, v, alpha, beta, s0) given dy and ds_final.
    Returns dict dq, dk, dv, dalpha, dbeta, ds0."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need(alpha, "alpha", torch.float32, (B, T, H))
    _need(beta, "beta", torch.float32, (B, T, H))
    _need(dy, "dy", dt, (B, T, H, dv))
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    _need(ds_final, "ds_final", torch.float32, (B, H, dk, dv), optional=True)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               dalpha=torch.empty_like(alpha), dbeta=torch.empty_like(beta),
               ds0=torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
               if want_ds0 else None)
    ws, wsb = _workspace(_abi.GDN_OP_BACKWARD, q.device, B, T, H, dk, dv, ws=ws)
    rc = _lib().gdn_backward(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s0), _p(dy),
                             _p(ds_final), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
                             _p(out["dalpha"]), _p(out["dbeta"]), _p(out["ds0"]), B, T, H, dk,
                             dv, _DT[dt], float(scale), int(bool(l2norm_qk)), _p(ws), wsb,
                             _stream(stream))
    _check(rc, "gdn_backward")
    return out


def gdn_backward_noalloc(q, k, v, alpha, beta, dy, s0=None, ds_final=None, scale=1.0,
                         l2norm_qk=True, want_ds0=True, out=None, stream=None):
    """gdn_backward on the library's fixed device scratch: no workspace is passed and the
    library allocates nothing.  ``out`` may supply preallocated gradient tensors (a dict with
    the keys of gdn_backward's result), so that a caller without an allocator can pass its
    own buffers.  Returns the gradient dict."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need(alpha, "alpha", torch.float32, (B, T, H))
    _need(beta, "beta", torch.float32, (B, T, H))
    _need(dy, "dy", dt, (B, T, H, dv))
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    _need(ds_final, "ds_final", torch.float32, (B, H, dk, dv), optional=True)
    if out is None:
        out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                   dalpha=torch.empty_like(alpha), dbeta=torch.empty_like(beta),
                   ds0=torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
                   if want_ds0 else None)
    rc = _lib().gdn_backward_noalloc(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(s0), _p(dy),
                                     _p(ds_final), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
                                     _p(out["dalpha"]), _p(out["dbeta"]), _p(out.get("ds0")), B,
                                     T, H, dk, dv, _DT[dt], float(scale), int(bool(l2norm_qk)),
                                     _stream(stream))
    _check(rc, "gdn_backward_noalloc")
    return out


def gdn_backward_noalloc_max_workspace():
    return int(_lib().gdn_backward_noalloc_max_workspace())


def _need_gate(a, b, A_log, b_alpha, shape, H):
    _need(a, "a", torch.float32, shape)
    _need(b, "b", torch.float32, shape)
    _need(A_log, "A_log", torch.float32, (H,))
    _need(b_alpha, "b_alpha", torch.float32, (H,))


def gdn_prefill_gated(q, k, v, a, b, A_log, b_alpha, s0=None, scale=1.0, l2norm_qk=True,
                      y=None, s_final=None, want_final=True, ws=None, stream=None):
    """gdn_prefill with alpha and beta given by eqs. (9)-(10): a = W_alpha x, b = W_beta x
    [B,T,H] fp32, A_log and b_alpha [H] fp32.  Returns (y, s_final)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need_gate(a, b, A_log, b_alpha, (B, T, H), H)
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (B, T, H, dv))
    if s_final is None and want_final:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (B, H, dk, dv), optional=True)
    ws, wsb = _workspace(_abi.GDN_OP_PREFILL, q.device, B, T, H, dk, dv, ws=ws)
    rc = _lib().gdn_prefill_gated(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(b_alpha),
                                  _p(s0), _p(y), _p(s_final), B, T, H, dk, dv, _DT[dt],
                                  float(scale), int(bool(l2norm_qk)), _p(ws), wsb,
                                  _stream(stream))
    _check(rc, "gdn_prefill_gated")
    return y, s_final


def gdn_prefill_varlen_gated(q, k, v, a, b, A_log, b_alpha, cu_seqlens, s0=None, scale=1.0,
                             l2norm_qk=True, y=None, s_final=None, ws=None, stream=None):
    """gdn_prefill_varlen with alpha and beta given by eqs. (9)-(10) (a, b [1,T,H] or [T,H]
    fp32; A_log, b_alpha [H]).  Returns (y, s_final)."""
    if q.dim() == 3:
        q, k, v, a, b = (x.unsqueeze(0) for x in (q, k, v, a, b))
    _, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    N = cu_seqlens.numel() - 1
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (1, T, H, dv))
    _need_gate(a, b, A_log, b_alpha, (1, T, H), H)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    _need(s0, "s0", torch.float32, (N, H, dk, dv), optional=True)
    if y is None:
        y = torch.empty((1, T, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (1, T, H, dv))
    if s_final is None:
        s_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    _need(s_final, "s_final", torch.float32, (N, H, dk, dv))
    ws, wsb = _workspace(_abi.GDN_OP_PREFILL_VARLEN, q.device, 1, T, H, dk, dv, N, ws=ws)
    rc = _lib().gdn_prefill_varlen_gated(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log),
                                         _p(b_alpha), _p(cu_seqlens), N, _p(s0), _p(y),
                                         _p(s_final), T, H, dk, dv, _DT[dt], float(scale),
                                         int(bool(l2norm_qk)), _p(ws), wsb, _stream(stream))
    _check(rc, "gdn_prefill_varlen_gated")
    return y, s_final


def gdn_decode_step_gated(q, k, v, a, b, A_log, b_alpha, state, scale=1.0, l2norm_qk=True,
                          y=None, stream=None):
    """gdn_decode_step with alpha and beta given by eqs. (9)-(10) (a, b [N,H] fp32; A_log,
    b_alpha [H]).  The state is updated in place.  Returns y [N,H,dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (N, H, dv))
    _need_gate(a, b, A_log, b_alpha, (N, H), H)
    _need(state, "state", torch.float32, (N, H, dk, dv))
    if y is None:
        y = torch.empty((N, H, dv), dtype=dt, device=q.device)
    _need(y, "y", dt, (N, H, dv))
    rc = _lib().gdn_decode_step_gated(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(b_alpha),
                                      _p(state), _p(y), N, H, dk, dv, _DT[dt], float(scale),
                                      int(bool(l2norm_qk)), _stream(stream))
    _check(rc, "gdn_decode_step_gated")
    return y


def gdn_backward_gated(q, k, v, a, b, A_log, b_alpha, dy, s0=None, ds_final=None, scale=1.0,
                       l2norm_qk=True, want_ds0=True, ws=None, stream=None):
    """Gradients of (y, s_final) for the gated form.  Returns dict dq, dk, dv, da, db,
    dA_log, db_alpha, ds0."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError("q/k/v must be bf16 or fp32")
    _need(q, "q", dt)
    _need(k, "k", dt, q.shape)
    _need(v, "v", dt, (B, T, H, dv))
    _need_gate(a, b, A_log, b_alpha, (B, T, H), H)
    _need(dy, "dy", dt, (B, T, H, dv))
    _need(s0, "s0", torch.float32, (B, H, dk, dv), optional=True)
    _need(ds_final, "ds_final", torch.float32, (B, H, dk, dv), optional=True)
    out = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
               da=torch.empty_like(a), db=torch.empty_like(b), dA_log=torch.empty_like(A_log),
               db_alpha=torch.empty_like(b_alpha),
               ds0=torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
               if want_ds0 else None)
    ws, wsb = _workspace(_abi.GDN_OP_BACKWARD, q.device, B, T, H, dk, dv, ws=ws)
    rc = _lib().gdn_backward_gated(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(b_alpha),
                                   _p(s0), _p(dy), _p(ds_final), _p(out["dq"]), _p(out["dk"]),
                                   _p(out["dv"]), _p(out["da"]), _p(out["db"]),
                                   _p(out["dA_log"]), _p(out["db_alpha"]), _p(out["ds0"]), B, T,
                                   H, dk, dv, _DT[dt], float(scale), int(bool(l2norm_qk)), _p(ws),
                                   wsb, _stream(stream))
    _check(rc, "gdn_backward_gated")
    return out


def gdn_gated_rmsnorm(y, z, w, eps=1e-6, o=None, stream=None):
    """The bracket of eq. (11): sigmoid(z) * (1 + w) * y / sqrt(mean(y^2) + eps) over the last
    axis.  y, z [..., dv] (bf16 or fp32, same dtype), w [dv] fp32.  Returns o like y."""
    dt = y.dtype
    if dt not in _DT:
        raise ValueError("y/z must be bf16 or fp32")
    dv = y.shape[-1]
    _need(y, "y", dt)
    _need(z, "z", dt, y.shape)
    _need(w, "w", torch.float32, (dv,))
    if o is None:
        o = torch.empty_like(y)
    _need(o, "o", dt, y.shape)
    rows = y.numel() // dv if dv else 0
    rc = _lib().gdn_gated_rmsnorm(_p(y), _p(z), _p(w), _p(o), rows, dv, _DT[dt], float(eps),
                                  _stream(stream))
    _check(rc, "gdn_gated_rmsnorm")
    return o


def gdn_gated_rmsnorm_backward(y, z, w, d_o, eps=1e-6, stream=None):
    """Gradients of gdn_gated_rmsnorm given d_o.  Returns dict dy, dz (like y) and dw [dv]."""
    dt = y.dtype
    if dt not in _DT:
        raise ValueError("y/z must be bf16 or fp32")
    dv = y.shape[-1]
    _need(y, "y", dt)
    _need(z, "z", dt, y.shape)
    _need(w, "w", torch.float32, (dv,))
    _need(d_o, "d_o", dt, y.shape)
    out = dict(dy=torch.empty_like(y), dz=torch.empty_like(z), dw=torch.empty_like(w))
    rows = y.numel() // dv if dv else 0
    rc = _lib().gdn_gated_rmsnorm_backward(_p(y), _p(z), _p(w), _p(d_o), _p(out["dy"]),
                                           _p(out["dz"]), _p(out["dw"]), rows, dv, _DT[dt],
                                           float(eps), _stream(stream))
    _check(rc, "gdn_gated_rmsnorm_backward")
    return out


def gdn_read_device_status(reset=True):
    st = ctypes.c_int(0)
    _check(_lib().gdn_read_device_status(int(bool(reset)), ctypes.byref(st)),
           "gdn_read_device_status")
    return int(st.value)


def gdn_selftest_wait_timeout(limit_ns=1_000_000, stream=None):
    """Launch the kernel whose bounded wait runs out (see include/gdn.h); afterwards
    gdn_read_device_status() reports GDN_ERR_TIMEOUT."""
    _check(_lib().gdn_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "gdn_selftest_wait_timeout")


_ACT = {"none": 0, "silu": 1}


def gdn_short_conv_varlen(x, w, cu_seqlens, conv_state=None, activation="none",
                          return_state=True, y=None, stream=None):
    """Short causal convolution of packed documents: x [T, C] (bf16 or fp32, C % 8 == 0),
    w [C, W] fp32, cu_seqlens [N+1] int32 (CUDA), conv_state [N, W-1, C] like x or None (zero).
    Returns (y [T, C], final conv state [N, W-1, C] or None)."""
    dt = x.dtype
    if dt not in _DT:
        raise ValueError("x must be bf16 or fp32")
    if x.dim() != 2 or w.dim() != 2:
        raise ValueError("x must be [T, C] and w [C, W]")
    T, C = x.shape
    W = w.shape[1]
    _need(x, "x", dt)
    _need(w, "w", torch.float32, (C, W))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    _need(conv_state, "conv_state", dt, (N, W - 1, C), optional=True)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", dt, (T, C))
    sf = torch.empty((N, W - 1, C), dtype=dt, device=x.device) if return_state else None
    rc = _lib().gdn_short_conv_varlen(_p(x), _p(w), _p(cu_seqlens), N, _p(conv_state), _p(sf),
                                      _p(y), T, C, W, _DT[dt], _ACT[activation], _stream(stream))
    _check(rc, "gdn_short_conv_varlen")
    return y, sf


def gdn_short_conv_step(x, w, conv_state, activation="none", y=None, stream=None):
    """One decode token per sequence: x [N, C], w [C, W] fp32, conv_state [N, W-1, C] like x,
    updated in place.  Returns y [N, C]."""
    dt = x.dtype
    if dt not in _DT:
        raise ValueError("x must be bf16 or fp32")
    N, C = x.shape
    W = w.shape[1]
    _need(x, "x", dt)
    _need(w, "w", torch.float32, (C, W))
    _need(conv_state, "conv_state", dt, (N, W - 1, C))
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", dt, (N, C))
    rc = _lib().gdn_short_conv_step(_p(x), _p(w), _p(conv_state), _p(y), N, C, W, _DT[dt],
                                    _ACT[activation], _stream(stream))
    _check(rc, "gdn_short_conv_step")
    return y


def _qsa_ld(max_doc_len):
    return ((max_doc_len // 4) + 3) // 4 * 4


def gdn_qsa_block_scores(q, k, g, cu_seqlens, max_doc_len, stream=None):
    """QSA indexer, pooled keys and block scores: q [T, 4, 128] bf16, k [T, 128] bf16, g [128]
    fp32, cu_seqlens [N+1] int32 (CUDA), every document at most max_doc_len tokens.  Returns
    (k_hat [T//4, 128] bf16, block_base [N+1] int32, scores [T, ld] fp32); row t of scores holds
    its visible blocks' scores (document-local block order), the rest is not written."""
    T = q.shape[0]
    _need(q, "q", torch.bfloat16, (T, 4, 128))
    _need(k, "k", torch.bfloat16, (T, 128))
    _need(g, "g", torch.float32, (128,))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    ld = _qsa_ld(max_doc_len)
    dev = q.device
    k_hat = torch.empty((T // 4, 128), dtype=torch.bfloat16, device=dev)
    base = torch.empty(N + 1, dtype=torch.int32, device=dev)
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn_workspace_bytes(_abi.GDN_OP_QSA_SCORES, 1, max(T, 1), 1, 128, 128, N),
                     dtype=torch.uint8, device=dev)
    rc = _lib().gdn_qsa_block_scores(_p(q), _p(k), _p(g), _p(cu_seqlens), N, T, int(max_doc_len),
                                     _p(k_hat), _p(base), _p(scores), ld, _p(ws), ws.numel(),
                                     _stream(stream))
    _check(rc, "gdn_qsa_block_scores")
    return k_hat, base, scores


def gdn_qsa_select_blocks(scores, cu_seqlens, budget=512, sel=None, stream=None):
    """Top-budget block selection from gdn_qsa_block_scores' scores: sel [T, budget] int32."""
    _need(scores, "scores", torch.float32)
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    T, ld = scores.shape
    if sel is None:
        sel = torch.empty((T, budget), dtype=torch.int32, device=scores.device)
    _need(sel, "sel", torch.int32, (T, budget))
    rc = _lib().gdn_qsa_select_blocks(_p(scores), ld, _p(cu_seqlens), cu_seqlens.numel() - 1, T,
                                      int(budget), _p(sel), _stream(stream))
    _check(rc, "gdn_qsa_select_blocks")
    return sel


def gdn_qsa_indexer(q, k, g, cu_seqlens, max_doc_len, budget=512, stream=None):
    """Both steps: returns (sel [T, budget] int32, k_hat, block_base, scores)."""
    k_hat, base, scores = gdn_qsa_block_scores(q, k, g, cu_seqlens, max_doc_len, stream)
    return gdn_qsa_select_blocks(scores, cu_seqlens, budget, stream=stream), k_hat, base, scores

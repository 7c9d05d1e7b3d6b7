"""ctypes declaration of libgdn.so's C ABI (include/gdn.h).

Loading fails loudly when the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
# GDN_LIBRARY selects another build of the library (e.g. libgdn_debug.so, the self-checking
# build); the default is the in-tree libgdn.so.
LIB_PATH = os.environ.get("GDN_LIBRARY") or os.path.join(PKG, "libgdn.so")
if not os.path.isabs(LIB_PATH):
    LIB_PATH = os.path.join(PKG, LIB_PATH)

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED_SHAPE = 2
GDN_ERR_WORKSPACE = 3
GDN_ERR_CUDA = 4
GDN_ERR_TIMEOUT = 5
GDN_ERR_UNSUPPORTED_DEVICE = 6

GDN_BF16 = 0
GDN_FP32 = 1

GDN_OP_PREFILL = 0
GDN_OP_PREFILL_VARLEN = 1
GDN_OP_DECODE = 2
GDN_OP_BACKWARD = 3
GDN_OP_PREFILL_SEGMENTED = 4
GDN_OP_QSA_SCORES = 5

_P = ctypes.c_void_p
_F = ctypes.c_float
_I = ctypes.c_int
_S = ctypes.c_size_t

# name -> (restype, argtypes), in the order of include/gdn.h
SIGNATURES = {
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_version": (ctypes.c_char_p, []),
    "gdn_workspace_bytes": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_S)]),
    "gdn_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P,
                         _S, _P]),
    "gdn_prefill_varlen": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _F,
                                _I, _P, _S, _P]),
    "gdn_prefill_varlen_prepare": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                                        _P, _S, _P]),
    "gdn_prefill_varlen_finish": (_I, [_P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P, _S,
                                       _P]),
    "gdn_decode_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "gdn_backward": (_I, [_P] * 14 + [_I] * 6 + [_F, _I, _P, _S, _P]),
    "gdn_backward_noalloc": (_I, [_P] * 14 + [_I] * 6 + [_F, _I, _P]),
    "gdn_backward_noalloc_max_workspace": (_S, []),
    "gdn_prefill_gated": (_I, [_P] * 10 + [_I] * 6 + [_F, _I, _P, _S, _P]),
    "gdn_prefill_varlen_gated": (_I, [_P] * 8 + [_I] + [_P] * 3 + [_I] * 5 + [_F, _I, _P, _S,
                                                                            _P]),
    "gdn_decode_step_gated": (_I, [_P] * 9 + [_I] * 5 + [_F, _I, _P]),
    "gdn_backward_gated": (_I, [_P] * 18 + [_I] * 6 + [_F, _I, _P, _S, _P]),
    "gdn_gated_rmsnorm": (_I, [_P] * 4 + [ctypes.c_int64, _I, _I, _F, _P]),
    "gdn_gated_rmsnorm_backward": (_I, [_P] * 7 + [ctypes.c_int64, _I, _I, _F, _P]),
    "gdn_read_device_status": (_I, [_I, ctypes.POINTER(_I)]),
    "gdn_short_conv_varlen": (_I, [_P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "gdn_short_conv_step": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "gdn_qsa_block_scores": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _I, _P, _S, _P]),
    "gdn_qsa_select_blocks": (_I, [_P, _I, _P, _I, _I, _I, _P, _P]),
    "gdn_qsa_indexer": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _S, _P]),
    "gdn_selftest_wait_timeout": (_I, [ctypes.c_uint64, _P]),
    "gdn_prefill_segmented": (_I, [_P] * 8 + [_I] * 6 + [_F, _I, _I, _P, _S, _P]),
}

_lock = threading.Lock()
_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load(path: str = LIB_PATH):
    """Load libgdn.so and declare every entry point; raises if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError(
                    f"libgdn.so not found at {path}; build it with "
                    "`python -m gated_deltanet_linear_eqs_b200.build` (no CPU fallback exists)")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()

"""Gated DeltaNet token-mixer recurrence on B200 (sm_100a).

The compute lives in ``libgdn.so`` (C ABI declared in ``include/gdn.h``); the functions
re-exported here are its thin torch bindings.  Importing this package does not load the
library; the first call does, and fails loudly if it has not been built.
"""
from ._abi import GdnError  # noqa: F401

__all__ = ["gdn_prefill", "gdn_prefill_varlen", "gdn_decode_step", "gdn_backward",
           "gdn_backward_noalloc", "gdn_backward_noalloc_max_workspace", "gdn_workspace_bytes",
           "gdn_read_device_status", "GdnError"]


def __getattr__(name):
    if name in __all__:
        from . import api

        return getattr(api, name)
    raise AttributeError(name)

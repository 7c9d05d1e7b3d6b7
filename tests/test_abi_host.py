"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry
point that include/gdn.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from gated_deltanet_linear_eqs_b200 import _abi
from gated_deltanet_linear_eqs_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _abi.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("gdn_prefill", "gdn_prefill_varlen", "gdn_decode_step", "gdn_backward"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings(lib):
    for code in range(7):
        s = lib.gdn_status_string(code).decode()
        assert s.startswith("GDN_")
    assert lib.gdn_status_string(99).decode() == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version().decode().startswith("gdn-b200")


def test_workspace_bytes(lib):
    n = ctypes.c_size_t(7)
    # prefill: per (chunk record, head) -W (d*64 bf16), P (64*64 bf16), Ut (64*d fp32),
    # 256 fp32 scalars and X (64*64 bf16); packed documents add the chunk-record base array
    rec = lambda d: d * 128 + 8192 + d * 256 + 1024 + 8192
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL, 1, 4096, 16, 128, 128, 0,
                                   ctypes.byref(n)) == 0
    assert n.value == 64 * 16 * rec(128)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL, 3, 65, 2, 64, 64, 0,
                                   ctypes.byref(n)) == 0
    assert n.value == 3 * 2 * 2 * rec(64)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL_VARLEN, 1, 32768, 16, 128, 128, 4,
                                   ctypes.byref(n)) == 0
    nrec = (32768 + 63 * 4) // 64  # bound on sum(ceil(len / 64)) over the documents
    up = lambda x: (x + 255) // 256 * 256
    # + the document chunk bases and one (first token, length) pair per record
    assert n.value == 256 + up(nrec * 8) + nrec * 16 * rec(128)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_DECODE, 4, 1, 2, 128, 128, 0,
                                   ctypes.byref(n)) == 0
    assert n.value == 0
    # chunked backward: per (sequence, chunk, head) record, fp32: W, Ut, U, dU (64 x d each),
    # P, T, A/beta (64 x 64 each), 256 scalars, S^c and dS' (d x d each); bf16 split images
    # (hi, lo) of -W (2 x 64 x d) and of P (2 x 64 x 64)
    brec = lambda d: 4 * (4 * 64 * d + 3 * 64 * 64 + 256 + 2 * d * d) + 2 * (2 * 64 * d + 2 * 64 * 64)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_BACKWARD, 8, 4096, 32, 128, 128, 0,
                                   ctypes.byref(n)) == 0
    assert n.value == 8 * 64 * 32 * brec(128)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_BACKWARD, 1, 65, 1, 64, 64, 0,
                                   ctypes.byref(n)) == 0
    assert n.value == 2 * brec(64)
    assert lib.gdn_workspace_bytes(42, 1, 1, 1, 64, 64, 0, ctypes.byref(n)) == \
        _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL_VARLEN, 1, 10, 1, 64, 64, 0,
                                   ctypes.byref(n)) == _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_workspace_bytes(0, 1, 1, 1, 64, 64, 0, None) == _abi.GDN_ERR_INVALID_ARG


A = 0x10000  # a 16-byte-aligned fake address: validation must reject before any access


def _prefill(lib, **kw):
    args = dict(q=A, k=A, v=A, alpha=A, beta=A, s0=0, y=A, sf=0, B=1, T=64, H=1, dk=128, dv=128,
                dt=0, scale=1.0, l2=1, ws=0, wsb=0)
    args.update(kw)
    return lib.gdn_prefill(args["q"], args["k"], args["v"], args["alpha"], args["beta"],
                           args["s0"], args["y"], args["sf"], args["B"], args["T"], args["H"],
                           args["dk"], args["dv"], args["dt"], args["scale"], args["l2"],
                           args["ws"], args["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), _abi.GDN_ERR_INVALID_ARG),
    (dict(v=0), _abi.GDN_ERR_INVALID_ARG),
    (dict(y=0), _abi.GDN_ERR_INVALID_ARG),
    (dict(k=A + 2), _abi.GDN_ERR_INVALID_ARG),        # misaligned
    (dict(s0=A + 4), _abi.GDN_ERR_INVALID_ARG),       # misaligned optional pointer
    (dict(B=0), _abi.GDN_ERR_INVALID_ARG),
    (dict(T=0), _abi.GDN_ERR_INVALID_ARG),
    (dict(H=-1), _abi.GDN_ERR_INVALID_ARG),
    (dict(dt=7), _abi.GDN_ERR_INVALID_ARG),
    (dict(dk=96, dv=96), _abi.GDN_ERR_UNSUPPORTED_SHAPE),
    (dict(dk=64, dv=128), _abi.GDN_ERR_UNSUPPORTED_SHAPE),
])
def test_prefill_rejects_bad_arguments(lib, kw, code):
    assert _prefill(lib, **kw) == code


def test_bf16_prefill_needs_its_workspace(lib):
    assert _prefill(lib, ws=0, wsb=0) == _abi.GDN_ERR_WORKSPACE
    assert _prefill(lib, ws=A, wsb=4096) == _abi.GDN_ERR_WORKSPACE
    assert _prefill(lib, ws=A + 8, wsb=1 << 30) == _abi.GDN_ERR_WORKSPACE  # misaligned


def test_split_phase_validation(lib):
    prep = lambda **kw: lib.gdn_prefill_varlen_prepare(
        *[kw.get(n, A) for n in ("q", "k", "v", "al", "be", "cu")], kw.get("n", 2),
        kw.get("T", 100), 2, kw.get("dk", 64), kw.get("dv", 64), kw.get("dt", 0), 1.0, 1,
        kw.get("ws", A), kw.get("wsb", 1 << 30), None)
    fin = lambda **kw: lib.gdn_prefill_varlen_finish(
        kw.get("q", A), kw.get("k", A), kw.get("cu", A), kw.get("n", 2), kw.get("s0", 0),
        kw.get("y", A), kw.get("sf", 0), kw.get("T", 100), 2, kw.get("dk", 64), kw.get("dv", 64),
        kw.get("dt", 0), kw.get("ws", A), kw.get("wsb", 1 << 30), None)
    for f in (prep, fin):
        assert f(q=0) == _abi.GDN_ERR_INVALID_ARG
        assert f(cu=0) == _abi.GDN_ERR_INVALID_ARG
        assert f(n=0) == _abi.GDN_ERR_INVALID_ARG
        assert f(dt=1) == _abi.GDN_ERR_INVALID_ARG          # fp32 has no split
        assert f(dk=96, dv=96) == _abi.GDN_ERR_UNSUPPORTED_SHAPE
        assert f(ws=0) == _abi.GDN_ERR_WORKSPACE
        assert f(wsb=16) == _abi.GDN_ERR_WORKSPACE
    assert fin(y=0) == _abi.GDN_ERR_INVALID_ARG
    assert fin(s0=A + 4) == _abi.GDN_ERR_INVALID_ARG


def test_varlen_rejects_bad_arguments(lib):
    f = lib.gdn_prefill_varlen
    ok = dict(q=A, k=A, v=A, al=A, be=A, cu=A, n=2, s0=0, y=A, sf=A, T=100, H=2, dk=64, dv=64,
              dt=0)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["al"], a["be"], a["cu"], a["n"], a["s0"], a["y"],
                 a["sf"], a["T"], a["H"], a["dk"], a["dv"], a["dt"], 1.0, 1, None, 0, None)

    assert call(cu=0) == _abi.GDN_ERR_INVALID_ARG
    assert call(n=0) == _abi.GDN_ERR_INVALID_ARG
    assert call(T=0) == _abi.GDN_ERR_INVALID_ARG
    assert call(dk=32, dv=32) == _abi.GDN_ERR_UNSUPPORTED_SHAPE


def test_decode_rejects_bad_arguments(lib):
    f = lib.gdn_decode_step
    assert f(A, A, A, A, A, 0, A, 4, 2, 128, 128, 0, 1.0, 1, None) == _abi.GDN_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, A, 0, 2, 128, 128, 0, 1.0, 1, None) == _abi.GDN_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, A, 4, 2, 256, 256, 0, 1.0, 1, None) == \
        _abi.GDN_ERR_UNSUPPORTED_SHAPE


def test_backward_needs_its_workspace(lib):
    f = lib.gdn_backward
    args = [A] * 6 + [A, 0] + [A] * 5 + [A] + [1, 64, 1, 64, 64, 0, 1.0, 1]
    assert f(*args, None, 0, None) == _abi.GDN_ERR_WORKSPACE
    assert f(*args, A, 16, None) == _abi.GDN_ERR_WORKSPACE
    bad = list(args)
    bad[6] = 0  # dy missing
    assert f(*bad, A, 1 << 30, None) == _abi.GDN_ERR_INVALID_ARG


def test_gated_calls_reject_bad_arguments(lib):
    """The gated entry points validate like the plain ones and also need A_log and b_alpha."""
    pre = lambda **kw: lib.gdn_prefill_gated(
        *[kw.get(n, A) for n in ("q", "k", "v", "a", "b", "Al", "ba")], 0, kw.get("y", A), 0, 1,
        64, 1, kw.get("dk", 64), 64, 0, 1.0, 1, kw.get("ws", A), 1 << 30, None)
    assert pre(Al=0) == _abi.GDN_ERR_INVALID_ARG
    assert pre(ba=A + 4) == _abi.GDN_ERR_INVALID_ARG
    assert pre(q=0) == _abi.GDN_ERR_INVALID_ARG
    assert pre(dk=96) == _abi.GDN_ERR_UNSUPPORTED_SHAPE
    assert pre(ws=0) == _abi.GDN_ERR_WORKSPACE
    var = lambda **kw: lib.gdn_prefill_varlen_gated(
        *[kw.get(n, A) for n in ("q", "k", "v", "a", "b", "Al", "ba", "cu")], 2, 0, A, A, 100, 2,
        64, 64, 0, 1.0, 1, A, 1 << 30, None)
    assert var(ba=0) == _abi.GDN_ERR_INVALID_ARG
    assert var(cu=0) == _abi.GDN_ERR_INVALID_ARG
    dec = lambda **kw: lib.gdn_decode_step_gated(
        *[kw.get(n, A) for n in ("q", "k", "v", "a", "b", "Al", "ba", "st", "y")], 4, 2, 128, 128,
        0, 1.0, 1, None)
    assert dec(Al=0) == _abi.GDN_ERR_INVALID_ARG
    assert dec(st=0) == _abi.GDN_ERR_INVALID_ARG
    bwd = lambda **kw: lib.gdn_backward_gated(
        *[kw.get(n, A) for n in ("q", "k", "v", "a", "b", "Al", "ba")], 0, A, 0,
        *[kw.get(n, A) for n in ("dq", "dk", "dv", "da", "db", "dA", "dba")], 0, 1, 64, 1, 64, 64,
        0, 1.0, 1, kw.get("ws", A), kw.get("wsb", 1 << 30), None)
    assert bwd(dA=0) == _abi.GDN_ERR_INVALID_ARG
    assert bwd(dba=A + 8) == _abi.GDN_ERR_INVALID_ARG
    assert bwd(Al=0) == _abi.GDN_ERR_INVALID_ARG
    assert bwd(ws=0) == _abi.GDN_ERR_WORKSPACE
    assert bwd(wsb=16) == _abi.GDN_ERR_WORKSPACE


def test_gated_rmsnorm_rejects_bad_arguments(lib):
    fwd = lambda **kw: lib.gdn_gated_rmsnorm(
        *[kw.get(n, A) for n in ("y", "z", "w", "o")], kw.get("rows", 10), kw.get("dv", 128),
        kw.get("dt", 0), kw.get("eps", 1e-6), None)
    assert fwd(y=0) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(w=A + 4) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(rows=-1) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(eps=-1.0) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(eps=float("nan")) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(dt=7) == _abi.GDN_ERR_INVALID_ARG
    assert fwd(dv=96) == _abi.GDN_ERR_UNSUPPORTED_SHAPE
    bwd = lambda **kw: lib.gdn_gated_rmsnorm_backward(
        *[kw.get(n, A) for n in ("y", "z", "w", "do", "dy", "dz", "dw")], kw.get("rows", 10),
        kw.get("dv", 64), 0, 1e-6, None)
    assert bwd(dw=0) == _abi.GDN_ERR_INVALID_ARG
    assert bwd(do=0) == _abi.GDN_ERR_INVALID_ARG
    assert bwd(dv=32) == _abi.GDN_ERR_UNSUPPORTED_SHAPE
def test_selftest_rejects_limits_out_of_range(lib):
    assert lib.gdn_selftest_wait_timeout(0, None) == _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_selftest_wait_timeout(999, None) == _abi.GDN_ERR_INVALID_ARG
    assert lib.gdn_selftest_wait_timeout(2_000_000_000, None) == _abi.GDN_ERR_INVALID_ARG


def test_segmented_workspace_and_validation(lib):
    n = ctypes.c_size_t(0)
    plain = ctypes.c_size_t(0)
    # one segment is the plain prefill, with its workspace
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL_SEGMENTED, 1, 4096, 16, 128, 128, 1,
                                   ctypes.byref(n)) == 0
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL, 1, 4096, 16, 128, 128, 0,
                                   ctypes.byref(plain)) == 0
    assert n.value == plain.value
    # four segments of 1024 tokens: the packed prefill's workspace for 4 documents, the zero
    # copy of v (bf16 here, fp32 for fp32 inputs: the larger is reported) and 4 state arrays
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL_SEGMENTED, 1, 4096, 16, 128, 128, 4,
                                   ctypes.byref(n)) == 0
    states = 4 * 4 * 16 * 128 * 128 * 4
    assert n.value >= 4096 * 16 * 128 * 4 + states
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_PREFILL_SEGMENTED, 1, 4096, 16, 128, 128, 0,
                                   ctypes.byref(n)) == _abi.GDN_ERR_INVALID_ARG
    f = lib.gdn_prefill_segmented
    args = [A] * 5 + [0, A, 0, 1, 4096, 2, 128, 128, 0, 1.0, 1]
    assert f(*args, 0, A, 1 << 40, None) == _abi.GDN_ERR_INVALID_ARG    # no segments
    assert f(*args, 4, None, 0, None) == _abi.GDN_ERR_WORKSPACE
    assert f(*args, 4, A, 16, None) == _abi.GDN_ERR_WORKSPACE


def test_short_conv_rejects_bad_arguments(lib):
    var = lambda **kw: lib.gdn_short_conv_varlen(
        kw.get("x", A), kw.get("w", A), kw.get("cu", A), kw.get("n", 2), kw.get("si", 0),
        kw.get("so", A), kw.get("y", A), kw.get("T", 100), kw.get("C", 2048), kw.get("W", 4),
        kw.get("dt", 0), kw.get("act", 0), None)
    assert var(x=0) == _abi.GDN_ERR_INVALID_ARG
    assert var(w=A + 4) == _abi.GDN_ERR_INVALID_ARG
    assert var(cu=0) == _abi.GDN_ERR_INVALID_ARG
    assert var(n=0) == _abi.GDN_ERR_INVALID_ARG
    assert var(T=-1) == _abi.GDN_ERR_INVALID_ARG
    assert var(C=2044) == _abi.GDN_ERR_INVALID_ARG      # not a multiple of 8
    assert var(W=0) == _abi.GDN_ERR_INVALID_ARG
    assert var(W=9) == _abi.GDN_ERR_INVALID_ARG
    assert var(dt=5) == _abi.GDN_ERR_INVALID_ARG
    assert var(act=2) == _abi.GDN_ERR_INVALID_ARG
    assert var(si=A, so=A) == _abi.GDN_ERR_INVALID_ARG  # the state may not be updated in place
    assert var(so=A + 8) == _abi.GDN_ERR_INVALID_ARG
    step = lambda **kw: lib.gdn_short_conv_step(
        kw.get("x", A), kw.get("w", A), kw.get("s", A), kw.get("y", A), kw.get("N", 4),
        kw.get("C", 64), kw.get("W", 4), 0, kw.get("act", 1), None)
    assert step(s=0) == _abi.GDN_ERR_INVALID_ARG       # W > 1 needs a state
    assert step(N=0) == _abi.GDN_ERR_INVALID_ARG
    assert step(C=12) == _abi.GDN_ERR_INVALID_ARG
    assert step(y=A + 2) == _abi.GDN_ERR_INVALID_ARG


def test_qsa_rejects_bad_arguments(lib):
    n = ctypes.c_size_t(0)
    assert lib.gdn_workspace_bytes(_abi.GDN_OP_QSA_SCORES, 1, 100, 1, 128, 128, 3,
                                   ctypes.byref(n)) == 0
    assert n.value >= 16 and n.value % 256 == 0
    sc = lambda **kw: lib.gdn_qsa_block_scores(
        kw.get("q", A), kw.get("k", A), kw.get("g", A), kw.get("cu", A), kw.get("n", 2),
        kw.get("T", 100), kw.get("ml", 60), kw.get("kh", A), kw.get("bb", A), kw.get("s", A),
        kw.get("ld", 16), kw.get("ws", A), kw.get("wsb", 256), None)
    assert sc(q=0) == _abi.GDN_ERR_INVALID_ARG
    assert sc(g=A + 4) == _abi.GDN_ERR_INVALID_ARG
    assert sc(n=0) == _abi.GDN_ERR_INVALID_ARG
    assert sc(ml=101) == _abi.GDN_ERR_INVALID_ARG     # longer than the stream
    assert sc(ld=12) == _abi.GDN_ERR_INVALID_ARG      # below floor(60 / 4)
    assert sc(ld=18) == _abi.GDN_ERR_INVALID_ARG      # not a multiple of 4
    assert sc(kh=0) == _abi.GDN_ERR_INVALID_ARG
    assert sc(ws=0) == _abi.GDN_ERR_WORKSPACE
    assert sc(wsb=8) == _abi.GDN_ERR_WORKSPACE
    sl = lambda **kw: lib.gdn_qsa_select_blocks(
        kw.get("s", A), kw.get("ld", 16), kw.get("cu", A), kw.get("n", 2), kw.get("T", 100),
        kw.get("b", 512), kw.get("sel", A), None)
    assert sl(b=0) == _abi.GDN_ERR_INVALID_ARG
    assert sl(sel=0) == _abi.GDN_ERR_INVALID_ARG
    assert sl(ld=6) == _abi.GDN_ERR_INVALID_ARG


def test_device_status_rejects_null(lib):
    assert lib.gdn_read_device_status(0, None) == _abi.GDN_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    """The Python binding computes nothing itself: tensors that are not on a CUDA device are
    rejected before any call, so no host path can stand in for the kernels."""
    import torch

    from gated_deltanet_linear_eqs_b200 import api
    q = torch.zeros((1, 64, 1, 64), dtype=torch.bfloat16)
    a = torch.full((1, 64, 1), 0.5)
    with pytest.raises(ValueError, match="CUDA"):
        api.gdn_prefill(q, q, q, a, a)
    with pytest.raises(ValueError, match="CUDA"):
        api.gdn_decode_step(q[:, 0], q[:, 0], q[:, 0], a[:, 0], a[:, 0],
                            torch.zeros((1, 1, 64, 64)))
    with pytest.raises(ValueError, match="CUDA"):
        api.gdn_backward(q, q, q, a, a, q)


def test_binding_fails_loudly_without_library(tmp_path):
    saved = _abi._lib
    try:
        _abi._lib = None
        with pytest.raises(ImportError):
            _abi.load(str(tmp_path / "missing" / "libgdn.so"))
    finally:
        _abi._lib = saved

"""C-ABI checks that need no GPU: the library loads, exports every function
include/attn.h declares, and rejects bad arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

from io_aware_attention_02_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from io_aware_attention_02_b200 import build
        build.build()
    return binding.load()


def test_header_declares_the_boundary():
    assert _declared() == sorted(["attn_fwd", "attn_quant_fp8", "attn_fwd_fp8", "attn_last_status",
                                  "attn_status_string", "attn_debug_set_fault",
                                  "attn_fwd_noalloc", "attn_fwd_strided", "attn_bwd",
                                  "attn_bwd_workspace_bytes", "attn_fwd_splitkv",
                                  "attn_fwd_splitkv_workspace_bytes", "attn_fwd_splitkv_auto_splits",
                                  "attn_fwd_host", "attn_fwd_host_workspace_bytes",
                                  "attn_noalloc_last_status", "attn_debug_status_allocated",
                                  "attn_debug_set_ablation"])


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(binding.SIGNATURES) == set(_declared())


def test_status_strings(lib):
    for code in range(6):
        assert binding.status_string(code)
    assert binding.status_string(99) == "unknown status"


GOOD = 0x10000  # 16-byte-aligned fake address: never dereferenced, validation fails first


def _fwd(lib, q=GOOD, k=GOOD, v=GOOD, o=GOOD, lse=None, B=1, H=1, N=128, d=64, scale=0.125,
         causal=0, dtype=0):
    return lib.attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), binding.ATTN_ERR_INVALID_ARG),
    (dict(o=None), binding.ATTN_ERR_INVALID_ARG),
    (dict(B=0), binding.ATTN_ERR_INVALID_ARG),
    (dict(N=0), binding.ATTN_ERR_INVALID_ARG),
    (dict(H=-1), binding.ATTN_ERR_INVALID_ARG),
    (dict(B=1 << 16, H=1 << 16, N=1), binding.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.ATTN_ERR_INVALID_ARG),
    (dict(scale=-1.0), binding.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), binding.ATTN_ERR_INVALID_ARG),
    (dict(d=0), binding.ATTN_ERR_INVALID_ARG),
    (dict(d=100), binding.ATTN_ERR_UNSUPPORTED),
    (dict(d=264), binding.ATTN_ERR_UNSUPPORTED),
    (dict(d=512), binding.ATTN_ERR_UNSUPPORTED),
    (dict(dtype=7), binding.ATTN_ERR_UNSUPPORTED),
    (dict(q=GOOD + 8), binding.ATTN_ERR_MISALIGNED),
    (dict(v=GOOD + 2), binding.ATTN_ERR_MISALIGNED),
    (dict(lse=GOOD + 2), binding.ATTN_ERR_MISALIGNED),
])
def test_fwd_validation_before_any_cuda_call(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_quant_and_fp8_validation(lib):
    Q = lib.attn_quant_fp8
    assert Q(None, GOOD, GOOD, 1, 1, 128, 128, 0, None, None) == binding.ATTN_ERR_INVALID_ARG
    assert Q(GOOD, GOOD, GOOD, 1, 1, 128, 128, 2, None, None) == binding.ATTN_ERR_INVALID_ARG
    assert Q(GOOD, GOOD, GOOD, 1, 1, 128, 96, 0, None, None) == binding.ATTN_ERR_UNSUPPORTED
    assert Q(GOOD, GOOD, GOOD, 1, 1, 128, 512, 0, None, None) == binding.ATTN_ERR_UNSUPPORTED
    assert Q(GOOD + 4, GOOD, GOOD, 1, 1, 128, 128, 0, None, None) == binding.ATTN_ERR_MISALIGNED
    F = lib.attn_fwd_fp8
    args = [GOOD] * 8 + [1, 1, 128, 128, 0.1, 0, 0, None]
    bad = list(args); bad[3] = None
    assert F(*bad) == binding.ATTN_ERR_INVALID_ARG
    bad = list(args); bad[11] = 96
    assert F(*bad) == binding.ATTN_ERR_UNSUPPORTED
    bad = list(args); bad[11] = 64; bad[14] = 1      # the V transposer needs 128-byte rows
    assert F(*bad) == binding.ATTN_ERR_UNSUPPORTED
    bad = list(args); bad[11] = 256; bad[14] = 1
    assert F(*bad) == binding.ATTN_ERR_UNSUPPORTED
    bad = list(args); bad[11] = 512
    assert F(*bad) == binding.ATTN_ERR_UNSUPPORTED
    bad = list(args); bad[0] = GOOD + 1
    assert F(*bad) == binding.ATTN_ERR_MISALIGNED
    bad = list(args); bad[14] = 3
    assert F(*bad) == binding.ATTN_ERR_INVALID_ARG


def test_strided_validation(lib):
    F = lib.attn_fwd_strided
    ok = (ctypes.c_longlong * 3)(16 * 128 * 64, 128 * 64, 64)
    bad_align = (ctypes.c_longlong * 3)(16 * 128 * 64, 128 * 64, 68)
    overlap = (ctypes.c_longlong * 3)(16 * 128 * 64, 128 * 64, 32)
    args = lambda qs: [GOOD] * 4 + [None, 1, 16, 128, 64, qs, ok, ok, ok, 0.125, 0, 0, None]
    assert F(*args(None)) == binding.ATTN_ERR_INVALID_ARG
    assert F(*args(bad_align)) == binding.ATTN_ERR_INVALID_ARG
    assert F(*args(overlap)) == binding.ATTN_ERR_INVALID_ARG


def test_bwd_workspace_size(lib):
    # two fp32 values per query row, rows padded to whole 128-row tiles, and
    # (fused mode) an fp32 dQ accumulator
    assert lib.attn_bwd_workspace_bytes(2, 3, 1, 64, 1) == 2 * 3 * 1 * 256 * 4
    assert lib.attn_bwd_workspace_bytes(1, 1, 129, 64, 1) == 2 * 256 * 4
    assert lib.attn_bwd_workspace_bytes(1, 1, 129, 64, 0) == 2 * 256 * 4 + 129 * 64 * 4
    assert lib.attn_bwd_workspace_bytes(1, 1, 0, 64, 0) == 0
    assert lib.attn_bwd_workspace_bytes(1, 1, 8, 64, 2) == 0


@pytest.mark.parametrize("det", [0, 1])
def test_bwd_validation(lib, det):
    F = lib.attn_bwd
    ws = lib.attn_bwd_workspace_bytes(1, 2, 256, 64, det)

    def call(**kw):
        a = dict(q=GOOD, k=GOOD, v=GOOD, o=GOOD, do=GOOD, lse=GOOD, dq=GOOD, dk=GOOD, dv=GOOD,
                 ws=GOOD, ws_bytes=ws, B=1, H=2, N=256, d=64, scale=0.125, causal=0, det=det, dtype=0)
        a.update(kw)
        return F(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"], a["ws"],
                 a["ws_bytes"], a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"], a["det"], a["dtype"],
                 None)

    assert call(lse=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(ws=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(do=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(ws_bytes=ws - 4) == binding.ATTN_ERR_INVALID_ARG
    assert call(N=0) == binding.ATTN_ERR_INVALID_ARG
    assert call(causal=3) == binding.ATTN_ERR_INVALID_ARG
    assert call(det=2) == binding.ATTN_ERR_INVALID_ARG
    assert call(d=256) == binding.ATTN_ERR_UNSUPPORTED
    assert call(d=100) == binding.ATTN_ERR_UNSUPPORTED
    assert call(dtype=2) == binding.ATTN_ERR_UNSUPPORTED
    assert call(dk=GOOD + 8) == binding.ATTN_ERR_MISALIGNED
    assert call(ws=GOOD + 4) == binding.ATTN_ERR_MISALIGNED
    assert call(lse=GOOD + 2) == binding.ATTN_ERR_MISALIGNED


def test_splitkv_workspace_size(lib):
    # fp32 partial O (n_splits x B*H x Nq x d) then LSE (padded to 16 bytes)
    assert lib.attn_fwd_splitkv_workspace_bytes(2, 3, 5, 64, 4) == 4 * 6 * 5 * 64 * 4 + 4 * 6 * 5 * 4
    assert lib.attn_fwd_splitkv_workspace_bytes(1, 1, 1, 8, 3) == 3 * 8 * 4 + 16
    assert lib.attn_fwd_splitkv_workspace_bytes(1, 1, 0, 8, 3) == 0
    assert lib.attn_fwd_splitkv_workspace_bytes(1, 1, 4, 8, 0) == 0


def test_splitkv_validation(lib):
    F = lib.attn_fwd_splitkv
    ws = lib.attn_fwd_splitkv_workspace_bytes(1, 2, 4, 64, 3)

    def call(**kw):
        a = dict(q=GOOD, k=GOOD, v=GOOD, o=GOOD, lse=None, B=1, H=2, Nq=4, Nk=1000, d=64, scale=0.125,
                 causal=0, ns=3, dtype=0, ws=GOOD, ws_bytes=ws)
        a.update(kw)
        return F(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["scale"],
                 a["causal"], a["ns"], a["dtype"], a["ws"], a["ws_bytes"], None)

    assert call(q=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(ws=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(Nq=0) == binding.ATTN_ERR_INVALID_ARG
    assert call(Nk=0) == binding.ATTN_ERR_INVALID_ARG
    assert call(causal=1, Nq=2000) == binding.ATTN_ERR_INVALID_ARG     # queries past the keys
    assert call(ns=-1) == binding.ATTN_ERR_INVALID_ARG
    assert call(scale=float("nan")) == binding.ATTN_ERR_INVALID_ARG
    assert call(d=264) == binding.ATTN_ERR_UNSUPPORTED
    assert call(d=100) == binding.ATTN_ERR_UNSUPPORTED
    assert call(dtype=5) == binding.ATTN_ERR_UNSUPPORTED
    assert call(o=GOOD + 8) == binding.ATTN_ERR_MISALIGNED
    assert call(lse=GOOD + 2) == binding.ATTN_ERR_MISALIGNED


def test_host_forward_validation(lib):
    F = lib.attn_fwd_host
    ws = lib.attn_fwd_host_workspace_bytes(1, 8, 256, 64)
    # two slots of (q, k, v, o) for one head (fewer than 16 heads), plus LSE, 256-byte rounded
    assert ws == 2 * (4 * 1 * 256 * 64 * 2 + 1 * 256 * 4)
    # 64 heads: chunks of ceil(64 / 16) = 4 heads
    assert lib.attn_fwd_host_workspace_bytes(4, 16, 100, 64) == 2 * (4 * 4 * 100 * 64 * 2 + 1792)
    assert lib.attn_fwd_host_workspace_bytes(1, 1, 0, 64) == 0

    def call(**kw):
        a = dict(q=GOOD, k=GOOD, v=GOOD, o=GOOD, lse=None, B=1, H=8, N=256, d=64, scale=0.125, causal=0, dtype=0,
                 ws=GOOD, ws_bytes=ws)
        a.update(kw)
        return F(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"],
                 a["dtype"], a["ws"], a["ws_bytes"], None)

    assert call(q=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(ws=None) == binding.ATTN_ERR_INVALID_ARG
    assert call(ws_bytes=ws - 1) == binding.ATTN_ERR_INVALID_ARG
    assert call(N=0) == binding.ATTN_ERR_INVALID_ARG
    assert call(d=264) == binding.ATTN_ERR_UNSUPPORTED
    assert call(dtype=3) == binding.ATTN_ERR_UNSUPPORTED
    assert call(ws=GOOD + 8) == binding.ATTN_ERR_MISALIGNED


def test_debug_hook_validation(lib):
    assert lib.attn_debug_set_fault(5, 0) == binding.ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_set_ablation(2) == binding.ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_set_ablation(-1) == binding.ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_set_fault(0, 0) == binding.ATTN_OK
    # mode 2 (a planted range-check failure) exists in the debug build only
    assert lib.attn_debug_set_fault(2, 0) == binding.ATTN_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.fwd(x, x, x)


def test_debug_build_exports_the_same_boundary():
    """The debug build (range checks in the forward kernel) is the same C ABI:
    it loads beside the release library, exports every declared entry point,
    and names the status code its checks report."""
    from io_aware_attention_02_b200 import build
    build.build(debug=True)
    dlib = binding.load_debug()
    for name in _declared():
        assert hasattr(dlib, name), name
    assert dlib.attn_status_string(binding.ATTN_ERR_BOUNDS) == b"debug bounds check failed"
    assert binding.load().attn_status_string(binding.ATTN_ERR_BOUNDS) == b"debug bounds check failed"
    assert dlib.attn_debug_set_fault(2, 0) == binding.ATTN_OK     # accepted here; reset it
    assert dlib.attn_debug_set_fault(0, 0) == binding.ATTN_OK

"""ctypes binding of libattn_sm100.so (C ABI in include/attn.h).

Argument marshalling only: torch provides device memory and the current
stream; every step of the computation runs in the library's CUDA kernels.
There is no fallback: if the library cannot be loaded, or a GPU is missing,
these functions raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn_sm100.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libattn_sm100_debug.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_MISALIGNED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT, ATTN_ERR_BOUNDS = range(7)
ATTN_BF16, ATTN_FP16 = 0, 1

# name -> (restype, argtypes); mirrors include/attn.h
_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P]),
    "attn_quant_fp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P]),
    "attn_last_status": (_I, [_P, ctypes.POINTER(ctypes.c_int)]),
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_debug_set_fault": (_I, [_I, _I]),
    "attn_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P]),
    "attn_noalloc_last_status": (_I, [_P, ctypes.POINTER(ctypes.c_int)]),
    "attn_debug_status_allocated": (_I, []),
    "attn_debug_set_ablation": (_I, [_I]),
    "attn_fwd_strided": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _F, _I, _I, _P]),
    "attn_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_fwd_splitkv": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P, ctypes.c_size_t, _P]),
    "attn_fwd_splitkv_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_fwd_splitkv_auto_splits": (_I, [_I, _I, _I, _I]),
    "attn_fwd_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P, ctypes.c_size_t, _P]),
    "attn_fwd_host_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _F, _I, _I, _I,
                      _P]),
}


class AttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and set every exported signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m io_aware_attention_02_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def lib() -> ctypes.CDLL:
    return load()


def load_debug(path: str = DEBUG_LIB_PATH) -> ctypes.CDLL:
    """The debug build (``build --debug``: range checks on every TMEM and
    shared-memory access of the forward kernel, ATTN_ERR_BOUNDS on a failed
    one), loaded beside the release library with the same signatures.  Call
    its entry points directly; the wrappers of this module use the release
    library."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m io_aware_attention_02_b200.build --debug`")
    dlib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(dlib, name)
        fn.restype = res
        fn.argtypes = args
    return dlib


def status_string(code: int) -> str:
    return load().attn_status_string(int(code)).decode()


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn: str, code: int):
    if code != ATTN_OK:
        raise AttnError(fn, code)


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous [B, H, N, d]")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D [B, H, N, d]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")


def _strides3(t):
    """(batch, head, row) element strides of a [B, H, N, d] view with a
    contiguous head dim, as a ctypes array."""
    if t.stride(-1) != 1:
        raise ValueError("the head dim (last) must be contiguous")
    return (ctypes.c_longlong * 3)(*t.stride()[:3])


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: float | None = None, out: torch.Tensor | None = None,
        lse: torch.Tensor | None = None, return_lse: bool = True):
    """O, LSE = attention(q, k, v) on the current stream.

    q, k, v: CUDA tensors [B, H, N, d] of bf16 or fp16.  Contiguous tensors go
    through ``attn_fwd``; other views with a contiguous head dim (for example
    ``x.transpose(1, 2)`` of a [B, N, H, d] tensor) through
    ``attn_fwd_strided``, without a copy.  ``out`` may be such a view too.
    Returns (o, lse) with lse fp32 [B, H, N] (None if ``return_lse`` is False).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D [B, H, N, d]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bf16 or all fp16")
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q, memory_format=torch.contiguous_format) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dtype = ATTN_BF16 if q.dtype == torch.bfloat16 else ATTN_FP16
    lse_p = _ptr(lse) if return_lse else None
    if all(t.is_contiguous() for t in (q, k, v, o)):
        code = load().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), lse_p, B, H, N, d, scale,
                               int(bool(causal)), dtype, _stream(q.device))
        _check("attn_fwd", code)
    else:
        code = load().attn_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), lse_p, B, H, N, d,
                                       _strides3(q), _strides3(k), _strides3(v), _strides3(o),
                                       scale, int(bool(causal)), dtype, _stream(q.device))
        _check("attn_fwd_strided", code)
    return o, (lse if return_lse else None)


def fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                scale: float | None = None, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, return_lse: bool = True):
    """Like :func:`fwd`, through ``attn_fwd_noalloc``: the library allocates
    no device memory for this call (its scratch is a static device array).
    The outputs here are still allocated by torch unless passed in."""
    _check_qkv(q, k, v)
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bf16 or all fp16")
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dtype = ATTN_BF16 if q.dtype == torch.bfloat16 else ATTN_FP16
    code = load().attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                   _ptr(lse) if return_lse else None, B, H, N, d, scale,
                                   int(bool(causal)), dtype, _stream(q.device))
    _check("attn_fwd_noalloc", code)
    return o, (lse if return_lse else None)


def bwd_workspace_bytes(B: int, H: int, N: int, d: int, deterministic: bool = False) -> int:
    return int(load().attn_bwd_workspace_bytes(int(B), int(H), int(N), int(d), int(bool(deterministic))))


def bwd(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None,
        dq=None, dk=None, dv=None, workspace=None, deterministic: bool = False):
    """dQ, dK, dV of attention through ``attn_bwd`` on the current stream.

    q, k, v, o, do: contiguous CUDA tensors [B, H, N, d] of one 16-bit dtype
    (o and lse from :func:`fwd` with the same causal and scale); lse fp32
    [B, H, N].  ``workspace`` (uint8, at least :func:`bwd_workspace_bytes`)
    is allocated here when not given.  ``deterministic`` selects the
    two-kernel path without atomics (bit-reproducible dQ).
    """
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        if not t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor [B, H, N, d]")
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("inputs must be bf16 or fp16")
    B, H, N, d = q.shape
    if lse is None or lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, N]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    nbytes = bwd_workspace_bytes(B, H, N, d, deterministic)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    dtype = ATTN_BF16 if q.dtype == torch.bfloat16 else ATTN_FP16
    code = load().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                           _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                           B, H, N, d, scale, int(bool(causal)), int(bool(deterministic)), dtype,
                           _stream(q.device))
    _check("attn_bwd", code)
    return dq, dk, dv


def fwd_splitkv(q, k, v, causal: bool = False, scale: float | None = None, n_splits: int = 0,
                out=None, lse=None, return_lse: bool = True, workspace=None):
    """O, LSE of q [B, H, Nq, d] against k, v [B, H, Nk, d] through
    ``attn_fwd_splitkv`` (keys split across CTAs, then merged).  Causal
    masking aligns the queries with the last Nq key positions."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor [B, H, rows, d]")
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bf16 or all fp16")
    B, H, Nq, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != H or k.shape[3] != d:
        raise ValueError("k and v must be [B, H, Nk, d] matching q")
    Nk = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    ns = int(n_splits) if n_splits else int(load().attn_fwd_splitkv_auto_splits(B, H, Nq, Nk))
    ns = max(1, min(ns, (Nk + 127) // 128))
    if workspace is None:
        nbytes = int(load().attn_fwd_splitkv_workspace_bytes(B, H, Nq, d, ns))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    dtype = ATTN_BF16 if q.dtype == torch.bfloat16 else ATTN_FP16
    code = load().attn_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse) if return_lse else None,
                                   B, H, Nq, Nk, d, scale, int(bool(causal)), ns, dtype, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(q.device))
    _check("attn_fwd_splitkv", code)
    return o, (lse if return_lse else None)


def fwd_host(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
             return_lse: bool = True, workspace=None, device=None):
    """O, LSE of host (CPU) tensors [B, H, N, d] through ``attn_fwd_host``:
    the copies to and from the GPU overlap the computation, chunk by chunk.

    Inputs should be pinned (``tensor.pin_memory()``) for the overlap; the
    outputs are allocated pinned when not given.  The call is asynchronous on
    the current stream of ``device`` (default: the current device):
    synchronize before reading the results.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor [B, H, N, d]")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape")
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must all be bf16 or all fp16")
    B, H, N, d = q.shape
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty(q.shape, dtype=q.dtype).pin_memory() if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    if workspace is None:
        nbytes = int(load().attn_fwd_host_workspace_bytes(B, H, N, d))
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    dtype = ATTN_BF16 if q.dtype == torch.bfloat16 else ATTN_FP16
    with torch.cuda.device(dev):
        code = load().attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse) if return_lse else None,
                                    B, H, N, d, scale, int(bool(causal)), dtype, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(dev))
    _check("attn_fwd_host", code)
    return o, (lse if return_lse else None)


def quant_fp8(x: torch.Tensor, hadamard: bool = False, signs: torch.Tensor | None = None,
              out: torch.Tensor | None = None, descale: torch.Tensor | None = None):
    """Per-block e4m3 quantisation through ``attn_quant_fp8``.

    Returns (codes uint8 [B, H, N, d], descale fp32 [B, H, ceil(N/128)]).
    """
    if not x.is_cuda or x.dtype != torch.bfloat16 or not x.is_contiguous() or x.dim() != 4:
        raise ValueError("x must be a contiguous CUDA bf16 tensor [B, H, N, d]")
    B, H, N, d = x.shape
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if out is None else out
    if descale is None:
        descale = torch.empty((B, H, (N + 127) // 128), dtype=torch.float32, device=x.device)
    if signs is not None:
        signs = signs.to(device=x.device, dtype=torch.float32).contiguous()
    code = load().attn_quant_fp8(_ptr(x), _ptr(codes), _ptr(descale), B, H, N, d,
                                 int(bool(hadamard)), _ptr(signs) if hadamard else None,
                                 _stream(x.device))
    _check("attn_quant_fp8", code)
    return codes, descale


def fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, causal: bool = False,
            scale: float | None = None, v_transpose: bool = False, out=None, lse=None,
            return_lse: bool = True):
    """O (bf16), LSE = e4m3 attention through ``attn_fwd_fp8``.

    q8, k8, v8: uint8 e4m3 codes [B, H, N, d] from :func:`quant_fp8`;
    descales fp32 [B, H, ceil(N/128)].
    """
    _check_qkv(q8, k8, v8)
    B, H, N, d = q8.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device) if out is None else out
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    code = load().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_descale), _ptr(k_descale),
                               _ptr(v_descale), _ptr(o), _ptr(lse) if return_lse else None,
                               B, H, N, d, scale, int(bool(causal)), int(bool(v_transpose)),
                               _stream(q8.device))
    _check("attn_fwd_fp8", code)
    return o, (lse if return_lse else None)


def last_status(stream=None):
    """(status code, [barrier id, block index]) of the current device; clears it."""
    where = (ctypes.c_int * 2)()
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    code = load().attn_last_status(ctypes.c_void_p(s), where)
    return code, [where[0], where[1]]


def noalloc_last_status(stream=None):
    """(status code, [barrier id, block index]) of the record attn_fwd_noalloc
    writes (the library's static device array); clears it."""
    where = (ctypes.c_int * 2)()
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    code = load().attn_noalloc_last_status(ctypes.c_void_p(s), where)
    return code, [where[0], where[1]]


def debug_status_allocated() -> int:
    """1 if attn_fwd's status word exists on the current device, else 0."""
    return int(load().attn_debug_status_allocated())


def debug_set_ablation(mode: int):
    """1: serialise the two query tiles of the 16-bit forward (no overlap of
    softmax and matmuls); 0: the normal ping-pong schedule."""
    _check("attn_debug_set_ablation", load().attn_debug_set_ablation(int(mode)))


def debug_set_fault(mode: int, wait_limit_ms: int = 0):
    _check("attn_debug_set_fault", load().attn_debug_set_fault(int(mode), int(wait_limit_ms)))

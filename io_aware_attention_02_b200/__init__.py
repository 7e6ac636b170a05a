"""B200-native (sm_100a) fused attention.

``O = softmax(scale * Q K^T [+ causal mask]) V`` with per-row log-sum-exp,
its backward (dQ, dK, dV), a split-KV form for decode shapes and an FP8
path, computed by hand-written tcgen05/TMA CUDA kernels behind a C ABI
(``include/attn.h``, ``libattn_sm100.so``).  The Python functions here only
marshal arguments: torch supplies device memory and the current stream.

The binding is imported lazily so that ``inputs`` (the seeded generator) can
be used on machines without the built library.
"""

import importlib

_BINDING_FUNCS = ("fwd", "fwd_noalloc", "fwd_host", "fwd_splitkv", "bwd", "fwd_fp8", "quant_fp8", "last_status")

__all__ = [*_BINDING_FUNCS, "binding", "inputs"]


def __getattr__(name):
    if name in ("binding", "inputs", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    if name in _BINDING_FUNCS:
        return getattr(importlib.import_module(f"{__name__}.binding"), name)
    raise AttributeError(name)

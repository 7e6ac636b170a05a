"""B200-native (sm_100a) fused attention forward.

``O = softmax(scale * Q K^T [+ causal mask]) V`` with per-row log-sum-exp,
computed by hand-written tcgen05/TMA CUDA kernels behind a C ABI
(``include/attn.h``, ``libattn_sm100.so``).  The Python functions here only
marshal arguments: torch supplies device memory and the current stream.

The binding is imported lazily so that ``inputs`` (the seeded generator) can
be used on machines without the built library.
"""

__all__ = ["fwd", "fwd_fp8", "quant_fp8", "lib"]


def __getattr__(name):
    if name in ("fwd", "fwd_fp8", "quant_fp8", "lib", "binding"):
        from . import binding

        return binding if name == "binding" else getattr(binding, name)
    raise AttributeError(name)

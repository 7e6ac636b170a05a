"""Low-precision baselines of the pages' accuracy experiment -- TEST INFRASTRUCTURE ONLY.

Only tests use this module; the CUDA product path never imports it.

The quantum-bit repost "H100 utilisation 75% ... FlashAttention-3"
(m.ruangu.net), section on the FP8 accuracy test, compares against:

* standard attention in FP16, whose intermediate softmax result is stored in
  FP16 (FlashAttention keeps its statistics in FP32 and is reported 1.7x
  more accurate);
* standard attention in FP8 with one scale per tensor, matmul accumulators
  in FP32 and the intermediate softmax result in FP16 (FlashAttention-3 FP8
  with block quantisation and incoherent processing is reported 2.6x more
  accurate).

These functions emulate those baselines step by step with explicit numpy
casts.  Readings where the page is silent: scores accumulate in fp32 from
the rounded inputs; the softmax is computed in fp32 and its normalised
result rounded to fp16; for FP8 the fp16 probabilities are rounded to e4m3
with one per-tensor scale (448 / max P) before the P.V product, which
accumulates in fp32; the output is rounded to fp16.  The fp16 baseline has a
second reading of "intermediate results in FP16" (``round_scores=True``):
the score matrix itself is also rounded to fp16 before the softmax, as an
eager fp16 attention does when its Q.K^T product returns fp16.

The ratios themselves are measured, not asserted by the pages' numbers:
"parity unpinned" for the 1.7x / 2.6x values.
"""

from __future__ import annotations

import numpy as np

from . import fp8 as F


def _masked(s, causal):
    if causal:
        n = s.shape[-1]
        s = np.where(np.tril(np.ones((s.shape[-2], n), dtype=bool)), s, -np.inf)
    return s


def standard_fp16_attention(q, k, v, scale, causal=False, round_scores=False):
    """FP16 standard attention of one head: fp16 inputs, fp32 scores (rounded
    to fp16 when ``round_scores``), softmax written out in fp16, fp32
    accumulation of P.V, fp16 output."""
    q16, k16, v16 = (np.asarray(x, dtype=np.float16) for x in (q, k, v))
    s = (q16.astype(np.float32) @ k16.astype(np.float32).T) * np.float32(scale)
    if round_scores:
        s = s.astype(np.float16).astype(np.float32)
    s = _masked(s, causal)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m, dtype=np.float32)
    p16 = (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float16)
    o = p16.astype(np.float32) @ v16.astype(np.float32)
    return o.astype(np.float16).astype(np.float64)


def per_tensor_fp8_attention(q, k, v, scale, causal=False):
    """FP8 standard attention of one head with one scale per tensor."""
    def quant(x):
        x = np.asarray(x, dtype=np.float32)
        amax = np.float32(np.abs(x).max())
        s = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(F.E4M3_MAX))
        return F.e4m3_decode(F.e4m3_encode((x / s).astype(np.float32))).astype(np.float32), s

    q8, sq = quant(q)
    k8, sk = quant(k)
    v8, sv = quant(v)
    s = (q8 @ k8.T) * np.float32(sq * sk * scale)
    s = _masked(s, causal)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m, dtype=np.float32)
    p16 = (e / e.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float16)
    pmax = np.float32(p16.astype(np.float32).max())
    sp = np.float32(pmax / np.float32(F.E4M3_MAX))
    p8 = F.e4m3_decode(F.e4m3_encode((p16.astype(np.float32) / sp).astype(np.float32))).astype(np.float32)
    o = (p8 @ v8) * np.float32(sp * sv)
    return o.astype(np.float16).astype(np.float64)


def rmse(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.sqrt(np.mean((a - b) ** 2)))

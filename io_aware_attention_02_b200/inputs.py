"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only draws numbers.  Both the
CUDA path and the CPU oracle receive what it returns, so the two sides see the
same values.

Recipe (the workloads of the FlashAttention-3 pages, synthetic):

* Q, K, V entries are i.i.d. N(0, 1) fp32, drawn per (tensor, batch, head)
  from ``numpy.random.Generator(Philox)`` keyed by (seed, tensor id, b, h), so
  any head can be regenerated alone (long-context checks need only a few
  heads' rows on the CPU).
* Outlier variant (the FP8 accuracy experiment in the quantum-bit repost
  "H100 utilisation 75% ... FlashAttention-3", m.ruangu.net): a Bernoulli
  mask with p = 0.001 drawn from the same keyed stream selects entries that
  are replaced by N(0, 10^2) draws.  ``outlier_mode="add"`` instead adds the
  N(0, 10^2) term, which is the page's own wording.
* The fp32 draws are rounded to bf16 (round-to-nearest-even, torch's CPU
  cast); that rounded tensor is what both the GPU and the oracle receive.
* The output gradient dO of the backward pass is drawn the same way (tensor
  id "do"), i.i.d. N(0, 1) rounded to the input dtype.
* Hadamard sign diagonals (+-1 per head-dim entry) are drawn here too, so the
  random part of incoherent processing is an input to both sides.
"""

from __future__ import annotations

import numpy as np
import torch

_TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}


def _rng(seed: int, tensor: str, b: int, h: int) -> np.random.Generator:
    return _philox(seed, _TENSOR_IDS[tensor], b, h)


def _philox(seed: int, a: int, b: int, c: int) -> np.random.Generator:
    """Philox-4x64 stream keyed by (seed, a, b, c); a, b, c < 2^21 each."""
    word = (int(a) << 42) | (int(b) << 21) | int(c)
    return np.random.Generator(np.random.Philox(key=np.array([int(seed), word], dtype=np.uint64)))


def head_f32(seed: int, tensor: str, b: int, h: int, N: int, d: int,
             outliers: bool = False, outlier_mode: str = "replace",
             outlier_p: float = 1e-3, outlier_std: float = 10.0) -> np.ndarray:
    """One head's [N, d] fp32 draws for tensor 'q', 'k' or 'v'."""
    g = _rng(seed, tensor, b, h)
    x = g.standard_normal((N, d), dtype=np.float32)
    if outliers:
        mask = g.random((N, d)) < outlier_p
        big = (g.standard_normal((N, d), dtype=np.float32) * np.float32(outlier_std))
        if outlier_mode == "replace":
            x = np.where(mask, big, x)
        elif outlier_mode == "add":
            x = np.where(mask, x + big, x)
        else:
            raise ValueError(outlier_mode)
    return x.astype(np.float32)


def head_bf16(seed: int, tensor: str, b: int, h: int, N: int, d: int, **kw) -> torch.Tensor:
    """One head's [N, d] tensor rounded to bf16 (CPU)."""
    return torch.from_numpy(head_f32(seed, tensor, b, h, N, d, **kw)).to(torch.bfloat16)


def qkv(B: int, H: int, N: int, d: int, seed: int = 0, dtype=torch.bfloat16,
        outliers: bool = False, outlier_mode: str = "replace"):
    """Full (q, k, v) CPU tensors [B, H, N, d] in ``dtype`` (bf16 or fp16)."""
    out = []
    for name in ("q", "k", "v"):
        t = torch.empty((B, H, N, d), dtype=dtype)
        for b in range(B):
            for h in range(H):
                x = head_f32(seed, name, b, h, N, d, outliers=outliers, outlier_mode=outlier_mode)
                t[b, h] = torch.from_numpy(x).to(dtype)
        out.append(t)
    return tuple(out)


def grad_out(B: int, H: int, N: int, d: int, seed: int = 0, dtype=torch.bfloat16) -> torch.Tensor:
    """Output gradient dO, a CPU tensor [B, H, N, d] in ``dtype``."""
    t = torch.empty((B, H, N, d), dtype=dtype)
    for b in range(B):
        for h in range(H):
            t[b, h] = torch.from_numpy(head_f32(seed, "do", b, h, N, d)).to(dtype)
    return t


def sample_rows(N: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted query-row sample: 0, 1, N/2, N-1 plus seeded uniform rows.

    Used where the oracle cannot afford every row (long sequences).
    """
    fixed = sorted({0, min(1, N - 1), N // 2, N - 1})
    if count >= N:
        return np.arange(N, dtype=np.int64)
    g = _philox(seed, 1 << 20 | 7, N, count)
    rest = np.setdiff1d(np.arange(N), fixed)
    pick = g.permutation(rest)[:max(0, count - len(fixed))]
    return np.sort(np.concatenate([np.array(fixed, dtype=np.int64), pick.astype(np.int64)]))


def stratified_rows(N: int, count: int, seed: int = 0) -> np.ndarray:
    """``count`` rows, one seeded draw per equal stratum of [0, N); 0 and N-1 included."""
    g = _philox(seed, 1 << 20 | 11, N, count)
    edges = np.linspace(0, N, count + 1).astype(np.int64)
    rows = [int(g.integers(lo, max(lo + 1, hi))) for lo, hi in zip(edges[:-1], edges[1:])]
    rows[0], rows[-1] = 0, N - 1
    return np.array(sorted(set(rows)), dtype=np.int64)


def hadamard_signs(d: int, seed: int = 0) -> np.ndarray:
    """Seeded +-1 diagonal (fp32) for the rotation applied before FP8 quantisation."""
    g = _philox(seed, 1 << 20 | 13, d, 0)
    return np.where(g.random(d) < 0.5, -1.0, 1.0).astype(np.float32)

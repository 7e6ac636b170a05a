"""Exact scaled-dot-product attention in fp64 -- TEST INFRASTRUCTURE ONLY.

Only tests, the smoke check and the bench's CPU baseline use this module; the
CUDA product path never imports it.

What is computed (the definition, not the tiled algorithm):

    s_ij  = scale * <q_i, k_j>            for j in J_i
    J_i   = {0..N-1}, or {0..i} when causal
    m_i   = max_j s_ij
    e_ij  = exp(s_ij - m_i)
    l_i   = sum_j e_ij
    O_i   = sum_j (e_ij / l_i) v_j
    LSE_i = m_i + ln(l_i)

Citations:

* The definition Softmax(Q K^T / sqrt(d)) V -- "FlashAttention-3" explainer
  (droidorbit.com), opening paragraph; the FAQ on linear attention states the
  method is exact, so the oracle is the definition itself.
* The statistics m (running max) and l (sum of exponentials) and the final
  normalisation -- "FlashAttention-3: como exprimir H100 al limite con
  atencion IO-aware" (dibro.site), "Arquitectura y metodo"; droidorbit.com,
  "Mathematical Formulation: The Online Softmax Rescaling Trick" (the
  streaming result equals the global softmax).
* Causal attention with the upper-triangular blocks skipped -- dibro.site,
  "Contribuciones clave".  With equal query and key lengths the mask keeps
  keys j <= i (a reading: the pages do not spell the alignment out).
* LSE is the natural-log log-sum-exp of the scaled scores, returned in fp64
  (a reading: the pages do not define an LSE output).

``scale`` is an argument; the workloads use 1/sqrt(d) as in the definition.
The one library primitive used is the fp64 matrix product.
"""

from __future__ import annotations

import numpy as np


def _as_f64(x) -> np.ndarray:
    """Widen a numpy array or a CPU torch tensor (any float dtype) to fp64."""
    if hasattr(x, "detach"):  # torch tensor; bf16 has no numpy dtype
        import torch

        x = x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def scores(q, k, scale: float, causal: bool = False, rows=None) -> np.ndarray:
    """Masked scaled scores s_ij for one head, -inf where j is not in J_i.

    q: [N_q, d], k: [N, d].  ``rows`` selects query rows (default: all);
    causal masking uses the selected rows' absolute indices.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    n_q = q.shape[0]
    rows = np.arange(n_q) if rows is None else np.asarray(rows, dtype=np.int64)
    s = float(scale) * (q[rows] @ k.T)
    if causal:
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j <= rows[:, None], s, -np.inf)
    return s


def probabilities(q, k, scale: float, causal: bool = False, rows=None) -> np.ndarray:
    """Softmax of the masked scores: P_ij = exp(s_ij - m_i) / l_i (one head)."""
    s = scores(q, k, scale, causal, rows)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def attention_head(q, k, v, scale: float, causal: bool = False, rows=None):
    """Exact attention for one head.

    Returns (O [R, d_v] fp64, LSE [R] fp64) for the selected query rows.
    """
    s = scores(q, k, scale, causal, rows)
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    o = (e / l[:, None]) @ _as_f64(v)
    lse = m + np.log(l)
    return o, lse


def attention(q, k, v, scale: float, causal: bool = False, rows=None):
    """Exact attention over [B, H, N, d] inputs (fp64 result).

    ``rows`` (optional) is a sequence of query-row indices applied to every
    (b, h); the result then has shape [B, H, len(rows), d].
    Returns (O, LSE) with LSE shaped [B, H, R].
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    B, H, N, _ = q.shape
    R = N if rows is None else len(rows)
    o = np.empty((B, H, R, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
    return o, lse


def flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Nominal forward FLOP count 4*B*H*N^2*d, halved for causal.

    This is the convention the throughput figures use (two matmuls of
    2*N^2*d each per head); causal halves it exactly.
    """
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f

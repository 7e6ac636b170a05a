"""Attention with fewer queries than keys, and the split-KV merge, in fp64 --
TEST INFRASTRUCTURE ONLY.

Only tests and the bench's CPU baseline use this module; the CUDA product
path never imports it.

* Decode alignment (a reading: the pages do not spell it out).  With Nq
  queries against Nk keys, query i stands at position Nk - Nq + i (the last
  Nq positions of the sequence), so causal masking keeps keys
  j <= Nk - Nq + i.  With Nq = Nk this is the forward's mask.  Otherwise the
  computation is the definition Softmax(Q K^T * scale) V ("FlashAttention-3"
  explainer, droidorbit.com, opening definition).
* Split-KV merge.  The pages contrast FlashAttention-3 with FlashDecoding,
  which parallelises decoding over the key/value length (droidorbit.com, FAQ
  "How does FlashAttention-3 compare to FlashDecoding?").  Partial results
  over disjoint key sets J_s combine by the online-softmax rescaling
  (droidorbit.com, "Mathematical Formulation: The Online Softmax Rescaling
  Trick"): with LSE_s = ln sum_{j in J_s} exp(s_j) and O_s the attention
  output over J_s alone,

      LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.

  A split with no visible key has LSE_s = -inf and weight 0.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64


def scores_kv(q, k, scale: float, causal: bool = False, rows=None) -> np.ndarray:
    """Masked scaled scores for Nq queries against Nk keys (one head); -inf
    where the key is not visible.  ``rows`` selects query rows."""
    q = _as_f64(q)
    k = _as_f64(k)
    nq, nk = q.shape[0], k.shape[0]
    rows = np.arange(nq) if rows is None else np.asarray(rows, dtype=np.int64)
    s = float(scale) * (q[rows] @ k.T)
    if causal:
        pos = nk - nq + rows
        j = np.arange(nk)[None, :]
        s = np.where(j <= pos[:, None], s, -np.inf)
    return s


def attention_kv_head(q, k, v, scale: float, causal: bool = False, rows=None, keys=None):
    """(O [R, d], LSE [R]) of one head for Nq queries against Nk keys.

    ``keys`` (optional) restricts the keys to that index set (the partial
    result of one split); rows that see no key there get O = 0, LSE = -inf.
    """
    s = scores_kv(q, k, scale, causal, rows)
    vv = _as_f64(v)
    if keys is not None:
        keys = np.asarray(keys, dtype=np.int64)
        s = s[:, keys]
        vv = vv[keys]
    m = s.max(axis=1)
    o = np.zeros((s.shape[0], vv.shape[1]))
    lse = np.full(s.shape[0], -np.inf)
    ok = np.isfinite(m)
    e = np.exp(s[ok] - m[ok, None])
    l = e.sum(axis=1)
    o[ok] = (e / l[:, None]) @ vv
    lse[ok] = m[ok] + np.log(l)
    return o, lse


def attention_kv(q, k, v, scale: float, causal: bool = False, rows=None):
    """(O, LSE) over [B, H, Nq, d] queries and [B, H, Nk, d] keys / values."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, nq, _ = q.shape
    R = nq if rows is None else len(rows)
    o = np.empty((B, H, R, v.shape[-1]))
    lse = np.empty((B, H, R))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_kv_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
    return o, lse


def merge_splits(parts):
    """Combine [(O_s [R, d], LSE_s [R]), ...] over disjoint key sets."""
    lses = np.stack([p[1] for p in parts])          # [S, R]
    outs = np.stack([p[0] for p in parts])          # [S, R, d]
    mx = lses.max(axis=0)
    ok = np.isfinite(mx)
    w = np.zeros_like(lses)
    w[:, ok] = np.exp(lses[:, ok] - mx[None, ok])
    tot = w.sum(axis=0)
    o = np.zeros(outs.shape[1:])
    o[ok] = np.einsum("sr,srd->rd", w[:, ok], outs[:, ok]) / tot[ok, None]
    lse = np.full(mx.shape, -np.inf)
    lse[ok] = mx[ok] + np.log(tot[ok])
    return o, lse


def flops_kv(B: int, H: int, Nq: int, Nk: int, d: int) -> float:
    """Nominal FLOP count of the two products, 4*B*H*Nq*Nk*d (no causal
    discount: decode shapes see nearly every key)."""
    return 4.0 * B * H * Nq * Nk * d

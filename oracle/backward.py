"""Gradients of exact attention in fp64 -- TEST INFRASTRUCTURE ONLY.

Only tests and the bench's CPU baseline use this module; the CUDA product
path never imports it.

The pages benchmark the backward pass next to the forward one (quantum-bit
repost "H100 utilisation 75% ... FlashAttention-3", attention benchmark:
forward and backward over the sequence sweep; backward 1.5-1.75x faster than
FlashAttention-2) but do not write it out; it is the chain rule applied to
the definition of the forward pass (the "FlashAttention-3" explainer,
droidorbit.com, opening definition):

    S  = scale * Q K^T   (masked to -inf above the diagonal when causal)
    P  = softmax_rows(S),    O = P V
    dV = P^T dO
    dP = dO V^T
    D  = rowsum(dO * O)      (= rowsum(P * dP))
    dS = P * (dP - D)
    dQ = scale * dS K,       dK = scale * dS^T Q

LSE is not differentiated (it is an auxiliary output).
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64, probabilities


def attention_backward_head(q, k, v, do, scale: float, causal: bool = False):
    """(dQ, dK, dV) of one head, fp64, for output gradient ``do``."""
    q, k, v, do = (_as_f64(x) for x in (q, k, v, do))
    p = probabilities(q, k, scale, causal)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    dvec = np.sum(do * o, axis=1, keepdims=True)
    ds = p * (dp - dvec)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def attention_backward(q, k, v, do, scale: float, causal: bool = False):
    """(dQ, dK, dV) over [B, H, N, d] inputs (fp64)."""
    q, k, v, do = (_as_f64(x) for x in (q, k, v, do))
    dq, dk, dv = (np.empty_like(q) for _ in range(3))
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            dq[b, h], dk[b, h], dv[b, h] = attention_backward_head(q[b, h], k[b, h], v[b, h], do[b, h],
                                                                   scale, causal)
    return dq, dk, dv


def row_dot(do, o) -> np.ndarray:
    """D = rowsum(dO * O) over the last axis (fp64)."""
    return np.sum(_as_f64(do) * _as_f64(o), axis=-1)


def backward_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Nominal backward FLOP count: five N x N x d products, 10*B*H*N^2*d,
    halved for causal (2.5x the forward convention)."""
    f = 10.0 * B * H * N * N * d
    return f / 2.0 if causal else f

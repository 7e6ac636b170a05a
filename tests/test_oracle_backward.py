"""Pins for the backward oracle (CPU only)."""

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import backward as Bw


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_float64(causal):
    """torch autograd of the SDPA definition (float64) is an independent
    differentiation of the same function."""
    n, d, scale = 37, 16, 0.3
    q, k, v, do = (_rand((n, d), s) for s in (1, 2, 3, 4))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(do))
    dq, dk, dv = Bw.attention_backward_head(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-13)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-13)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    n, d, scale = 6, 3, 0.7
    q, k, v, do = (_rand((n, d), s) for s in (5, 6, 7, 8))
    dq, dk, dv = Bw.attention_backward_head(q, k, v, do, scale, causal)

    def loss(q_, k_, v_):
        o, _ = A.attention_head(q_, k_, v_, scale, causal)
        return float(np.sum(o * do))

    eps = 1e-6
    for x, g, pos in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[pos], args_m[pos] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7)


def test_constant_v_has_no_q_or_k_gradient():
    """If every row of V is the same, O does not depend on Q or K."""
    n, d = 20, 8
    q, k, do = _rand((n, d), 9), _rand((n, d), 10), _rand((n, d), 11)
    v = np.tile(_rand((d,), 12), (n, 1))
    for causal in (False, True):
        dq, dk, dv = Bw.attention_backward_head(q, k, v, do, 0.5, causal)
        np.testing.assert_allclose(dq, 0, atol=1e-13)
        np.testing.assert_allclose(dk, 0, atol=1e-13)
        np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)  # columns of P sum over rows


def test_causal_row0_query_gradient_is_zero():
    n, d = 10, 4
    q, k, v, do = (_rand((n, d), s) for s in (13, 14, 15, 16))
    dq, _, _ = Bw.attention_backward_head(q, k, v, do, 0.9, causal=True)
    np.testing.assert_allclose(dq[0], 0, atol=1e-14)


def test_row_dot_equals_rowsum_p_dp():
    n, d, scale = 15, 8, 0.4
    q, k, v, do = (_rand((n, d), s) for s in (17, 18, 19, 20))
    p = A.probabilities(q, k, scale)
    o = p @ v
    np.testing.assert_allclose(Bw.row_dot(do, o), np.sum(p * (do @ v.T), axis=1), atol=1e-12)


def test_planted_sign_mistake_is_caught():
    """A backward with dS = P * (D - dP) (sign flipped) fails the autograd pin."""
    n, d, scale = 9, 4, 0.5
    q, k, v, do = (_rand((n, d), s) for s in (21, 22, 23, 24))
    p = A.probabilities(q, k, scale)
    o = p @ v
    ds_bad = p * (np.sum(do * o, axis=1, keepdims=True) - do @ v.T)
    dq_bad = scale * ds_bad @ k
    dq, _, _ = Bw.attention_backward_head(q, k, v, do, scale)
    assert not np.allclose(dq_bad, dq, atol=1e-6)

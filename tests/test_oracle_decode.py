"""Pins of oracle/decode.py (CPU): Nq < Nk attention with the decode causal
alignment, and the split-KV merge rule."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import attention as A
from oracle import decode as DC


def _qkv(nq, nk, d, seed):
    q = inputs.head_bf16(seed, "q", 0, 0, nq, d)
    k = inputs.head_bf16(seed, "k", 0, 0, nk, d)
    v = inputs.head_bf16(seed, "v", 0, 0, nk, d)
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_reduce_to_the_forward_oracle(causal):
    q, k, v = _qkv(50, 50, 16, 1)
    o, l = DC.attention_kv_head(q, k, v, 0.25, causal)
    o2, l2 = A.attention_head(q, k, v, 0.25, causal)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, l2, rtol=0, atol=1e-13)


def test_single_query_causal_sees_every_key():
    """Nq = 1 sits at the last position: causal equals non-causal."""
    q, k, v = _qkv(1, 77, 32, 2)
    o, l = DC.attention_kv_head(q, k, v, 0.2, True)
    o2, l2 = DC.attention_kv_head(q, k, v, 0.2, False)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(l, l2)


def test_decode_alignment_mask_shape():
    """Query i sees exactly Nk - Nq + i + 1 keys."""
    q, k, _ = _qkv(5, 12, 8, 3)
    s = DC.scores_kv(q, k, 1.0, True)
    assert [int(np.isfinite(r).sum()) for r in s] == [12 - 5 + i + 1 for i in range(5)]


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64_with_bottom_right_mask(causal):
    nq, nk, d = 9, 40, 16
    q, k, v = _qkv(nq, nk, d, 4)
    qt, kt, vt = (x.to(torch.float64)[None, None] for x in (q, k, v))
    mask = None
    if causal:
        mask = torch.arange(nk)[None, :] <= (nk - nq + torch.arange(nq))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
    o, _ = DC.attention_kv_head(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, ref[0, 0].numpy(), rtol=0, atol=1e-12)


def test_brute_force_tiny():
    q, k, v = _qkv(2, 5, 3, 5)
    qf, kf, vf = (x.double().numpy() for x in (q, k, v))
    o, l = DC.attention_kv_head(q, k, v, 0.7, True)
    for i in range(2):
        keys = range(5 - 2 + i + 1)
        s = [0.7 * math.fsum(qf[i, t] * kf[j, t] for t in range(3)) for j in keys]
        mx = max(s)
        e = [math.exp(x - mx) for x in s]
        tot = math.fsum(e)
        assert abs(l[i] - (mx + math.log(tot))) < 1e-12
        for c in range(3):
            assert abs(o[i, c] - math.fsum(e[jj] * vf[j, c] for jj, j in enumerate(keys)) / tot) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cuts", [[0, 40, 100], [0, 1, 2, 99, 100], [0, 100]])
def test_merge_of_splits_equals_whole(causal, cuts):
    """Partial results over disjoint key ranges merge to the full attention,
    including splits where some rows see no key (causal)."""
    q, k, v = _qkv(30, 100, 16, 6)
    parts = [DC.attention_kv_head(q, k, v, 0.25, causal, keys=np.arange(a, b)) for a, b in zip(cuts[:-1], cuts[1:])]
    o, l = DC.merge_splits(parts)
    o2, l2 = DC.attention_kv_head(q, k, v, 0.25, causal)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, l2, rtol=0, atol=1e-12)


def test_empty_split_has_no_weight():
    q, k, v = _qkv(4, 64, 8, 7)
    o, l = DC.attention_kv_head(q, k, v, 0.5, True, keys=np.arange(63, 64))
    # query 3 (position 63) sees key 63; queries 0-2 see no key in {63}
    assert np.isneginf(l[:3]).all() and np.isfinite(l[3])
    assert (o[:3] == 0).all()


@pytest.mark.parametrize("mutant", ["no_max_shift_weights", "plain_average", "lse_sum"])
def test_merge_pin_catches_planted_mistakes(mutant):
    q, k, v = _qkv(6, 50, 8, 8)
    parts = [DC.attention_kv_head(q, k, v, 0.5, False, keys=np.arange(a, b)) for a, b in ((0, 10), (10, 50))]
    lses = np.stack([p[1] for p in parts])
    outs = np.stack([p[0] for p in parts])
    if mutant == "no_max_shift_weights":
        w = lses / lses.sum(axis=0)                           # weights from LSE values, not exp
        o = np.einsum("sr,srd->rd", w, outs)
    elif mutant == "plain_average":
        o = outs.mean(axis=0)
    else:
        o = np.einsum("sr,srd->rd", np.exp(lses), outs)       # unnormalised
    ref, _ = DC.attention_kv_head(q, k, v, 0.5, False)
    assert np.abs(o - ref).max() > 1e-3
    good, _ = DC.merge_splits(parts)
    assert np.abs(good - ref).max() < 1e-12

"""GPU parity of the split-KV forward (attn_fwd_splitkv) against the fp64
decode oracle, through the C ABI, on seeded synthetic inputs.  Same bar as
the forward: max |dO| <= 2e-2, RMSE <= 3e-3, |dLSE| <= 1e-3."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import decode as DC
from parity_util import assert_bf16_ok, errors

pytestmark = pytest.mark.gpu


def _qkv(B, H, Nq, Nk, d, seed, dtype=torch.bfloat16):
    q = torch.empty((B, H, Nq, d), dtype=dtype)
    k = torch.empty((B, H, Nk, d), dtype=dtype)
    v = torch.empty((B, H, Nk, d), dtype=dtype)
    for b in range(B):
        for h in range(H):
            q[b, h] = torch.from_numpy(inputs.head_f32(seed, "q", b, h, Nq, d)).to(dtype)
            k[b, h] = torch.from_numpy(inputs.head_f32(seed, "k", b, h, Nk, d)).to(dtype)
            v[b, h] = torch.from_numpy(inputs.head_f32(seed, "v", b, h, Nk, d)).to(dtype)
    return q, k, v


def _run(lib, B, H, Nq, Nk, d, causal, n_splits=0, seed=0, dtype=torch.bfloat16, heads=None):
    q, k, v = _qkv(B, H, Nq, Nk, d, seed, dtype)
    scale = 1.0 / math.sqrt(d)
    o, lse = lib.fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, n_splits=n_splits)
    torch.cuda.synchronize()
    code, where = lib.last_status()
    assert code == 0, where
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    refs = [DC.attention_kv_head(q[b, h], k[b, h], v[b, h], scale, causal) for b, h in heads]
    o_ref = np.stack([r[0] for r in refs])
    l_ref = np.stack([r[1] for r in refs])
    o_g = torch.stack([o[b, h] for b, h in heads]).cpu()
    l_g = torch.stack([lse[b, h] for b, h in heads]).cpu()
    return errors(o_g, l_g, o_ref, l_ref)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 128), (1, 129), (1, 4096), (7, 1000), (16, 3000), (128, 2048),
                                   (129, 700), (300, 300), (1, 20000)])
def test_shapes(lib, d, causal, Nq, Nk):
    err = _run(lib, 2, 3, Nq, Nk, d, causal, seed=Nq + Nk)
    assert_bf16_ok(err, (Nq, Nk, d, causal))


@pytest.mark.parametrize("n_splits", [1, 2, 3, 7, 31, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_split_counts(lib, n_splits, causal):
    """Explicit split counts, including one split (no merge) and more splits
    than key tiles (clamped)."""
    err = _run(lib, 1, 4, 5, 3900, 128, causal, n_splits=n_splits, seed=n_splits)
    assert_bf16_ok(err, (n_splits, causal))


@pytest.mark.parametrize("d", [8, 40, 96, 120, 136, 248])
def test_head_dims_padded(lib, d):
    err = _run(lib, 1, 2, 3, 1500, d, True, seed=d)
    assert_bf16_ok(err, ("d", d))


@pytest.mark.parametrize("causal", [False, True])
def test_fp16(lib, causal):
    err = _run(lib, 2, 2, 10, 2500, 128, causal, dtype=torch.float16, seed=3)
    assert_bf16_ok(err, ("fp16", causal))


def test_many_heads_wrap_the_grid(lib):
    err = _run(lib, 4, 32, 1, 5000, 128, True, n_splits=4, seed=9, heads=[(0, 0), (1, 13), (3, 31)])
    assert_bf16_ok(err, "wrap")


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_attn_fwd(lib, causal):
    """With Nq = Nk the split path computes attn_fwd's attention; the two
    kernels round differently (P per split, fp32 merge), so they agree to the
    parity bar, not bitwise."""
    q, k, v = (t.cuda() for t in inputs.qkv(1, 2, 640, 128, seed=12))
    o1, l1 = lib.fwd(q, k, v, causal=causal)
    o2, l2 = lib.fwd_splitkv(q, k, v, causal=causal, n_splits=3)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_workspace_contents_irrelevant_and_repeatable(lib):
    q, k, v = (t.cuda() for t in _qkv(2, 4, 3, 4000, 128, 21))
    ns = int(lib.lib().attn_fwd_splitkv_auto_splits(2, 4, 3, 4000))
    ws = torch.full((int(lib.lib().attn_fwd_splitkv_workspace_bytes(2, 4, 3, 128, ns)),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    a = lib.fwd_splitkv(q, k, v, causal=True, n_splits=ns, workspace=ws)
    b = lib.fwd_splitkv(q, k, v, causal=True, n_splits=ns)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_auto_split_count_covers_the_sms(lib):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ns = int(lib.lib().attn_fwd_splitkv_auto_splits(2, 8, 1, 32768))
    assert 1 <= ns <= 32768 // 128 // 2
    assert 16 * ns >= sms


def test_bad_arguments_raise(lib):
    q = torch.zeros(1, 1, 4, 264, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError):
        lib.fwd_splitkv(q, q, q)
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError):
        lib.fwd_splitkv(q, k, k, causal=True)   # more queries than keys

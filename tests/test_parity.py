"""GPU parity of the 16-bit tcgen05 forward kernel against the fp64 oracle,
called through the C ABI (ctypes binding) on seeded synthetic inputs."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import attention as A
from parity_util import assert_bf16_ok, errors, run_and_compare

pytestmark = pytest.mark.gpu


def test_small_workload_full(lib):
    """B=1, H=1, N=128, d=64, non-causal, seed 0: every row against the oracle."""
    err, _ = run_and_compare(lib, 1, 1, 128, 64, False)
    assert_bf16_ok(err, "small workload")
    code, where = lib.last_status()
    assert code == 0, where


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 100, 127, 128, 129, 255, 256, 257, 500, 1000])
def test_ragged_and_multi_tile(lib, d, causal, N):
    err, _ = run_and_compare(lib, 1, 2, N, d, causal, seed=N)
    assert_bf16_ok(err, (N, d, causal))


@pytest.mark.parametrize("d", [8, 40, 96, 136, 200, 248])
@pytest.mark.parametrize("causal", [False, True])
def test_head_dims_padded(lib, d, causal):
    """Head dims that are not 64, 128 or 256 run zero-padded to the next of
    those (the padding changes no score and no stored column)."""
    err, _ = run_and_compare(lib, 1, 3, 333, d, causal, seed=d)
    assert_bf16_ok(err, ("d", d, causal))


@pytest.mark.parametrize("d", [64, 256])
def test_hidden_2048_sweep_shape(lib, d):
    """Sweep shapes with hidden size 2048 (H = 2048 / d), total tokens 16K."""
    N = 2048
    rows = inputs.sample_rows(N, 32, seed=7)
    err, _ = run_and_compare(lib, 16384 // N, 2048 // d, N, d, True, rows=rows,
                             heads=[(0, 0), (7, 2048 // d - 1)])
    assert_bf16_ok(err, ("hidden 2048", d))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_fp16(lib, d, causal):
    err, _ = run_and_compare(lib, 2, 3, 300, d, causal, dtype=torch.float16, seed=5)
    assert_bf16_ok(err, ("fp16", d, causal))


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_persistent_grid_wraps(lib, causal, d):
    """More work units than SMs, so each CTA takes several of them."""
    err, _ = run_and_compare(lib, 2, 96, 512, d, causal, seed=3)
    assert_bf16_ok(err, ("wrap", causal, d))


@pytest.mark.parametrize("causal", [False, True])
def test_headline_shape_sampled_rows(lib, causal):
    """B=4, H=16, N=8192, d=128: 64 sampled rows per head, every head."""
    rows = inputs.sample_rows(8192, 64, seed=1)
    err, (o, lse) = run_and_compare(lib, 4, 16, 8192, 128, causal, rows=rows)
    assert_bf16_ok(err, ("8k", causal))
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("N,d", [(512, 64), (2048, 128), (16384, 64), (16384, 128), (1024, 256),
                                 (16384, 256)])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_sweep_sampled(lib, N, d, causal):
    """Sweep shapes: total tokens B*N = 16K, H = 16; sampled heads and rows."""
    B = 16384 // N
    rows = inputs.sample_rows(N, 48, seed=2)
    heads = [(0, 0), (B - 1, 15), (B // 2, 7)]
    err, _ = run_and_compare(lib, B, 16, N, d, causal, rows=rows, heads=heads)
    assert_bf16_ok(err, ("sweep", N, d, causal))


def test_long_context_causal_sampled(lib):
    """B=1, H=32, N=65536, d=128 causal: stratified rows on a few heads."""
    N = 65536
    rows = inputs.stratified_rows(N, 256, seed=4)
    err, _ = run_and_compare(lib, 1, 32, N, 128, True, rows=rows, heads=[(0, 0), (0, 31)])
    assert_bf16_ok(err, "64k causal")


# ---------------------------------------------------------------- edge cases

def _dev(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_closed_form(lib, causal):
    q, k, _ = inputs.qkv(1, 2, 333, 128, seed=9)
    v = torch.empty_like(q)
    c = torch.randn(128, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    v[:] = c
    o, _ = lib.fwd(*_dev(q, k, v), causal=causal)
    torch.cuda.synchronize()
    want = c.double().expand(1, 2, 333, 128).numpy()
    err = errors(o.cpu(), None, want, None)
    # P rows sum to 1 in fp32 up to rounding of P to bf16: a few bf16 ulps of |c|
    assert err["max_abs"] <= 2e-2, err


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_is_uniform_attention(lib, causal):
    _, k, v = inputs.qkv(1, 1, 300, 64, seed=10)
    q = torch.zeros_like(k)
    o, lse = lib.fwd(*_dev(q, k, v), causal=causal)
    torch.cuda.synchronize()
    vv = v[0, 0].double().numpy()
    if causal:
        want = np.cumsum(vv, axis=0) / np.arange(1, 301)[:, None]
        lwant = np.log(np.arange(1, 301))
    else:
        want = np.broadcast_to(vv.mean(axis=0), vv.shape)
        lwant = np.full(300, math.log(300))
    err = errors(o[0, 0].cpu(), lse[0, 0].cpu(), want, lwant)
    assert err["max_abs"] <= 2e-2 and err["lse_max_abs"] <= 1e-3, err


def test_causal_row0_and_two_token_example(lib):
    """The hand-worked two-token example embedded in d=64 by zero padding."""
    q = torch.zeros(1, 1, 2, 64)
    k = torch.zeros(1, 1, 2, 64)
    v = torch.zeros(1, 1, 2, 64)
    q[0, 0, 1, 0] = 1.0
    k[0, 0, 1, 0] = math.log(3.0)
    v[0, 0, 1, 0] = 1.0
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    k13 = float(k[0, 0, 1, 0])  # bf16(ln 3): recompute the expected values from it
    for causal in (False, True):
        o, lse = lib.fwd(*_dev(q, k, v), causal=causal, scale=1.0)
        torch.cuda.synchronize()
        p1 = math.exp(k13) / (1 + math.exp(k13))
        o0 = 0.0 if causal else 0.5
        l0 = 0.0 if causal else math.log(2.0)
        assert abs(float(o[0, 0, 0, 0]) - o0) <= 4e-3
        assert abs(float(o[0, 0, 1, 0]) - p1) <= 4e-3
        assert abs(float(lse[0, 0, 0]) - l0) <= 1e-4
        assert abs(float(lse[0, 0, 1]) - math.log(1 + math.exp(k13))) <= 1e-4
        assert float(o[0, 0, :, 1:].abs().max()) == 0.0


def test_large_scores_stay_finite(lib):
    """Scores of magnitude ~1e3 exercise the max tracking and rescaling."""
    q, k, v = inputs.qkv(1, 2, 640, 64, seed=11)
    q = (q.float() * 30).to(torch.bfloat16)
    o, lse = lib.fwd(*_dev(q, k, v), causal=False, scale=1.0)
    torch.cuda.synchronize()
    o_ref, l_ref = A.attention(q, k, v, 1.0, False)
    err = errors(o.cpu(), lse.cpu(), o_ref, l_ref)
    # scores reach a few hundred: fp32 accumulation error of LSE scales with them
    assert err["max_abs"] <= 2e-2 and err["lse_max_abs"] <= 1e-2, err


def test_deterministic(lib):
    q, k, v = _dev(*inputs.qkv(2, 4, 1000, 128, seed=12))
    o1, l1 = lib.fwd(q, k, v, causal=True)
    o2, l2 = lib.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_may_be_omitted_and_stream_respected(lib):
    q, k, v = _dev(*inputs.qkv(1, 2, 256, 64, seed=13))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        o, lse = lib.fwd(q, k, v, return_lse=False)
    s.synchronize()
    assert lse is None
    o2, _ = lib.fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)
    assert lib.last_status()[0] == 0


@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (256, False), (96, True)])
def test_strided_bshd_views_match_contiguous(lib, d, causal):
    """[B, N, H, d] (BSHD) tensors passed as transposed views, and an output
    written into a BSHD buffer, give bit-identical results to the contiguous
    path; both match the oracle."""
    B, H, N = 2, 3, 300
    q, k, v = inputs.qkv(B, H, N, d, seed=21)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_ref, l_ref = lib.fwd(qd, kd, vd, causal=causal)
    qs, ks, vs = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (qd, kd, vd))
    assert not qs.is_contiguous()
    o_buf = torch.empty(B, N, H, d, dtype=q.dtype, device="cuda")
    o_s, l_s = lib.fwd(qs, ks, vs, causal=causal, out=o_buf.transpose(1, 2))
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_ref) and torch.equal(l_s, l_ref)
    assert torch.equal(o_buf.transpose(1, 2), o_ref)
    err = errors(o_s.cpu(), l_s.cpu(), *A.attention(q, k, v, 1 / math.sqrt(d), causal))
    assert_bf16_ok(err, ("bshd", d))


def test_strided_padded_rows_and_mixed_layouts(lib):
    """Rows with padding between them (row stride > d) and a different layout
    per tensor."""
    B, H, N, d = 1, 2, 257, 64
    q, k, v = inputs.qkv(B, H, N, d, seed=22)
    big = torch.zeros(B, H, N, d + 32, dtype=q.dtype)
    big[..., :d] = k
    kp = big.cuda()[..., :d]                       # row stride d + 32
    assert kp.stride(2) == d + 32
    qs = q.transpose(1, 2).contiguous().cuda().transpose(1, 2)
    o, lse = lib.fwd(qs, kp, v.cuda())
    torch.cuda.synchronize()
    err = errors(o.cpu(), lse.cpu(), *A.attention(q, k, v, 1 / math.sqrt(d), False))
    assert_bf16_ok(err, "padded rows")


@pytest.mark.parametrize("causal,N", [(False, 1000), (True, 777), (True, 2048)])
def test_serialised_tile_schedule_is_bit_identical(lib, causal, N):
    """The ablation switch (attn_debug_set_ablation) changes only the
    schedule of the two query tiles, not the arithmetic: outputs are equal
    bit for bit to the ping-pong schedule's.  Other head dims are refused
    while it is on."""
    q, k, v = (t.cuda() for t in inputs.qkv(1, 3, N, 128, seed=N))
    o0, l0 = lib.fwd(q, k, v, causal=causal)
    x64 = q[..., :64].contiguous()
    try:
        lib.debug_set_ablation(1)
        o1, l1 = lib.fwd(q, k, v, causal=causal)
        with pytest.raises(lib.AttnError) as e:
            lib.fwd(x64, x64, x64)
        assert e.value.code == lib.ATTN_ERR_UNSUPPORTED
    finally:
        lib.debug_set_ablation(0)
    torch.cuda.synchronize()
    assert lib.last_status()[0] == 0
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_single_key_with_negative_score_returns_v(lib, d, causal):
    """N = 1: the only key gets P = 1, so O = V bit for bit and LSE = the
    score, also when that score is negative and every other column of the
    128-key tile is masked (the row max must see only the masked tile: a max
    that also took in the masked columns' zero scores would lift m to 0,
    round P = exp(s) < 1 to 16 bits and move O off V)."""
    q = inputs.qkv(2, 3, 1, d, seed=d)[0]
    k = -q                                          # <q, k> < 0 for every head
    v = inputs.qkv(2, 3, 1, d, seed=d + 1)[2]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = lib.fwd(qd, kd, vd, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, vd)
    s = (q.double() * k.double()).sum(-1) / math.sqrt(d)
    assert float((lse.double().cpu() - s).abs().max()) <= 1e-5 * max(1.0, float(s.abs().max()))

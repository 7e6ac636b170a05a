"""GPU checks of the FP8 path: the quantisation kernel against the oracle's
per-block e4m3 quantiser, and FP8 attention against the fp64 oracle on
Gaussian inputs with outliers (with and without Hadamard rotation)."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import attention as A
from oracle import fp8 as F
from parity_util import FP8_RMSE, errors

pytestmark = pytest.mark.gpu


def _x(B, H, N, d, seed, outliers=True):
    return inputs.qkv(B, H, N, d, seed=seed, outliers=outliers)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [128, 300, 1024])
def test_quant_plain_bit_exact(lib, d, N):
    x = _x(2, 3, N, d, seed=N)[0]
    codes, desc = lib.quant_fp8(x.cuda())
    torch.cuda.synchronize()
    c_ref, d_ref, _ = F.quantize_blocks(x.double().numpy())
    np.testing.assert_array_equal(desc.cpu().numpy(), d_ref)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("signed", [False, True])
def test_quant_hadamard_close(lib, d, signed):
    """With rotation the kernel's fp32 butterflies round differently from the
    oracle's fp64 product: scales agree to fp32 rounding, codes agree except
    where the value sits next to a rounding boundary (then one step apart)."""
    x = _x(1, 4, 640, d, seed=7)[1]
    signs = inputs.hadamard_signs(d, seed=3) if signed else None
    codes, desc = lib.quant_fp8(x.cuda(), hadamard=True,
                                signs=torch.from_numpy(signs) if signed else None)
    torch.cuda.synchronize()
    c_ref, d_ref, y = F.quantize_blocks(x.double().numpy(), True, signs)
    np.testing.assert_allclose(desc.cpu().numpy(), d_ref, rtol=2e-6)
    c = codes.cpu().numpy()
    diff = c != c_ref
    assert diff.mean() < 2e-3, diff.mean()
    # where they differ both decode within one e4m3 step of y / s
    vals = F.e4m3_decode(c)
    s = np.repeat(d_ref.astype(np.float64), 128, axis=2)[:, :, :640, None]
    t = y / s
    step = np.maximum(np.abs(t) * 2.0 ** -3, 2.0 ** -9)
    assert np.all(np.abs(vals[diff] - t[diff]) <= step[diff])


@pytest.mark.parametrize("d,B,H,N", [(128, 1, 16, 32768 + 40), (64, 2, 8, 16384)])
def test_quant_ring_of_copies_sampled_heads(lib, d, B, H, N):
    """Sizes whose blocks outnumber the resident CTAs many times over, so each
    CTA cycles its ring of block copies several times: plain quantisation is
    bit-exact with the oracle on sampled heads (ragged last block included),
    and the rotated one agrees as in the small cases."""
    x = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            x[b, h] = inputs.head_bf16(11, "k", b, h, N, d, outliers=True)
    xc = x.cuda()
    codes, desc = lib.quant_fp8(xc)
    signs = inputs.hadamard_signs(d, seed=4)
    codes_r, desc_r = lib.quant_fp8(xc, hadamard=True, signs=torch.from_numpy(signs))
    torch.cuda.synchronize()
    assert lib.last_status()[0] == 0
    for b, h in [(0, 0), (B - 1, H // 2 + 1), (B - 1, H - 1)]:
        xh = x[b:b + 1, h:h + 1].double().numpy()
        c_ref, d_ref, _ = F.quantize_blocks(xh)
        np.testing.assert_array_equal(desc[b:b + 1, h:h + 1].cpu().numpy(), d_ref)
        np.testing.assert_array_equal(codes[b:b + 1, h:h + 1].cpu().numpy(), c_ref)
    c_ref, d_ref, _ = F.quantize_blocks(x[B - 1:B, H - 1:H].double().numpy(), True, signs)
    np.testing.assert_allclose(desc_r[B - 1:B, H - 1:H].cpu().numpy(), d_ref, rtol=2e-6)
    assert (codes_r[B - 1:B, H - 1:H].cpu().numpy() != c_ref).mean() < 2e-3


def _fp8_attention(lib, q, k, v, causal, hadamard, signs=None):
    sg = torch.from_numpy(signs) if signs is not None else None
    q8, qd = lib.quant_fp8(q.cuda(), hadamard=hadamard, signs=sg)
    k8, kd = lib.quant_fp8(k.cuda(), hadamard=hadamard, signs=sg)
    v8, vd = lib.quant_fp8(v.cuda())
    o, lse = lib.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=causal)
    torch.cuda.synchronize()
    return o, lse, (q8, k8, v8, qd, kd, vd)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("N", [128, 520])
def test_fp8_attention_vs_fp64_oracle(lib, causal, hadamard, N):
    q, k, v = _x(1, 4, N, 128, seed=30 + N)
    signs = inputs.hadamard_signs(128, seed=1)
    o, lse, packed = _fp8_attention(lib, q, k, v, causal, hadamard, signs)
    scale = 1 / math.sqrt(128)
    o_ref, l_ref = A.attention(q, k, v, scale, causal)
    err = errors(o.cpu(), lse.cpu(), o_ref, l_ref)
    assert err["rmse"] <= FP8_RMSE, err
    # tighter: exact attention on the dequantised operands isolates the
    # kernel's own arithmetic (P rounded to e4m3, fp32 accumulation)
    q8, k8, v8, qd, kd, vd = (t.cpu().numpy() for t in packed)
    qq = F.dequantize_blocks(q8, qd)
    kk = F.dequantize_blocks(k8, kd)
    vv = F.dequantize_blocks(v8, vd)
    o_q, l_q = A.attention(qq, kk, vv, scale, causal)
    err_q = errors(o.cpu(), lse.cpu(), o_q, l_q)
    assert err_q["rmse"] <= 1.5e-2 and err_q["lse_max_abs"] <= 5e-3, err_q


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("N", [1, 128, 300, 1500])
def test_fp8_head_dim_64(lib, causal, hadamard, N):
    """Head dim 64: 64-byte e4m3 rows (64-byte swizzle for TMA and the
    tensor-core operands), same parity bars as d = 128 against the fp64
    oracle on outlier inputs, and against exact attention on the
    dequantised operands.  (At N = 1 the output is one row of V after e4m3
    rounding, with nothing to average the rounding out: only the second
    comparison applies there.)"""
    q, k, v = _x(2, 3, N, 64, seed=40 + N)
    signs = inputs.hadamard_signs(64, seed=2)
    o, lse, packed = _fp8_attention(lib, q, k, v, causal, hadamard, signs)
    assert lib.last_status()[0] == 0
    scale = 1 / math.sqrt(64)
    if N > 1:
        o_ref, l_ref = A.attention(q, k, v, scale, causal)
        err = errors(o.cpu(), lse.cpu(), o_ref, l_ref)
        assert err["rmse"] <= FP8_RMSE, err
    q8, k8, v8, qd, kd, vd = (t.cpu().numpy() for t in packed)
    o_q, l_q = A.attention(F.dequantize_blocks(q8, qd), F.dequantize_blocks(k8, kd),
                           F.dequantize_blocks(v8, vd), scale, causal)
    err_q = errors(o.cpu(), lse.cpu(), o_q, l_q)
    assert err_q["rmse"] <= 1.5e-2 and err_q["lse_max_abs"] <= 5e-3, err_q


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("N", [1, 128, 300, 1500])
def test_fp8_head_dim_256(lib, causal, hadamard, N):
    """Head dim 256: the one-tile kernel with S double-buffered in TMEM, its
    e4m3 rows loaded as two 128-byte chunks; the rotation's last two
    butterfly stages cross lanes in the quantiser.  Same bars as d = 64 and
    128 (only the dequantised comparison at N = 1, as there)."""
    q, k, v = _x(2, 3, N, 256, seed=50 + N)
    signs = inputs.hadamard_signs(256, seed=5)
    o, lse, packed = _fp8_attention(lib, q, k, v, causal, hadamard, signs)
    assert lib.last_status()[0] == 0
    scale = 1 / math.sqrt(256)
    if N > 1:
        o_ref, l_ref = A.attention(q, k, v, scale, causal)
        err = errors(o.cpu(), lse.cpu(), o_ref, l_ref)
        assert err["rmse"] <= FP8_RMSE, err
    q8, k8, v8, qd, kd, vd = (t.cpu().numpy() for t in packed)
    o_q, l_q = A.attention(F.dequantize_blocks(q8, qd), F.dequantize_blocks(k8, kd),
                           F.dequantize_blocks(v8, vd), scale, causal)
    err_q = errors(o.cpu(), lse.cpu(), o_q, l_q)
    assert err_q["rmse"] <= 1.5e-2 and err_q["lse_max_abs"] <= 5e-3, err_q


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_head_dim_256_many_units(lib, causal):
    """Head dim 256 with several work units per CTA (4 x 16 heads x 8 row
    tiles = 512 units), sampled rows of three heads against the fp64
    oracle."""
    B, H, N = 4, 16, 1024
    q, k, v = _x(B, H, N, 256, seed=60)
    signs = inputs.hadamard_signs(256, seed=6)
    o, lse, _ = _fp8_attention(lib, q, k, v, causal, True, signs)
    assert lib.last_status()[0] == 0
    rows = inputs.sample_rows(N, 48, seed=9)
    scale = 1 / math.sqrt(256)
    for b, h in [(0, 0), (1, 7), (3, 15)]:
        o_ref, l_ref = A.attention_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
        err = errors(o[b, h][rows].cpu(), lse[b, h][rows].cpu(), o_ref, l_ref)
        assert err["rmse"] <= FP8_RMSE, (b, h, err)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_headline_shape_sampled(lib, causal):
    """B=4, H=16, N=8192, d=128 with outliers; Hadamard on; sampled rows."""
    q, k, v = _x(4, 16, 8192, 128, seed=0)
    signs = inputs.hadamard_signs(128, seed=0)
    o, lse, _ = _fp8_attention(lib, q, k, v, causal, True, signs)
    rows = inputs.sample_rows(8192, 32, seed=5)
    heads = [(0, 0), (1, 5), (3, 15)]
    scale = 1 / math.sqrt(128)
    for b, h in heads:
        o_ref, l_ref = A.attention_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
        err = errors(o[b, h][rows].cpu(), lse[b, h][rows].cpu(), o_ref, l_ref)
        assert err["rmse"] <= FP8_RMSE, (b, h, err)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 700, 2048])
def test_v_transpose_matches_mn_major(lib, causal, N):
    """The in-shared-memory V transpose feeds the same values to the tensor
    core in K-major order: the output equals the MN-major path's."""
    q, k, v = _x(2, 3, N, 128, seed=40 + N)
    signs = inputs.hadamard_signs(128, seed=2)
    sg = torch.from_numpy(signs)
    q8, qd = lib.quant_fp8(q.cuda(), hadamard=True, signs=sg)
    k8, kd = lib.quant_fp8(k.cuda(), hadamard=True, signs=sg)
    v8, vd = lib.quant_fp8(v.cuda())
    o0, l0 = lib.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=causal, v_transpose=False)
    o1, l1 = lib.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=causal, v_transpose=True)
    torch.cuda.synchronize()
    assert lib.last_status()[0] == 0
    # same products in the same order: bit-identical
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    o_ref, _ = A.attention(q, k, v, 1 / math.sqrt(128), causal)
    assert errors(o1.cpu(), None, o_ref, None)["rmse"] <= FP8_RMSE


def test_accuracy_vs_low_precision_baselines(lib):
    """The pages' accuracy experiment (outlier inputs): FP8 with per-block
    scales and Hadamard rotation is more accurate than a per-tensor FP8
    attention, and the fp16 kernel (fp32 statistics) more accurate than a
    standard fp16 attention that writes its softmax out in fp16.  The pages
    report 2.6x and 1.7x (baselines whose rounding they do not describe);
    measured here 1.59x and, for the fp16 baseline, 1.03x when only its
    softmax output is fp16 and more when its scores are rounded to fp16 as
    well; only the direction is asserted."""
    from oracle import baselines as Bl
    N, d = 1024, 128
    scale = 1 / math.sqrt(d)
    q, k, v = _x(1, 2, N, d, seed=77)
    signs = torch.from_numpy(inputs.hadamard_signs(d, seed=5))
    o8, _, _ = _fp8_attention(lib, q, k, v, False, True, inputs.hadamard_signs(d, seed=5))
    q16, k16, v16 = (t.to(torch.float16) for t in (q, k, v))
    o16, _ = lib.fwd(q16.cuda(), k16.cuda(), v16.cuda(), scale=scale)
    torch.cuda.synchronize()
    e8, e8b, e16, e16b, e16s = [], [], [], [], []
    for h in range(2):
        qq, kk, vv = (t[0, h].double().numpy() for t in (q, k, v))
        o_ref, _ = A.attention_head(qq, kk, vv, scale)
        e8.append(Bl.rmse(o8[0, h].double().cpu().numpy(), o_ref))
        e8b.append(Bl.rmse(Bl.per_tensor_fp8_attention(qq, kk, vv, scale), o_ref))
        q6, k6, v6 = (t[0, h].double().numpy() for t in (q16, k16, v16))
        o_ref16, _ = A.attention_head(q6, k6, v6, scale)
        e16.append(Bl.rmse(o16[0, h].double().cpu().numpy(), o_ref16))
        e16b.append(Bl.rmse(Bl.standard_fp16_attention(q6, k6, v6, scale), o_ref16))
        e16s.append(Bl.rmse(Bl.standard_fp16_attention(q6, k6, v6, scale, round_scores=True), o_ref16))
    ratio8 = float(np.mean(e8b) / np.mean(e8))
    ratio16 = float(np.mean(e16b) / np.mean(e16))
    ratio16s = float(np.mean(e16s) / np.mean(e16))
    print(f"RMSE ratios: per-tensor FP8 / ours {ratio8:.2f} (pages 2.6), standard fp16 / ours {ratio16:.2f} "
          f"(fp16 softmax output), {ratio16s:.2f} (fp16 scores and softmax output) (pages 1.7)")
    assert np.mean(e16) < np.mean(e16s), (e16, e16s)
    assert np.mean(e8) < np.mean(e8b), (e8, e8b)
    assert np.mean(e16) < np.mean(e16b), (e16, e16b)

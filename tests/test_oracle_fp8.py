"""Pins for the oracle's FP8 pieces (CPU only): e4m3 rounding, the Hadamard
rotation and per-block quantisation."""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import fp8 as F
from io_aware_attention_02_b200 import inputs


def test_e4m3_table_known_values():
    v = F.e4m3_values()
    assert v[0] == 0.0
    assert v[1] == 2.0 ** -9            # smallest subnormal
    assert v[7] == 7 * 2.0 ** -9        # largest subnormal
    assert v[8] == 2.0 ** -6            # smallest normal
    assert v[0x38] == 1.0
    assert v[126] == 448.0              # largest finite
    assert np.all(np.diff(v) > 0)
    assert math.isnan(F.e4m3_decode([0x7F])[0]) and math.isnan(F.e4m3_decode([0xFF])[0])
    assert F.e4m3_decode([0xB8])[0] == -1.0


def _torch_codes(x32):
    return torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_cast_random():
    """torch's float8_e4m3fn cast (round-to-nearest-even) is the library reference."""
    g = np.random.default_rng(0)
    x = np.concatenate([
        g.standard_normal(200000) * 50,
        g.standard_normal(20000) * 2.0 ** -7,          # subnormal range
        g.uniform(-448, 448, 20000),
    ]).astype(np.float32)
    np.testing.assert_array_equal(F.e4m3_encode(x), _torch_codes(x))


def test_e4m3_encode_ties_and_boundaries():
    v = F.e4m3_values()
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)   # exact midpoints (representable in fp32)
    assert np.all(mids.astype(np.float64) == (v[:-1] + v[1:]) / 2)
    x = np.concatenate([mids, -mids, v.astype(np.float32), np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1e9))]).astype(np.float32)
    np.testing.assert_array_equal(F.e4m3_encode(x), _torch_codes(x))
    # ties go to the even code
    codes = F.e4m3_encode(mids)
    assert np.all(codes % 2 == 0)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.9, 1e6, -1e6], dtype=np.float32)
    assert list(F.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_sylvester_hadamard():
    np.testing.assert_array_equal(F.sylvester_hadamard(2), [[1, 1], [1, -1]])
    for d in (1, 2, 4, 64, 128, 256):
        h = F.sylvester_hadamard(d)
        np.testing.assert_array_equal(h @ h.T, d * np.eye(d))
        np.testing.assert_array_equal(h, h.T)
    with pytest.raises(ValueError):
        F.sylvester_hadamard(96)


def test_rotation_is_orthogonal_and_keeps_qkt():
    d = 64
    s = inputs.hadamard_signs(d, seed=3)
    assert set(np.unique(s)) <= {-1.0, 1.0}
    r = F.rotation(d, s)
    np.testing.assert_allclose(r @ r.T, np.eye(d), atol=1e-14)
    g = np.random.default_rng(1)
    q, k, v = g.standard_normal((50, d)), g.standard_normal((50, d)), g.standard_normal((50, d))
    np.testing.assert_allclose(F.rotate(q, s) @ F.rotate(k, s).T, q @ k.T, atol=1e-12)
    for causal in (False, True):
        o1, l1 = A.attention_head(q, k, v, 0.125, causal)
        o2, l2 = A.attention_head(F.rotate(q, s), F.rotate(k, s), v, 0.125, causal)
        np.testing.assert_allclose(o2, o1, atol=1e-12)
        np.testing.assert_allclose(l2, l1, atol=1e-12)


def test_rotation_spreads_an_outlier():
    """A single large coordinate is spread evenly: |y_j| = |x| / sqrt(d)."""
    d = 128
    x = np.zeros(d)
    x[5] = 100.0
    y = F.rotate(x[None, :], inputs.hadamard_signs(d))[0]
    np.testing.assert_allclose(np.abs(y), 100.0 / math.sqrt(d), rtol=1e-14)


@pytest.mark.parametrize("hadamard", [False, True])
def test_quantize_blocks_scale_and_error_bound(hadamard):
    B, H, N, d = 1, 2, 300, 64          # 3 blocks, the last one ragged (44 rows)
    x = np.stack([np.stack([inputs.head_bf16(0, "q", b, h, N, d, outliers=True).float().numpy()
                            for h in range(H)]) for b in range(B)]).astype(np.float64)
    signs = inputs.hadamard_signs(d)
    codes, desc, y = F.quantize_blocks(x, hadamard, signs)
    assert codes.shape == x.shape and desc.shape == (B, H, 3)
    y32 = y.astype(np.float32)
    for t in range(3):
        blk = y32[:, :, t * 128:(t + 1) * 128]
        amax = np.abs(blk).max(axis=(2, 3))
        np.testing.assert_array_equal(desc[:, :, t], (amax / np.float32(448)).astype(np.float32))
        # the block's largest magnitude lands on (or next to) the top code
        mags = codes[:, :, t * 128:(t + 1) * 128] & 0x7F
        assert mags.max() >= 125
    deq = F.dequantize_blocks(codes, desc)
    s_full = np.repeat(desc.astype(np.float64), 128, axis=2)[:, :, :N, None]
    # e4m3: 3 mantissa bits -> relative error <= 2^-4 for normals; subnormal step 2^-9 * s
    err = np.abs(deq - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, s_full * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_quantize_zero_block_gives_unit_scale():
    x = np.zeros((1, 1, 130, 64))
    x[0, 0, 129, 3] = 2.0
    codes, desc, _ = F.quantize_blocks(x)
    assert desc[0, 0, 0] == 1.0 and np.all(codes[0, 0, :128] == 0)
    assert desc[0, 0, 1] == np.float32(2.0 / 448.0)
    assert codes[0, 0, 129, 3] == 0x7E


def test_quantize_blocks_planted_mistake_is_caught():
    """A quantiser that used one scale for the whole tensor fails the per-block scale pin."""
    x = np.zeros((1, 1, 256, 64))
    x[0, 0, :128] = 1.0
    x[0, 0, 128:] = 100.0
    codes, desc, _ = F.quantize_blocks(x)
    assert desc[0, 0, 0] == np.float32(1 / 448) and desc[0, 0, 1] == np.float32(100 / 448)
    per_tensor = np.float32(100 / 448)
    assert per_tensor != desc[0, 0, 0]

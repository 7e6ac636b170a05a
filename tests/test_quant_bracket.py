"""CPU check of the rounding argument the quantisation kernel relies on.

The kernel rounds y / s to e4m3 without dividing: with r = RN(1/s) nudged
down and up by a relative 2^-20 (r_lo, r_hi), the fp32 products RN(y r_lo)
and RN(y r_hi) bracket the IEEE quotient RN(y / s), and rounding to e4m3 is
monotone, so when both products give the same code the quotient gives it
too; otherwise the kernel divides.  Here numpy's fp32 arithmetic (IEEE,
round to nearest even) replays those steps over many scales, including
awkward ones, and over values planted on and next to every e4m3 rounding
midpoint; the codes come from the oracle's e4m3 rounding."""

import numpy as np

from oracle import fp8 as F

f32 = np.float32


def _bits_to_f32(u):
    return np.frombuffer(np.uint32(u).tobytes(), np.float32)[0]


def _scales(rng):
    out = [f32(1.0), _bits_to_f32(0x3F7FFFFF)]
    for _ in range(12):
        out.append(f32(rng.uniform(0.5, 2.0) * 2.0 ** int(rng.integers(-60, 60))))
    for e in (-90, -20, 0, 7, 40, 90):        # all-ones mantissas
        out.append(_bits_to_f32(((127 + e) << 23) | 0x7FFFFF))
    for e in (-45, 3, 33):                    # smallest mantissas
        out.append(_bits_to_f32(((127 + e) << 23) | 1))
    return out


def _check_block(bmax, rng):
    s = f32(bmax / f32(448.0))
    y = (rng.uniform(-1, 1, 20000).astype(f32) * bmax).astype(f32)
    codes = np.arange(0, 127, dtype=np.uint8)
    vals = F.e4m3_decode(codes).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    ym = (mids * np.float64(s)).astype(f32)
    y = np.concatenate([y, ym, -ym, np.nextafter(ym, f32(np.inf)), np.nextafter(ym, f32(0)), [f32(0), -f32(0), bmax, -bmax]])
    y = y[np.abs(y) <= bmax].astype(f32)
    q = (y / s).astype(f32)
    r = (f32(1.0) / s).astype(f32)
    r_lo = f32(r * f32(1 - 2.0 ** -20))
    r_hi = f32(r * f32(1 + 2.0 ** -20))
    lo = (y * r_lo).astype(f32)
    hi = (y * r_hi).astype(f32)
    assert np.all((np.minimum(lo, hi) <= q) & (q <= np.maximum(lo, hi)))
    c_q, c_lo, c_hi = F.e4m3_encode(q), F.e4m3_encode(lo), F.e4m3_encode(hi)
    same = c_lo == c_hi
    np.testing.assert_array_equal(c_q[same], c_lo[same])
    return same.mean()


def test_bracket_gives_the_quotients_code():
    rng = np.random.default_rng(0)
    fast = [_check_block(f32(448.0) * s, rng) for s in _scales(rng)]
    # the division is the exception, not the rule
    assert min(fast) > 0.95, fast


def test_a_wider_nudge_is_needed_than_the_rounding_error():
    """Without the nudge (r_lo = r_hi = r) the product can land on the other
    side of a rounding midpoint from the quotient: the nudge is what makes
    the bracket safe."""
    rng = np.random.default_rng(1)
    mismatches = 0
    for scale in _scales(rng):
        bmax = f32(448.0) * scale
        s = f32(bmax / f32(448.0))
        vals = F.e4m3_decode(np.arange(0, 127, dtype=np.uint8)).astype(np.float64)
        mids = (vals[:-1] + vals[1:]) / 2
        ym = (mids * np.float64(s)).astype(f32)
        y = np.concatenate([ym, np.nextafter(ym, f32(np.inf)), np.nextafter(ym, f32(0))]).astype(f32)
        y = y[np.abs(y) <= bmax]
        q = (y / s).astype(f32)
        p = (y * (f32(1.0) / s).astype(f32)).astype(f32)
        mismatches += int((F.e4m3_encode(q) != F.e4m3_encode(p)).sum())
    assert mismatches > 0

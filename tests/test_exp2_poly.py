"""CPU checks of the FMA-pipe exp2 the softmax kernels use for part of their
exponentials (Cody-Waite split, minimax polynomial, exponent shift-add).

The coefficients in csrc/fwd_sm100.cuh must be the fp32 rounding of the
Remez fit that fit_exp2_poly.py computes, and the whole evaluation, replayed
step by step in fp32 with numpy, must stay within the fit's error bound over
the arguments the softmax produces (x = s - m in log2 units: at most 8 above
zero because of the lazy max, clamped at -125 below)."""

import os
import re

import numpy as np
import pytest

from io_aware_attention_02_b200 import fit_exp2_poly as fit

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "io_aware_attention_02_b200", "csrc", "fwd_sm100.cuh")


def _kernel_coefficients():
    """(degree 3, degree 2) coefficient lists c0..cn from the kernel source."""
    src = open(SRC).read()
    body = src[src.index("__device__ __forceinline__ float2 exp2_poly2"):]
    body = body[body.index("if constexpr (kDeg == 3)"):body.index("return make_float2")]
    deg3, deg2 = body.split("} else {")
    nums = lambda s: [float(x) for x in re.findall(r"make_float2\(([0-9.eE+-]+)f, \1f\)", s)]
    # Horner order in the source: c_n, c_{n-1}, ..., c_0
    return nums(deg3)[::-1], nums(deg2)[::-1]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly_fp32(x, coef):
    magic = np.float32(12582912.0)                       # 1.5 * 2^23
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = _fma32(r, np.full_like(r, -1.0), x)
    c = [np.float32(v) for v in coef]
    p = np.full_like(f, c[-1])
    for ci in c[-2::-1]:
        p = _fma32(p, f, np.full_like(f, ci))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("degree,which", [(3, 0), (2, 1)])
def test_kernel_coefficients_are_the_fit(degree, which):
    coef, _ = fit.remez_exp2(degree)
    kernel = _kernel_coefficients()[which]
    assert len(kernel) == degree + 1
    np.testing.assert_array_equal(np.array(kernel, dtype=np.float32), coef.astype(np.float32))


@pytest.mark.parametrize("degree,which,stated", [(3, 0, 7.5e-5), (2, 1, 1.7e-3)])
def test_fp32_evaluation_within_the_bound(degree, which, stated):
    coef = _kernel_coefficients()[which]
    # the bound of the fp32 Horner evaluation on [-1/2, 1/2]; the kernel's
    # comment states it to two digits
    bound = fit.fp32_error(np.array(coef, dtype=np.float32))
    assert abs(bound - stated) <= 0.02 * stated, bound
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = _exp2_poly_fp32(x, coef).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= bound * (1 + 1e-3) + 2.0 ** -22, rel.max()
    # and the bound is not loose: the fit's error is reached
    assert rel.max() >= 0.9 * bound


def test_a_dropped_exponent_term_is_caught():
    """Mutant: without the shift-add of 2^j the result is wrong away from 0."""
    coef = _kernel_coefficients()[0]
    x = np.array([-3.2, 2.7], dtype=np.float32)
    good = _exp2_poly_fp32(x, coef)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = x - (t - magic)
    p = np.polyval(np.array(coef[::-1], dtype=np.float64), f.astype(np.float64))
    assert np.allclose(good, np.exp2(x.astype(np.float64)), rtol=1e-4)
    assert not np.allclose(p, np.exp2(x.astype(np.float64)), rtol=1e-2)

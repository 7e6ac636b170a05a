"""FP8 (e4m3) quantisation pieces of the method, written out -- TEST INFRASTRUCTURE ONLY.

Only tests, the smoke check and the bench's CPU baseline use this module; the
CUDA product path never imports it.

Citations:

* Block-wise quantisation, one scale per block instead of one per tensor --
  quantum-bit repost "H100 utilisation 75% ... FlashAttention-3"
  (m.ruangu.net), third technical upgrade (FP8: block quantisation and
  incoherent processing); dibro.site "Arquitectura y metodo" (FP8 with
  in-line per-block quantisation).
* Incoherent processing: Q and K are multiplied by a random orthogonal matrix
  such as a Hadamard matrix before quantisation; because the matrix is
  orthogonal the product Q K^T is unchanged -- "FlashAttention-3 (HE)"
  (systems-analysis.info), "Technical innovations", item 3, steps 1-4; the
  same repost, incoherent-processing paragraph.

Readings where the pages are silent (each one is listed in the design notes):

* e4m3 is the "fn" variant (no infinities, max finite 448, one NaN pattern per
  sign); rounding is round-to-nearest-even with saturation to +-448.
* A block is 128 consecutive rows of one (batch, head) by the full head dim;
  the last block of a head may be shorter (ragged N).
* scale s = amax / 448 in fp32 (amax = 0 gives s = 1); code = e4m3(fp32(y / s));
  the stored factor is the descale s, so y ~= value(code) * s.  The division
  and the e4m3 rounding are taken in fp32, the kernel's precision, because
  they decide an integer code.
* The random orthogonal matrix is R = D H_d / sqrt(d): a diagonal of +-1 signs
  (passed in as an input; all +1 when absent) followed by the Sylvester
  Hadamard matrix.  It is applied to rows: y = x R.  V is not rotated.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BLOCK_ROWS = 128


def e4m3_values() -> np.ndarray:
    """The 127 non-negative finite e4m3fn values, indexed by their 7-bit code.

    Code layout: eeee mmm with exponent bias 7.  Exponent field 0 encodes
    subnormals 2^-6 * m/8; fields 1..15 encode 2^(e-7) * (1 + m/8); the
    pattern e=15, m=7 (code 127) is NaN and is excluded.
    """
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        if e == 0:
            vals[code] = 2.0 ** -6 * (m / 8.0)
        else:
            vals[code] = 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return vals


_VALS = e4m3_values()


def e4m3_decode(codes) -> np.ndarray:
    """Decode uint8 e4m3fn codes to fp64 (NaN for the two NaN patterns)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    mag = c & 0x7F
    out = np.where(mag == 127, np.nan, _VALS[np.minimum(mag, 126)])
    return np.where(c & 0x80, -out, out)


def e4m3_encode(x) -> np.ndarray:
    """Round values to e4m3fn codes: nearest value, ties to the even code, saturating.

    ``x`` is taken exactly as given (fp32 or fp64 values); NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # index of the largest table value <= a (table is increasing)
    hi = np.searchsorted(_VALS, a, side="left")          # first value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(np.where(_VALS[hi] > a, hi - 1, hi), 0)
    d_lo = a - _VALS[lo]
    d_hi = _VALS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a >= E4M3_MAX, 126, mag)              # saturate to 448
    code = mag | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix H_d (d a power of two), entries +-1.

    H_1 = [1];  H_2n = [[H_n, H_n], [H_n, -H_n]].
    """
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation(d: int, signs=None) -> np.ndarray:
    """The orthogonal matrix R = D H_d / sqrt(d) applied to rows (y = x R)."""
    s = np.ones(d) if signs is None else np.asarray(signs, dtype=np.float64)
    return (s[:, None] * sylvester_hadamard(d)) / np.sqrt(d)


def rotate(x, signs=None) -> np.ndarray:
    """Rotate the last axis of ``x`` by R (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    return x @ rotation(x.shape[-1], signs)


def quantize_blocks(x, hadamard: bool = False, signs=None, block: int = BLOCK_ROWS):
    """Per-block e4m3 quantisation of a [B, H, N, d] tensor.

    Returns (codes uint8 [B, H, N, d], descale fp32 [B, H, ceil(N/block)],
    y fp64 [B, H, N, d]) where y is the (optionally rotated) input before
    rounding, so a test can see how close each value lies to a rounding
    boundary.
    """
    x = np.asarray(x, dtype=np.float64)
    y = rotate(x, signs) if hadamard else x
    y32 = y.astype(np.float32)
    B, H, N, d = x.shape
    nb = (N + block - 1) // block
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    desc = np.empty((B, H, nb), dtype=np.float32)
    for t in range(nb):
        r0, r1 = t * block, min(N, (t + 1) * block)
        blk = y32[:, :, r0:r1, :]
        amax = np.abs(blk).max(axis=(2, 3))                     # fp32, exact
        s = (amax / np.float32(E4M3_MAX)).astype(np.float32)    # fp32 division
        s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
        desc[:, :, t] = s
        qv = (blk / s[:, :, None, None]).astype(np.float32)     # fp32 division
        codes[:, :, r0:r1, :] = e4m3_encode(qv)
    return codes, desc, y


def dequantize_blocks(codes, descale, block: int = BLOCK_ROWS) -> np.ndarray:
    """value(code) * descale of the code's block, fp64 [B, H, N, d]."""
    vals = e4m3_decode(codes)
    N = vals.shape[2]
    rep = np.repeat(np.asarray(descale, dtype=np.float64), block, axis=2)[:, :, :N]
    return vals * rep[..., None]

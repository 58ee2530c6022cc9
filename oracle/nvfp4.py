"""NVFP4 block quantizer for the alternative page format (oracle; test infrastructure only).

Source: "KV Cache Quantization" topic page, item 3 (LMSYS Org, SGLang): the
paged KV cache stored in NVFP4, about 56 % of the bytes of FP8 per token.  The
page names the format and nothing more; its public definition is: FP4 E2M1
elements (1 sign, 2 exponent bits with bias 1, 1 mantissa bit), blocks of 16
consecutive elements sharing one FP8 E4M3 scale, and a per-tensor FP32 scale.
16 codes of 4 bits plus one byte per 16 give 0.5625 bytes per element against
1 for FP8: the page's 56 %.

Readings of this library (the page gives none of these details):

* A block is 16 consecutive dims of one (token, KV head, K or V) row of the
  rotated values, the same rows the INT4 format quantizes token-wise.
* The per-tensor FP32 scale is 1: the cache is calibration-free like the
  method's INT4 cache, so there is nothing to derive another one from.  Block
  maxima up to 6 * 448 = 2688 are represented; beyond that the codes saturate.
* Values are first clamped to the finite fp16 range, as for the INT4 format.
* Block scale: amax = max |x_i| over the block (exact), s = fp32(amax / 6)
  (IEEE division), s8 = s rounded to the nearest E4M3 value (ties to an even
  mantissa, subnormals kept) and saturated at 448.  This is the usual NVFP4
  recipe: the largest element then lands within one rounding of the top
  code 6.
* Codes: q_i = fp32(x_i / s8) (IEEE division) rounded to the nearest E2M1
  magnitude (ties to the even mantissa bit), saturated at 6; the sign bit is
  set for a negative q_i whose magnitude code is not zero, so zero is always
  stored as code 0.  A block with s8 = 0 stores all codes 0.
* Dequantized value x^_i = e2m1(c_i) * s8, exact in fp32 (at most 5
  significant bits).
"""

import numpy as np

FP16_MAX = np.float32(65504.0)
E2M1_MAX = 6.0
E4M3_MAX = 448.0
BLOCK = 16


def e2m1_value(code):
    """Value of a 4-bit E2M1 code: sign bit 3, exponent bits 2-1 (bias 1), mantissa bit 0.

    Exponent 0 is subnormal: 0.5 * m; otherwise 2^(e - 1) * (1 + m / 2)."""
    c = np.asarray(code, np.int64)
    s = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return (s * mag).astype(np.float64)


def e4m3_value(code):
    """Value of an 8-bit E4M3 (fn) code without its sign: exponent bits 6-3 (bias 7), mantissa bits 2-0.

    Exponent 0 is subnormal: m * 2^-9.  Code 0x7F is NaN (not produced here)."""
    c = np.asarray(code, np.int64) & 0x7F
    e = (c >> 3) & 15
    m = c & 7
    return np.where(e == 0, np.ldexp(m.astype(np.float64), -9), np.ldexp(1.0 + m / 8.0, e - 7))


# the 8 non-negative E2M1 magnitudes in code order, and the 127 finite non-negative E4M3 values
E2M1_GRID = e2m1_value(np.arange(8))
E4M3_GRID = e4m3_value(np.arange(127))


def _nearest_even(x, grid):
    """Index of the grid value nearest to each x >= 0 (grid ascending, index parity = mantissa parity).

    Ties go to the even index; values above the top of the grid take the top."""
    x = np.asarray(x, np.float64)
    d = np.abs(x[..., None] - grid)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    idx = np.arange(len(grid))
    # among the (at most two) nearest values, the even index
    even = cand & (idx % 2 == 0)
    return np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))


def e4m3_round(s):
    """E4M3 code of the value nearest to s >= 0 (ties to even), saturated at 448 (code 0x7E)."""
    s = np.asarray(s, np.float64)
    if np.any(s < 0) or np.any(np.isnan(s)):
        raise ValueError("block scales are non-negative")
    return _nearest_even(np.minimum(s, E4M3_MAX), E4M3_GRID).astype(np.uint8)


def e2m1_round(q):
    """E2M1 code of q: nearest magnitude (ties to even mantissa), saturated at 6, sign only when nonzero."""
    q = np.asarray(q, np.float64)
    mag = _nearest_even(np.minimum(np.abs(q), E2M1_MAX), E2M1_GRID)
    sign = (q < 0) & (mag != 0)
    return (mag | np.where(sign, 8, 0)).astype(np.uint8)


def quantize_nvfp4(x):
    """Quantize rows of fp32 values, last axis D (a multiple of 16), in blocks of 16.

    Returns (codes uint8 [..., D] holding 4-bit E2M1 codes, scales uint8 [..., D/16] E4M3 codes).
    """
    x = np.asarray(x, np.float32)
    D = x.shape[-1]
    if D % BLOCK:
        raise ValueError("the row length must be a multiple of 16")
    x = np.fmin(np.fmax(x, -FP16_MAX), FP16_MAX).astype(np.float32)
    xb = x.reshape(x.shape[:-1] + (D // BLOCK, BLOCK))
    amax = np.abs(xb).max(axis=-1)
    s = (amax / np.float32(E2M1_MAX)).astype(np.float32)            # one fp32 division
    s8 = e4m3_round(s)
    sv = e4m3_value(s8).astype(np.float32)
    safe = np.where(sv > 0, sv, np.float32(1.0))
    q = (xb / safe[..., None]).astype(np.float32)                    # one fp32 division per element
    codes = np.where((sv > 0)[..., None], e2m1_round(q), 0).astype(np.uint8)
    return codes.reshape(x.shape), s8


def dequantize_nvfp4(codes, s8):
    """x^ = e2m1(code) * e4m3(scale), exact, as fp32 [..., D]."""
    codes = np.asarray(codes)
    D = codes.shape[-1]
    v = e2m1_value(codes).reshape(codes.shape[:-1] + (D // BLOCK, BLOCK))
    out = v * e4m3_value(np.asarray(s8))[..., None]
    return out.reshape(codes.shape).astype(np.float32)

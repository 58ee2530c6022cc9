"""The exact-arithmetic facts the attention kernels build their tensor-core
operands on, checked on the host by enumeration (no GPU, no oracle).

* Magic exponent: a code c placed in the mantissa of the fp16 0x6400 (1024)
  at bit P reads as 1024 + c * 2^P while c * 2^P < 1024; one multiply by 2^-P
  and one add of -(1024 * 2^-P + centre) give c - centre exactly (INT4
  nibbles at bits 0 and 4, centre 8; INT2 crumbs at bits 0..8, centre 2;
  INT8 bytes at bit 0, centre 128).
* Paired query columns: a 16-bit integer query q with |q| <= 32639 splits
  into two signed bytes hi = floor((q + 128) / 256), lo = q - 256 hi with
  q = 256 hi + lo; a bf16 value scaled by 2^e into [2^14, 2^15) reaches at
  most 32640, the one value two signed bytes cannot hold (the kernels then
  use one bit less).
* Unsigned-byte K codes times a signed 16-bit query summed over 128 dims
  (the integer score) stays inside int32 for INT8 codes.
"""

import numpy as np


def f16_bits(v):
    return int(np.array([v], np.float16).view(np.uint16)[0])


def f16_of_bits(b):
    return float(np.array([b], np.uint16).view(np.float16)[0])


def fma16(x, a, b):
    """fp16 fused multiply-add: the exact product plus b, rounded once to fp16."""
    return float(np.float16(np.float64(x) * np.float64(a) + np.float64(b)))


def test_magic_exponent_int4_nibbles():
    for c in range(16):
        lo = f16_of_bits(0x6400 | c)                   # nibble at bits 0-3
        hi = f16_of_bits(0x6400 | (c << 4))            # nibble at bits 4-7
        assert lo == 1024 + c and hi == 1024 + 16 * c
        assert fma16(lo, 1.0, -1032.0) == c - 8        # centred: c - 8
        assert fma16(hi, 1 / 16, -72.0) == c - 8
        assert fma16(lo, 1.0, -1024.0) == c            # uncentred form


def test_magic_exponent_int2_crumbs_at_every_position():
    for p in range(9):                                 # crumb bits p, p+1 inside the 10-bit mantissa
        scale, bias = 2.0 ** -p, -(1024.0 * 2.0 ** -p + 2.0)
        assert np.float16(scale) == scale and np.float16(bias) == bias   # both constants exact in fp16
        for c in range(4):
            x = f16_of_bits(0x6400 | (c << p))
            assert x == 1024 + c * 2 ** p
            assert fma16(x, scale, bias) == c - 2
    # at bit 9 the crumb reaches into the exponent: the form stops being linear in c
    assert f16_of_bits(0x6400 | (3 << 9)) != 1024 + 3 * 512


def test_magic_exponent_int8_bytes():
    for c in range(256):
        x = f16_of_bits(0x6400 | c)
        assert x == 1024 + c
        assert fma16(x, 1.0, -1152.0) == c - 128


def test_paired_query_planes_split_exactly():
    q = np.arange(-32640, 32640, dtype=np.int64)       # every 16-bit query the paired operand holds
    hi = (q + 128) >> 8                                 # arithmetic shift: floor
    lo = q - 256 * hi
    assert hi.min() >= -128 and hi.max() <= 127
    assert lo.min() >= -128 and lo.max() <= 127
    assert np.array_equal(256 * hi + lo, q)
    # 32640 is the first value past the range
    assert ((32640 + 128) >> 8) == 128


def test_scaled_bf16_queries_reach_32640_and_no_further():
    # every positive bf16 value with exponent 0 (all 128 mantissas), scaled so that its binade is [2^14, 2^15)
    bits = np.arange(0x3F80, 0x4000, dtype=np.uint32) << 16
    vals = bits.view(np.float32).astype(np.float64)     # 1.0 .. 1.9921875
    scaled = vals * 2.0 ** 14
    assert np.all(scaled == np.rint(scaled))            # bf16 values scale to integers exactly
    assert scaled.max() == 32640 and np.count_nonzero(scaled > 32639) == 1
    # one bit less (2^13 .. 2^14) always fits
    assert (vals * 2.0 ** 13).max() <= 32639


def test_integer_scores_fit_int32():
    # INT8 codes (0..255) against a 16-bit query (|q| < 2^15) over D = 128 dims, both plane sums combined
    worst = 255 * 32768 * 128
    assert worst < 2 ** 31
    # the paired form's high-plane sum times 256 plus the low-plane sum is the same number
    hi_sum = 255 * 128 * 128                            # |hi| <= 128
    lo_sum = 255 * 128 * 128
    assert 256 * hi_sum + lo_sum < 2 ** 31

"""Pins of the oracle's quantizer: exact rational checks, bounds, brute force and a worked example."""

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import quantize_groups, dequantize_groups, fp16_round_down, fp16_round_up, bf16_round, clamp_fp16_range

HERE = os.path.dirname(os.path.abspath(__file__))


def _all_fp16_finite():
    bits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    v = bits.view(np.float16).astype(np.float64)
    return np.unique(v[np.isfinite(v)])


FP16 = _all_fp16_finite()


def _random_f32(n, seed):
    rng = np.random.default_rng(seed)
    mags = np.exp(rng.uniform(np.log(1e-9), np.log(60000.0), n))
    x = (mags * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    return np.concatenate([x, FP16[::97].astype(np.float32), np.float32([0.0, -0.0, 65504, -65504, 6e-8])])


def test_fp16_round_down_up_exact():
    x = _random_f32(20000, 0)
    x = x[np.abs(x) <= 65504]
    down = fp16_round_down(x).astype(np.float64)
    up = fp16_round_up(x).astype(np.float64)
    xd = x.astype(np.float64)
    # down is the largest fp16 <= x; up is the smallest fp16 >= x (checked against the full fp16 list)
    idx = np.searchsorted(FP16, xd, side="right") - 1
    np.testing.assert_array_equal(down, FP16[idx])
    idx_up = np.searchsorted(FP16, xd, side="left")
    np.testing.assert_array_equal(up, FP16[idx_up])


def _golden():
    vals = {}
    with open(os.path.join(HERE, "golden", "quant_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split(":")
            vals[k.strip()] = np.array([float(t) for t in v.split()], np.float64)
    return vals


def test_worked_example():
    g = _golden()
    x = g["x"].astype(np.float32)[None]
    for bits in (2, 4, 8):
        c, s, z = quantize_groups(x, bits)
        p = "int%d." % bits
        np.testing.assert_array_equal(c[0], g[p + "codes"].astype(np.uint8))
        assert float(s[0]) == g[p + "s"][0]
        assert float(z[0]) == g[p + "z"][0]
        np.testing.assert_array_equal(dequantize_groups(c, s, z)[0], g[p + "deq"].astype(np.float32))


def _groups(seed, n=400, D=128):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D)) * rng.uniform(0.01, 30, (n, 1))
    x += rng.standard_normal((n, 1)) * rng.uniform(0, 50, (n, 1))      # offset groups
    x[: n // 4, 3] *= 40                                                   # outliers
    x[n // 4: n // 2] = np.round(x[n // 4: n // 2])                      # integer-valued
    x[-3:] = 0.0                                                           # constant groups
    x[-6:-3] = 1.5
    return x.astype(np.float32)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_codes_in_range_and_error_bound(bits):
    Q = 2 ** bits - 1
    x = _groups(1)
    c, s, z = quantize_groups(x, bits)
    assert c.dtype == np.uint8 and c.max() <= Q
    xh = dequantize_groups(c, s, z).astype(np.float64)
    s64 = s.astype(np.float64)[:, None]
    err = np.abs(xh - x.astype(np.float64))
    # s/2 plus the fp32 roundings of (x - z), the division and the fma
    slack = 4 * 2.0 ** -24 * np.maximum(np.abs(x), np.abs(z.astype(np.float64))[:, None]) + 2.0 ** -24 * s64 * Q
    assert np.all(err <= s64 / 2 + slack)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_scale_zero_definition(bits):
    Q = 2 ** bits - 1
    x = _groups(2)
    c, s, z = quantize_groups(x, bits)
    mn, mx = x.min(1).astype(np.float64), x.max(1).astype(np.float64)
    zd, sd = z.astype(np.float64), s.astype(np.float64)
    # z is the largest fp16 not above mn
    idx = np.searchsorted(FP16, mn, side="right") - 1
    np.testing.assert_array_equal(zd, FP16[idx])
    # s covers the range: z + Q*s >= mx up to the fp32 rounding of r/Q
    r = mx - zd
    assert np.all(zd + Q * sd >= mx - 2.0 ** -23 * r)
    # s is the smallest fp16 >= fp32(r/Q) (or 1 for a constant group)
    sf = (r.astype(np.float32) / np.float32(Q)).astype(np.float64)
    want = FP16[np.searchsorted(FP16, sf, side="left")]
    want = np.where(r == 0, 1.0, want)
    np.testing.assert_array_equal(sd, want)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_exact_round_trip_on_representable_groups(bits):
    Q = 2 ** bits - 1
    rng = np.random.default_rng(3)
    for _ in range(200):
        s = float(np.float16(2.0 ** rng.integers(-6, 2)))   # dyadic scales keep c*s + z exact
        z = float(np.float16(rng.uniform(-30, 30)))
        codes = rng.integers(0, Q + 1, 64)
        i0, i1 = rng.choice(64, 2, replace=False)
        codes[i0], codes[i1] = 0, Q
        x = (codes * s + z).astype(np.float32)[None]
        if not np.all(x.astype(np.float64) == codes * s + z):
            continue
        c, s16, z16 = quantize_groups(x, bits)
        np.testing.assert_array_equal(c[0], codes.astype(np.uint8))
        np.testing.assert_array_equal(dequantize_groups(c, s16, z16), x)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_brute_force_nearest_code(bits):
    Q = 2 ** bits - 1
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((60, 6)) * 2).astype(np.float32)
    c, s, z = quantize_groups(x, bits)
    for g in range(x.shape[0]):
        S, Z = Fraction(float(s[g])), Fraction(float(z[g]))
        for i in range(x.shape[1]):
            X = Fraction(float(x[g, i]))
            dists = [abs(X - (k * S + Z)) for k in range(Q + 1)]
            best = min(dists)
            # the chosen code is a nearest one (ties and fp32 rounding of the
            # quotient allow a code whose distance exceeds the best by < 2^-20 s)
            assert dists[int(c[g, i])] - best <= S * Fraction(1, 2 ** 20)
            ties = [k for k, dd in enumerate(dists) if dd == best]
            if len(ties) == 2:
                assert int(c[g, i]) % 2 == 0


def test_constant_groups():
    x = np.full((3, 128), 1.5, np.float32)
    x[1] = -3.25
    x[2] = 0.0
    for bits in (4, 8):
        c, s, z = quantize_groups(x, bits)
        assert np.all(c == 0) and np.all(s == np.float16(1.0))
        np.testing.assert_array_equal(dequantize_groups(c, s, z), x)
    # not fp16-representable constant: equal codes, error below s/2
    y = np.full((1, 64), 1000.3, np.float32)
    c, s, z = quantize_groups(y, 4)
    assert len(np.unique(c)) == 1
    assert np.all(np.abs(dequantize_groups(c, s, z) - y) <= float(s[0]) / 2)


def test_clamp_and_nan():
    x = np.array([[np.nan, 1e6, -1e6, 3.0]], np.float32)
    np.testing.assert_array_equal(clamp_fp16_range(x), np.float32([[-65504, 65504, -65504, 3.0]]))
    c, s, z = quantize_groups(x, 8)
    assert np.all(np.isfinite(dequantize_groups(c, s, z)))


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 100,
                        # exact ties between two bf16 values
                        (np.arange(1, 1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
                        np.float32([0.0, -0.0, np.inf, -np.inf, 3.4e38, 1e-40])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(bf16_round(x), want)

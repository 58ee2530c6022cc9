"""Pins of the NVFP4 page format in the oracle: the E2M1 and E4M3 value sets and
roundings against independent definitions (the published value table, torch's
float8_e4m3fn, brute force over exact fractions), the hand-derived worked
example, the quantizer's error bound, the tile layout (bijection, byte
ownership, operand order) and the cache's page copy.

Source of the format: "KV Cache Quantization" topic page, item 3 (LMSYS Org /
SGLang NVFP4 paged KV storage); the rounding readings are the library's (see
oracle/nvfp4.py)."""

import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nvfp4 as F
from oracle import layout as L
from oracle.layout import TILE
from oracle.hadamard import fwht_fp32
from oracle.quant import bf16_round
from oracle import OracleKV4Cache

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = {}
    with open(os.path.join(HERE, "golden", "nvfp4_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, vals = line.split(":")
            rows[key] = [float(v) for v in vals.split()]
    return rows


@pytest.mark.parametrize("blk", list("abcdef"))
def test_worked_example(blk):
    g = _golden()
    x = np.array(g[blk + ".x"], np.float32)[None]
    codes, s8 = F.quantize_nvfp4(x)
    assert int(s8[0, 0]) == int(g[blk + ".scale"][0])
    np.testing.assert_array_equal(codes[0], np.array(g[blk + ".codes"], np.uint8))
    np.testing.assert_array_equal(F.dequantize_nvfp4(codes, s8)[0], np.array(g[blk + ".deq"], np.float32))


def test_e2m1_value_set():
    """The 16 codes give the published E2M1 value set, +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}, sign in bit 3."""
    table = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    np.testing.assert_array_equal(F.e2m1_value(np.arange(8)), table)
    np.testing.assert_array_equal(F.e2m1_value(np.arange(8, 16)), [-v for v in table])


def test_e4m3_values_match_torch():
    codes = torch.arange(127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(F.e4m3_value(np.arange(127)), ref)
    assert F.e4m3_value(126) == 448.0


def test_e4m3_rounding_matches_torch():
    """Nearest E4M3 with ties to even (torch's fp32 -> float8_e4m3fn) on random values, the exact
    midpoints between neighbours, and fp32 neighbours of every grid value."""
    rng = np.random.default_rng(3)
    grid = F.E4M3_GRID
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    near = np.concatenate([np.nextafter(grid.astype(np.float32), np.float32(0)),
                           np.nextafter(grid.astype(np.float32), np.float32(1000))])
    rand = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(-12, 6, 20000))]).astype(np.float32)
    s = np.concatenate([mids, near, rand, grid.astype(np.float32)])
    s = s[(s >= 0) & (s <= 448)]
    ref = torch.from_numpy(s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(F.e4m3_round(s), ref)
    # saturation (the library's reading: satfinite)
    np.testing.assert_array_equal(F.e4m3_round(np.array([449, 464, 1e6], np.float32)), [126, 126, 126])


def _e2m1_brute(q):
    """Nearest E2M1 magnitude by exact fractions; ties to the even code; sign only when nonzero."""
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
            Fraction(6)]
    a = abs(Fraction(float(q)))
    d = [abs(a - m) for m in mags]
    best = min(d)
    cand = [i for i in range(8) if d[i] == best]
    i = cand[0] if len(cand) == 1 else [c for c in cand if c % 2 == 0][0]
    return i | (8 if (q < 0 and i != 0) else 0)


def test_e2m1_rounding_brute_force_and_thresholds():
    rng = np.random.default_rng(4)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(10))])
    q = np.concatenate([ties, near, -ties, -near, rng.uniform(-8, 8, 3000).astype(np.float32),
                        np.array([0, -0.0, 6, -6, 7, -100, 1e-30, -1e-30], np.float32)])
    got = F.e2m1_round(q)
    np.testing.assert_array_equal(got, [_e2m1_brute(v) for v in q])
    # the same rule as seven comparisons on |q| (ties at 0.25, 1.25, 2.5, 5 stay down, at 0.75, 1.75, 3.5 go up)
    a = np.abs(q.astype(np.float64))
    mag = ((a > 0.25).astype(int) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5) + (a >= 3.5) + (a > 5))
    np.testing.assert_array_equal(got & 7, mag)


def test_quantizer_error_bound():
    """|x - x^| <= s8 for every element (a half grid step at most, or the saturation of the block
    maximum, which the E4M3 rounding bounds by 6 / (1 - 2^-4) in units of s8), and s8 within one
    E4M3 rounding of amax / 6."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((400, 128)) * np.exp(rng.uniform(-6, 6, (400, 1)))).astype(np.float32)
    x[:5, 3] = 2000.0
    codes, s8 = F.quantize_nvfp4(x)
    xh = F.dequantize_nvfp4(codes, s8)
    amax = np.abs(x.reshape(400, 8, 16)).max(-1)
    ok = (amax / 6 >= 2.0 ** -6)            # normal E4M3 range: relative rounding error <= 2^-4
    sv = F.e4m3_value(s8)
    err = np.abs(x.astype(np.float64) - xh).reshape(400, 8, 16).max(-1)
    assert ok.sum() > 1000 and (~ok).sum() > 100
    assert np.all(err[ok] <= sv[ok])
    rel = np.abs(sv - amax / 6) / (amax / 6)
    assert np.all(rel[ok] <= 2.0 ** -4 + 1e-12)
    # below the normal range the scale is the nearest subnormal (m * 2^-9) or 0, and 0 only when
    # amax / 6 is at most half the smallest subnormal
    assert np.all((sv == 0) == (amax / 6 <= 2.0 ** -10))
    assert np.all(np.abs(sv - amax / 6)[~ok] <= 2.0 ** -10 + 1e-12)


@pytest.mark.parametrize("D", [64, 128])
def test_fp4_layout_bijection_and_ownership(D):
    seen_k, seen_v = {}, {}
    for r in range(TILE):
        for d in range(D):
            k = L.fp4_k_nibble(D, r, d)
            v = L.fp4_v_nibble(D, r, d)
            assert 0 <= k[0] < 8 * D and 0 <= v[0] < 8 * D
            assert k not in seen_k and v not in seen_v
            seen_k[k] = r
            seen_v[v] = (r, d)
    assert len(seen_k) == len(seen_v) == 16 * D
    for byte in range(8 * D):
        assert seen_k[(byte, 0)] == seen_k[(byte, 1)]                   # a K byte belongs to one token
        (r0, d0), (r1, d1) = seen_v[(byte, 0)], seen_v[(byte, 1)]
        assert d0 == d1 and r0 % 2 == 0 and r1 == r0 + 1                 # a V byte: one dim of tokens 2i, 2i+1
    sc = {L.fp4_k_scale_byte(D, r, b) for r in range(TILE) for b in range(D // 16)} | \
         {L.fp4_v_scale_byte(D, r, b) for r in range(TILE) for b in range(D // 16)}
    assert sc == set(range(16 * D, 18 * D)) and L.fp4_tile_bytes(D) == 18 * D


@pytest.mark.parametrize("D", [64, 128])
def test_fp4_operand_order(D):
    """Lane 4g + t finds its 16x8x16 fp16 A-operand pairs in one word per 16-dim block: bytes 0/1 =
    tokens g / g + 8 at dims (4t, 4t+1) of the block, bytes 2/3 = the same tokens at dims
    (4t+2, 4t+3), the lower dim in the low nibble; the B operand of the query uses the same dim
    order.  For P.V (A = V^T, rows = dims) bytes 0/1 = dims g / g + 8 at tokens (2t, 2t+1), bytes
    2/3 = the same dims at tokens (2t+8, 2t+9), the even token in the low nibble."""
    for lane in range(32):
        g, t = divmod(lane, 4)
        for b in range(D // 16):
            w = 16 * lane + 4 * (b % 4) + 512 * (b // 4)
            for byte, (tok, d0) in enumerate([(g, 4 * t), (g + 8, 4 * t), (g, 4 * t + 2), (g + 8, 4 * t + 2)]):
                assert L.fp4_k_nibble(D, tok, 16 * b + d0) == (w + byte, 0)
                assert L.fp4_k_nibble(D, tok, 16 * b + d0 + 1) == (w + byte, 1)
            for byte, (dim, t0) in enumerate([(g, 2 * t), (g + 8, 2 * t), (g, 2 * t + 8), (g + 8, 2 * t + 8)]):
                assert L.fp4_v_nibble(D, t0, 16 * b + dim) == (w + byte, 0)
                assert L.fp4_v_nibble(D, t0 + 1, 16 * b + dim) == (w + byte, 1)


def _cfg(fmt, D=128):
    return dict(num_layers=1, max_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=D, page_size=32,
                num_pages=12, max_pages_per_seq=4, hadamard_block=D, sink_tokens=4, recent_window=16,
                page_format=fmt)


@pytest.mark.parametrize("D", [64, 128])
def test_cache_pages_hold_the_block_quantized_rotation(D):
    """Appends in ragged pieces (so the two tokens sharing a V byte arrive in different calls):
    the page view is the NVFP4 round trip of the rotated inputs, the protected view is the INT8
    path of the INT4 cache, and the sequence lengths advance alike."""
    rng = np.random.default_rng(6)
    bt = rng.permutation(12).reshape(3, 4)
    a, b = OracleKV4Cache(_cfg(1, D), bt), OracleKV4Cache(_cfg(0, D), bt)
    lens = [0, 0, 0]
    for step in range(6):
        n = rng.integers(0, 9, 3)
        tot = int(n.sum())
        k = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32) * 2)
        v = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32))
        cu = np.concatenate([[0], np.cumsum(n)])
        for c in (a, b):
            c.append(0, [0, 1, 2], cu, k, v)
        for s in range(3):
            lens[s] += int(n[s])
    ks, vs = {}, {}
    np.testing.assert_array_equal(a.seq_lens, b.seq_lens)
    # the inputs again, in order, to compare the page copies
    rng = np.random.default_rng(6)
    rng.permutation(12)
    for s in range(3):
        ks[s], vs[s] = [], []
    for step in range(6):
        n = rng.integers(0, 9, 3)
        tot = int(n.sum())
        k = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32) * 2)
        v = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32))
        off = 0
        for s in range(3):
            ks[s].append(k[off:off + n[s]])
            vs[s].append(v[off:off + n[s]])
            off += int(n[s])
    for s in range(3):
        if lens[s] == 0:
            continue
        kr = fwht_fp32(np.concatenate(ks[s]), D)
        vr = fwht_fp32(np.concatenate(vs[s]), D)
        kp, vp = a.view(0, s, protected=False)
        np.testing.assert_array_equal(kp, F.dequantize_nvfp4(*F.quantize_nvfp4(kr)))
        np.testing.assert_array_equal(vp, F.dequantize_nvfp4(*F.quantize_nvfp4(vr)))
        ke, ve = a.view(0, s)
        kb, vb = b.view(0, s)
        L_ = lens[s]
        prot = np.array([p < 4 or p >= L_ - 16 for p in range(L_)])
        np.testing.assert_array_equal(ke[prot], kb[prot])
        np.testing.assert_array_equal(ve[prot], vb[prot])
        np.testing.assert_array_equal(ke[~prot], kp[~prot])


def test_tie_rule_mistake_fails_the_worked_example(monkeypatch):
    """A plausible slip -- ties rounded away from zero instead of to the even code -- breaks block a."""
    def away(x, grid):
        x = np.asarray(x, np.float64)
        d = np.abs(x[..., None] - grid)
        best = d.min(axis=-1, keepdims=True)
        return (len(grid) - 1 - np.argmax((d == best)[..., ::-1], axis=-1))
    monkeypatch.setattr(F, "_nearest_even", away)
    g = _golden()
    codes, _ = F.quantize_nvfp4(np.array(g["a.x"], np.float32)[None])
    assert not np.array_equal(codes[0], np.array(g["a.codes"], np.uint8))


def _e4m3_truncate(s):
    """E4M3 code of the largest value not above s (a mistake: truncation instead of the nearest value)."""
    s = np.minimum(np.asarray(s, np.float64), F.E4M3_MAX)
    return (np.searchsorted(F.E4M3_GRID, s, side="right") - 1).astype(np.uint8)


@pytest.mark.parametrize("mistake", ["scale from amax / 4", "scale truncated to E4M3"])
def test_block_scale_mistakes_fail_the_worked_example(monkeypatch, mistake):
    """Two plausible slips in the block scale -- dividing amax by 4 (the largest normal E2M1 power of two)
    instead of by 6, or truncating it to E4M3 instead of rounding to the nearest value -- each break at
    least one hand-derived block."""
    if mistake == "scale from amax / 4":
        monkeypatch.setattr(F, "E2M1_MAX", 4.0)
    else:
        monkeypatch.setattr(F, "e4m3_round", _e4m3_truncate)
    failed = 0
    for blk in "abcdef":
        try:
            test_worked_example(blk)
        except AssertionError:
            failed += 1
    assert failed >= 1

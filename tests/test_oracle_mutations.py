"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one.

Each case swaps one oracle function for a mutated copy inside the test only
(monkeypatch) and re-runs the property that pins that function.
"""

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle import hadamard, quant, cache as cache_mod, attention as attn_mod
from oracle.hadamard import rotation_constant_fp32


def _fwht_swapped_signs(x, Bh):
    x = np.asarray(x, np.float32)
    lead, D = x.shape[:-1], x.shape[-1]
    y = x.reshape(lead + (D // Bh, Bh)).copy()
    h = 1
    while h < Bh:
        y = y.reshape(lead + (D // Bh, Bh // (2 * h), 2, h))
        a, b = y[..., 0, :], y[..., 1, :]
        y = np.stack([a - b, a + b], axis=-2)      # mistake: outputs swapped
        h *= 2
    return (y.reshape(lead + (D,)) * rotation_constant_fp32(Bh)).astype(np.float32)


def _fwht_unscaled(x, Bh):
    return (hadamard.fwht_fp32(x, Bh) / rotation_constant_fp32(Bh)).astype(np.float32)  # mistake: no 1/sqrt(Bh)


@pytest.mark.parametrize("bad", [_fwht_swapped_signs, _fwht_unscaled])
def test_fwht_mistakes_fail_the_column_pin(bad):
    Bh = 64
    out = bad(np.eye(Bh, dtype=np.float32), Bh)
    expect = (scipy.linalg.hadamard(Bh) / np.sqrt(Bh)).T.astype(np.float32)
    assert not np.array_equal(out, expect)


def _quantize_rne_zero(x, bits):
    Q = np.float32(2 ** bits - 1)
    x = quant.clamp_fp16_range(x)
    mn, mx = x.min(-1), x.max(-1)
    z16 = mn.astype(np.float16)                      # mistake: nearest instead of downward
    z = z16.astype(np.float32)
    r = (mx - z).astype(np.float32)
    s16 = quant.fp16_round_up((r / Q).astype(np.float32))
    s16 = np.where(r == 0, np.float16(1), s16).astype(np.float16)
    s = s16.astype(np.float32)
    c = np.clip(np.rint(((x - z[..., None]) / s[..., None]).astype(np.float32)), 0, Q).astype(np.uint8)
    return c, s16, z16


def test_zero_point_rounding_mistake_fails_the_definition_pin():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((300, 64)) * 3 + 40).astype(np.float32)
    c, s, z = _quantize_rne_zero(x, 4)
    assert np.any(z.astype(np.float64) > x.min(1))    # the pin requires z <= min


def test_dropped_zero_point_fails_the_round_trip_pin():
    x = (np.arange(16, dtype=np.float32) * 0.5 - 3.0)[None]
    c, s, z = quant.quantize_groups(x, 4)
    wrong = (c.astype(np.float64) * s.astype(np.float64)[..., None]).astype(np.float32)   # mistake: no + z
    assert not np.array_equal(wrong, x)
    np.testing.assert_array_equal(quant.dequantize_groups(c, s, z), x)


def test_wrong_gqa_mapping_fails_the_sdpa_pin(monkeypatch):
    def bad_attention(q, k, v, scale):
        q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
        Hq, D = q.shape
        Hkv = k.shape[1]
        o = np.zeros((Hq, D))
        for j in range(Hq):
            h = j % Hkv                                  # mistake: interleaved grouping
            s = scale * (k[:, h] @ q[j])
            a = np.exp(s - s.max())
            o[j] = (a / a.sum()) @ v[:, h]
        return o
    rng = np.random.default_rng(1)
    q = rng.standard_normal((8, 16))
    k = rng.standard_normal((9, 2, 16))
    v = rng.standard_normal((9, 2, 16))
    good = attn_mod.attention_fp64(q, k, v, 0.25)
    assert not np.allclose(bad_attention(q, k, v, 0.25), good)


def test_wrong_ring_slot_fails_the_direct_construction_pin(monkeypatch):
    cfg = dict(num_layers=1, max_seqs=1, num_q_heads=4, num_kv_heads=1, head_dim=64, page_size=16,
               num_pages=16, max_pages_per_seq=16, hadamard_block=64, sink_tokens=4, recent_window=32)
    table = np.arange(16, dtype=np.int32)[None]
    rng = np.random.default_rng(2)
    k = oracle.bf16_round(rng.standard_normal((80, 1, 64)).astype(np.float32))
    v = k.copy()
    good = cache_mod.OracleKV4Cache(cfg, table)
    for i in range(80):
        good.append(0, [0], [0, 1], k[i:i + 1], v[i:i + 1])
    monkeypatch.setattr(cache_mod, "prot_slot", lambda p, S, W: p if p < S else S + (p - S + 1) % W)
    bad = cache_mod.OracleKV4Cache(cfg, table)
    for i in range(80):
        bad.append(0, [0], [0, 1], k[i:i + 1], v[i:i + 1])
    monkeypatch.undo()
    # reading the mutated store through the correct slot rule gives wrong values
    assert not np.array_equal(bad.view(0, 0)[0], good.view(0, 0)[0])


def _extend_with_visibility(shift):
    """The oracle's multi-token attention with the visible range moved by `shift` positions (a mistake)."""
    def run(cache, layer, seq_ids, q, scale=None, protected=True):
        q = np.asarray(q, np.float32)
        scale = scale if scale else 1.0 / np.sqrt(cache.D)
        H = oracle.block_diag_hadamard(cache.D, cache.Bh)
        T = q.shape[1]
        out = np.zeros(q.shape, np.float64)
        q_rot = attn_mod.rotate_query(q, cache.Bh)
        for b, seq in enumerate(seq_ids):
            kh, vh = cache.view(layer, int(seq), protected=protected)
            L = kh.shape[0]
            for i in range(T):
                vis = min(L, L - T + i + 1 + shift)
                if vis > 0:
                    out[b, i] = attn_mod.attention_fp64(q_rot[b, i], kh[:vis], vh[:vis], scale) @ H.T
        return out
    return run


@pytest.mark.parametrize("shift", [-1, 1])
def test_causal_off_by_one_fails_the_masked_sdpa_pin(shift):
    from test_oracle_attention import _sdpa_causal
    cfg = dict(num_layers=1, max_seqs=1, num_q_heads=4, num_kv_heads=2, head_dim=64, page_size=16,
               num_pages=8, max_pages_per_seq=8, hadamard_block=1, sink_tokens=4, recent_window=16)
    rng = np.random.default_rng(3)
    L, T = 50, 3
    codes = rng.integers(0, 16, (L, 2, 64))
    codes[:, :, 0], codes[:, :, 1] = 0, 15
    k = (codes * (17 / 64) - 2.0).astype(np.float32)
    v = (np.roll(codes, 5, axis=2) * (17 / 128) + 1.0).astype(np.float32)
    q = oracle.bf16_round(rng.standard_normal((1, T, 4, 64)).astype(np.float32))
    c = cache_mod.OracleKV4Cache(cfg, np.arange(8, dtype=np.int32)[None])
    c.append(0, [0], [0, L], k, v)
    want = _sdpa_causal(q[0], k, v, 0.125)
    np.testing.assert_allclose(_extend_with_visibility(0)(c, 0, [0], q)[0], want, atol=1e-12)
    assert not np.allclose(_extend_with_visibility(shift)(c, 0, [0], q)[0], want, atol=1e-6)


def test_output_rotated_twice_fails_the_inverse_pin():
    # a mistake that applies H to the output in the rotated mode as well
    cfg = dict(num_layers=1, max_seqs=1, num_q_heads=4, num_kv_heads=1, head_dim=64, page_size=16,
               num_pages=8, max_pages_per_seq=8, hadamard_block=64, sink_tokens=4, recent_window=16)
    rng = np.random.default_rng(4)
    k = oracle.bf16_round(rng.standard_normal((30, 1, 64)).astype(np.float32))
    c = cache_mod.OracleKV4Cache(cfg, np.arange(8, dtype=np.int32)[None])
    c.append(0, [0], [0, 30], k, k)
    q = oracle.bf16_round(rng.standard_normal((1, 4, 64)).astype(np.float32))
    H = oracle.block_diag_hadamard(64, 64)
    base = attn_mod.decode_attention(c, 0, [0], q)["out_f64"]
    wrong = base                                      # mistake: rotated mode returns the unrotated output
    assert not np.allclose(wrong, base @ H, atol=1e-6)
    np.testing.assert_allclose(attn_mod.decode_attention(c, 0, [0], q, out_rotated=True)["out_f64"], base @ H,
                               atol=1e-12)


def test_scale_rounded_down_fails_the_definition_pin(monkeypatch):
    import test_oracle_quant as tq
    monkeypatch.setattr(quant, "fp16_round_up", quant.fp16_round_down)   # mistake: s may no longer cover the range
    for bits in (2, 4, 8):
        with pytest.raises(AssertionError):
            tq.test_scale_zero_definition(bits)


def _quantize_extra_level(x, bits):
    """The quantizer with 2^bits levels above zero instead of 2^bits - 1 (a mistake)."""
    Q = np.float32(2 ** bits)
    x = quant.clamp_fp16_range(x)
    z16 = quant.fp16_round_down(x.min(-1))
    z = z16.astype(np.float32)
    r = (x.max(-1) - z).astype(np.float32)
    s16 = np.where(r == 0, np.float16(1), quant.fp16_round_up((r / Q).astype(np.float32))).astype(np.float16)
    s = s16.astype(np.float32)
    c = np.clip(np.rint(((x - z[..., None]).astype(np.float32) / s[..., None]).astype(np.float32)), 0, Q)
    return c.astype(np.uint8), s16, z16


def test_extra_quantization_level_fails_the_range_pins(monkeypatch):
    import test_oracle_quant as tq
    monkeypatch.setattr(tq, "quantize_groups", _quantize_extra_level)
    for bits in (2, 4, 8):
        with pytest.raises(AssertionError):
            tq.test_codes_in_range_and_error_bound(bits)


PROTECTION_MISTAKES = {
    "window one short": lambda p, L, S, W: p < S or p > L - W,
    "one sink too many": lambda p, L, S, W: p <= S or p >= L - W,
    "window one long": lambda p, L, S, W: p < S or p >= L - W - 1,
}


@pytest.mark.parametrize("name", sorted(PROTECTION_MISTAKES))
def test_protection_boundary_mistakes_fail_the_view_pins(monkeypatch, name):
    import test_oracle_cache as tc
    bad = PROTECTION_MISTAKES[name]
    S, W = 4, 32
    # the rule itself: its protected slots must be the prefix [0, min(L, S + W)) of the store
    assert any(sorted(cache_mod.prot_slot(p, S, W) for p in range(L) if bad(p, L, S, W)) != list(range(min(L, S + W)))
               for L in range(1, 200))
    # the cache's effective view read through it differs from the per-position construction
    monkeypatch.setattr(cache_mod, "is_protected", bad)
    with pytest.raises(AssertionError):
        tc.test_effective_view_equals_direct_construction([1] * 120)


def test_rope_turned_backwards_fails_the_complex_pin():
    import workloads
    R = 64
    cs = workloads.rope_cos_sin(5000, R, base=1e4)
    x = oracle.bf16_round(np.random.default_rng(9).standard_normal((6, 128)).astype(np.float32))
    pos = np.array([1, 17, 255, 1024, 3333, 4999])
    c, s = cs[pos, :R // 2], cs[pos, R // 2:]
    a, b = x[:, 0:R:2], x[:, 1:R:2]
    wrong = np.empty_like(x[:, :R])
    wrong[:, 0::2], wrong[:, 1::2] = a * c + b * s, b * c - a * s      # mistake: turned by -theta
    z = (a.astype(np.float64) + 1j * b) * (c.astype(np.float64) + 1j * s)
    assert not np.allclose(wrong[:, 0::2], z.real, rtol=0, atol=4e-6 * np.abs(x).max())
    right = oracle.rope_fp32(x, pos, cs, R, oracle.ROPE_GPTJ)
    np.testing.assert_allclose(right[:, 0:R:2], z.real, rtol=0, atol=4e-6 * np.abs(x).max())

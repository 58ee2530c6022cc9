"""Pins of the oracle's RoPE (rotary embedding in front of the block Hadamard):
complex-multiplication form, the neox/gptj pair layouts as permutations of each
other, identity at angle 0, partial rotary, the relative-position property, and
the position bookkeeping of the cache append and of the query."""

import numpy as np
import pytest

import workloads
from oracle import (rope_fp32, ROPE_NEOX, ROPE_GPTJ, OracleKV4Cache, decode_attention, extend_attention,
                    bf16_round)


def _x(shape, seed):
    return bf16_round(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("R", [32, 64, 128])
def test_gptj_is_complex_multiplication(R):
    cs = workloads.rope_cos_sin(5000, R, base=1e4)
    x = _x((7, 128), R)
    pos = np.array([0, 1, 17, 255, 1024, 3333, 4999])
    y = rope_fp32(x, pos, cs, R, ROPE_GPTJ)
    z = (x[:, 0:R:2].astype(np.float64) + 1j * x[:, 1:R:2]) * (cs[pos, :R // 2].astype(np.float64)
                                                                + 1j * cs[pos, R // 2:])
    np.testing.assert_allclose(y[:, 0:R:2], z.real, rtol=0, atol=4e-6 * np.abs(x).max())
    np.testing.assert_allclose(y[:, 1:R:2], z.imag, rtol=0, atol=4e-6 * np.abs(x).max())
    np.testing.assert_array_equal(y[:, R:], x[:, R:])                      # partial rotary: untouched


@pytest.mark.parametrize("R", [32, 128])
def test_neox_is_gptj_on_permuted_dims(R):
    cs = workloads.rope_cos_sin(100, R)
    x = _x((5, 128), 3)
    pos = np.array([0, 3, 50, 77, 99])
    perm = np.arange(128)
    perm[:R] = np.stack([np.arange(R // 2), R // 2 + np.arange(R // 2)], axis=1).reshape(-1)   # (i, i + R/2) -> (2i, 2i+1)
    inv = np.argsort(perm)
    np.testing.assert_array_equal(rope_fp32(x, pos, cs, R, ROPE_NEOX),
                                  rope_fp32(x[:, perm], pos, cs, R, ROPE_GPTJ)[:, inv])


def test_angle_zero_is_identity_and_norms_are_kept():
    cs = workloads.rope_cos_sin(64, 128)
    x = _x((3, 128), 4)
    for style in (ROPE_NEOX, ROPE_GPTJ):
        np.testing.assert_array_equal(rope_fp32(x, 0, cs, 128, style), x)
        y = rope_fp32(x, np.array([5, 40, 63]), cs, 128, style)
        np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)


@pytest.mark.parametrize("style", [ROPE_NEOX, ROPE_GPTJ])
def test_scores_depend_on_the_relative_position(style):
    cs = workloads.rope_cos_sin(4000, 128, base=1e4)
    q, k = _x((128,), 5), _x((128,), 6)
    ref = float(rope_fp32(q, 700, cs, 128, style) @ rope_fp32(k, 650, cs, 128, style))
    for shift in (-650, 1, 1000, 2300):
        got = float(rope_fp32(q, 700 + shift, cs, 128, style) @ rope_fp32(k, 650 + shift, cs, 128, style))
        assert abs(got - ref) <= 2e-4 * np.linalg.norm(q) * np.linalg.norm(k)
    other = float(rope_fp32(q, 700, cs, 128, style) @ rope_fp32(k, 600, cs, 128, style))
    assert abs(other - ref) > 1e-2


def _cfg():
    return dict(num_layers=1, max_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=64, page_size=16, num_pages=20,
                max_pages_per_seq=10, hadamard_block=64, sink_tokens=4, recent_window=16)


@pytest.mark.parametrize("style,R", [(ROPE_NEOX, 64), (ROPE_GPTJ, 32)])
def test_cache_append_takes_each_key_at_its_position(style, R):
    # chunked appends with RoPE == one append of keys turned by hand at positions 0 .. L-1
    cs = workloads.rope_cos_sin(200, R)
    k, v = _x((90, 2, 64), 7), _x((90, 2, 64), 8)
    table = np.arange(20, dtype=np.int32).reshape(2, 10)
    a = OracleKV4Cache(_cfg(), table)
    for lo, hi in ((0, 33), (33, 34), (34, 90)):
        a.append(0, [1], [0, hi - lo], k[lo:hi], v[lo:hi], rope=(cs, R, style))
    b = OracleKV4Cache(_cfg(), table)
    b.append(0, [1], [0, 90], rope_fp32(k, np.arange(90)[:, None], cs, R, style), v)
    for key in a.pages:
        np.testing.assert_array_equal(a.pages[key], b.pages[key])
    for key in a.prot:
        np.testing.assert_array_equal(a.prot[key], b.prot[key])


@pytest.mark.parametrize("style", [ROPE_NEOX, ROPE_GPTJ])
def test_query_rope_sits_at_the_query_position(style):
    cs = workloads.rope_cos_sin(200, 64)
    rope = (cs, 64, style)
    k, v = _x((60, 2, 64), 9), _x((60, 2, 64), 10)
    c = OracleKV4Cache(_cfg(), np.arange(20, dtype=np.int32).reshape(2, 10))
    c.append(0, [0, 1], [0, 45, 60], k, v, rope=rope)          # lengths 45 and 15
    q = _x((2, 8, 64), 11)
    turned = rope_fp32(q, np.array([44, 14])[:, None], *rope)  # decode: position L - 1
    np.testing.assert_array_equal(decode_attention(c, 0, [0, 1], q, rope=rope)["out_f64"],
                                  decode_attention(c, 0, [0, 1], turned)["out_f64"])
    qx = _x((2, 3, 8, 64), 12)
    turned = rope_fp32(qx, np.array([[42, 43, 44], [12, 13, 14]])[:, :, None], *rope)   # L - 3 + i
    np.testing.assert_array_equal(extend_attention(c, 0, [0, 1], qx, rope=rope)["out_f64"],
                                  extend_attention(c, 0, [0, 1], turned)["out_f64"])

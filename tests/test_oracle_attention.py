"""Pins of the oracle's attention: library SDPA, rotation invariance, special cases, brute force."""

import numpy as np
import pytest
import torch

from oracle import (attention_fp64, decode_attention, decode_attention_bf16, extend_attention, OracleKV4Cache,
                    OracleBF16Cache, block_diag_hadamard, bf16_round)


def _sdpa(q, k, v, scale):
    Hq, D = q.shape
    L, Hkv, _ = k.shape
    G = Hq // Hkv
    qt = torch.from_numpy(np.asarray(q, np.float64))[:, None, :]                 # [Hq, 1, D]
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0, :].numpy()


@pytest.mark.parametrize("Hq,Hkv,L", [(4, 1, 37), (32, 8, 300), (8, 8, 5), (16, 2, 1)])
def test_matches_torch_sdpa(Hq, Hkv, L):
    rng = np.random.default_rng(0)
    q = rng.standard_normal((Hq, 64))
    k = rng.standard_normal((L, Hkv, 64)) * 2
    v = rng.standard_normal((L, Hkv, 64))
    np.testing.assert_allclose(attention_fp64(q, k, v, 0.125), _sdpa(q, k, v, 0.125), rtol=1e-12, atol=1e-13)


def test_brute_force_loops():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((4, 8))
    k = rng.standard_normal((6, 2, 8))
    v = rng.standard_normal((6, 2, 8))
    out = attention_fp64(q, k, v, 0.3)
    for j in range(4):
        h = j // 2
        s = [0.3 * sum(q[j, d] * k[p, h, d] for d in range(8)) for p in range(6)]
        m = max(s)
        e = [np.exp(x - m) for x in s]
        o = [sum(e[p] * v[p, h, d] for p in range(6)) / sum(e) for d in range(8)]
        np.testing.assert_allclose(out[j], o, rtol=1e-13)


def test_rotation_invariance():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((8, 128))
    k = rng.standard_normal((50, 2, 128))
    v = rng.standard_normal((50, 2, 128))
    for Bh in (128, 64, 16):
        H = block_diag_hadamard(128, Bh)
        rot = attention_fp64(q @ H.T, k @ H.T, v @ H.T, 0.1) @ H    # H^{-1} = H^T
        np.testing.assert_allclose(rot, attention_fp64(q, k, v, 0.1), atol=1e-12)


def test_gqa_grouping_is_contiguous():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((8, 16))
    k = rng.standard_normal((9, 2, 16))
    v = rng.standard_normal((9, 2, 16))
    a = attention_fp64(q, k, v, 0.25)
    v2 = v.copy()
    v2[:, 0] += 1.0
    b = attention_fp64(q, k, v2, 0.25)
    assert np.all(np.abs(a[:4] - b[:4]) > 0.5) and np.array_equal(a[4:], b[4:])


def _cfg(D=64, Bh=64, S=4, W=32, Hkv=1, Hq=4):
    return dict(num_layers=1, max_seqs=2, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, page_size=16,
                num_pages=40, max_pages_per_seq=20, hadamard_block=Bh, sink_tokens=S, recent_window=W)


def _table():
    t = np.arange(40, dtype=np.int32).reshape(2, 20)[:, ::-1].copy()
    return t


def test_quantization_free_reduction_to_textbook():
    # Bh = 1 and values z + c4*17*2^-k with codes c4 = 0..15 present: the INT4
    # scale is 17*2^-k and the INT8 scale 2^-k (codes 17*c4), so both encodings
    # are exact and decode attention is textbook attention on the inputs.
    cfg = _cfg(Bh=1)
    rng = np.random.default_rng(4)
    L = 70
    codes = rng.integers(0, 16, (L, 1, 64))
    codes[:, :, 0], codes[:, :, 1] = 0, 15
    k = (codes * (17 / 64) - 2.0).astype(np.float32)
    v = (np.roll(codes, 3, axis=2) * (17 / 128) + 1.0).astype(np.float32)
    q = bf16_round(rng.standard_normal((1, 4, 64)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [1], [0, L], k, v)
    res = decode_attention(cache, 0, [1], q)
    np.testing.assert_allclose(res["out_f64"][0], _sdpa(q[0], k, v, 0.125), atol=1e-12)
    np.testing.assert_allclose(decode_attention(cache, 0, [1], q, protected=False)["out_f64"][0],
                               _sdpa(q[0], k, v, 0.125), atol=1e-12)


def test_single_token_context_returns_its_value():
    cfg = _cfg()
    rng = np.random.default_rng(5)
    k = bf16_round(rng.standard_normal((1, 1, 64)).astype(np.float32))
    v = bf16_round(rng.standard_normal((1, 1, 64)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0], [0, 1], k, v)
    q = bf16_round(rng.standard_normal((1, 4, 64)).astype(np.float32))
    out = decode_attention(cache, 0, [0], q)["out_f64"][0]
    vh = cache.view(0, 0)[1][0, 0].astype(np.float64) @ block_diag_hadamard(64, 64).T
    for j in range(4):
        np.testing.assert_allclose(out[j], vh, atol=1e-12)
    # the INT8 sink is within its s/2 of the input
    assert np.max(np.abs(vh - v[0, 0])) < 0.02


def test_uniform_keys_give_the_mean_value():
    # identical keys stay identical only inside one encoding: check the INT4-only
    # view, and a window covering the whole context (every position INT8)
    rng = np.random.default_rng(6)
    L = 48
    k = np.repeat(bf16_round(rng.standard_normal((1, 1, 64)).astype(np.float32)), L, axis=0)
    v = bf16_round(rng.standard_normal((L, 1, 64)).astype(np.float32))
    q = bf16_round(rng.standard_normal((1, 4, 64)).astype(np.float32))
    for W, protected in ((16, False), (64, True)):
        cache = OracleKV4Cache(_cfg(S=0, W=W), _table())
        cache.append(0, [0], [0, L], k, v)
        out = decode_attention(cache, 0, [0], q, protected=protected)["out_f64"][0]
        vh = cache.view(0, 0, protected=protected)[1][:, 0].astype(np.float64) @ block_diag_hadamard(64, 64).T
        for j in range(4):
            np.testing.assert_allclose(out[j], vh.mean(0), atol=1e-12)


def test_quantized_attention_close_to_exact():
    # INT4 with rotation stays near the unquantized answer (sanity of the whole chain).
    cfg = _cfg(D=128, Bh=128, W=32)
    rng = np.random.default_rng(7)
    L = 300
    k = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    v = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0], [0, L], k, v)
    q = bf16_round(rng.standard_normal((1, 4, 128)).astype(np.float32))
    out = decode_attention(cache, 0, [0], q)["out_f64"][0]
    exact = attention_fp64(q[0], k, v, 1 / np.sqrt(128))
    assert np.linalg.norm(out - exact) / np.linalg.norm(exact) < 0.2


def test_bf16_baseline_oracle():
    cfg = _cfg(D=128, Bh=128)
    rng = np.random.default_rng(8)
    k = bf16_round(rng.standard_normal((77, 1, 128)).astype(np.float32))
    v = bf16_round(rng.standard_normal((77, 1, 128)).astype(np.float32))
    cache = OracleBF16Cache(cfg, _table())
    cache.append(0, [1], [0, 77], k, v)
    q = bf16_round(rng.standard_normal((1, 4, 128)).astype(np.float32))
    out = decode_attention_bf16(cache, 0, [1], q)["out_f64"][0]
    np.testing.assert_allclose(out, _sdpa(q[0], k, v, 1 / np.sqrt(128)), atol=1e-12)


def test_empty_sequence_gives_zero_row():
    cache = OracleKV4Cache(_cfg(), _table())
    rng = np.random.default_rng(9)
    k = bf16_round(rng.standard_normal((5, 1, 64)).astype(np.float32))
    cache.append(0, [1], [0, 5], k, k)
    q = bf16_round(rng.standard_normal((2, 4, 64)).astype(np.float32))
    out = decode_attention(cache, 0, [0, 1], q)["out_f64"]
    assert np.all(out[0] == 0) and np.all(np.abs(out[1]) > 0)


# ---- several query tokens per sequence (causal over the last T positions)

def _sdpa_causal(q, k, v, scale):
    """torch SDPA with an explicit boolean mask: query token i of T sees keys 0 .. L - T + i."""
    T, Hq, D = q.shape
    L, Hkv, _ = k.shape
    G = Hq // Hkv
    qt = torch.from_numpy(np.asarray(q, np.float64)).permute(1, 0, 2)          # [Hq, T, D]
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]     # [T, L]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale).permute(
        1, 0, 2).numpy()


def test_extend_quantization_free_reduction_to_causal_sdpa():
    # exact encodings (as in the decode reduction above): the multi-token result
    # is torch's causally masked attention on the inputs, for the protected view
    # (INT8 sinks and window, INT4 in between) and for the INT4-only view
    cfg = _cfg(Bh=1, W=16, Hkv=2, Hq=4)
    rng = np.random.default_rng(10)
    L, T = 70, 3
    codes = rng.integers(0, 16, (L, 2, 64))
    codes[:, :, 0], codes[:, :, 1] = 0, 15
    k = (codes * (17 / 64) - 2.0).astype(np.float32)
    v = (np.roll(codes, 5, axis=2) * (17 / 128) + 1.0).astype(np.float32)
    q = bf16_round(rng.standard_normal((1, T, 4, 64)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [1], [0, L], k, v)
    want = _sdpa_causal(q[0], k, v, 0.125)
    for protected in (True, False):
        got = extend_attention(cache, 0, [1], q, protected=protected)["out_f64"][0]
        np.testing.assert_allclose(got, want, atol=1e-12)


def test_extend_brute_force_loops():
    # tiny, exact encodings, every score and weight written out by hand
    cfg = _cfg(Bh=1, S=0, W=4, Hkv=1, Hq=2)
    rng = np.random.default_rng(11)
    L, T, D = 6, 3, 64
    codes = rng.integers(0, 16, (L, 1, D))
    codes[:, :, 0], codes[:, :, 1] = 0, 15
    k = (codes * (17 / 64)).astype(np.float32)
    v = (codes[:, :, ::-1] * (17 / 64) - 1.0).astype(np.float32)
    q = bf16_round(rng.standard_normal((1, T, 2, D)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0], [0, L], k, v)
    got = extend_attention(cache, 0, [0], q, scale=0.2)["out_f64"][0]
    for i in range(T):
        last = L - T + i
        for j in range(2):
            s = [0.2 * sum(float(q[0, i, j, d]) * float(k[p, 0, d]) for d in range(D)) for p in range(last + 1)]
            m = max(s)
            e = [np.exp(x - m) for x in s]
            o = [sum(e[p] * float(v[p, 0, d]) for p in range(last + 1)) / sum(e) for d in range(D)]
            np.testing.assert_allclose(got[i, j], o, rtol=1e-12, atol=1e-13)


def test_extend_later_positions_do_not_reach_earlier_tokens():
    # changing the newest position changes only the last query token's row
    cfg = _cfg(D=128, Bh=128, W=32, Hkv=1, Hq=4)
    rng = np.random.default_rng(12)
    L, T = 90, 4
    k = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    v = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    q = bf16_round(rng.standard_normal((1, T, 4, 128)).astype(np.float32))
    outs = []
    for bump in (0.0, 3.0):
        v2 = v.copy()
        v2[L - 1] += bump
        cache = OracleKV4Cache(cfg, _table())
        cache.append(0, [0], [0, L], k, v2)
        outs.append(extend_attention(cache, 0, [0], q)["out_f64"][0])
    assert np.array_equal(outs[0][:T - 1], outs[1][:T - 1])
    assert np.all(np.abs(outs[0][T - 1] - outs[1][T - 1]).max(axis=-1) > 1e-3)


def test_extend_one_token_is_decode_and_short_sequences_give_zero_rows():
    cfg = _cfg(D=64, Bh=64, W=8)
    rng = np.random.default_rng(13)
    k = bf16_round(rng.standard_normal((40, 1, 64)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0, 1], [0, 38, 40], k, k * 0.5)                 # lengths 38 and 2
    q1 = bf16_round(rng.standard_normal((2, 4, 64)).astype(np.float32))
    np.testing.assert_array_equal(extend_attention(cache, 0, [0, 1], q1[:, None])["out_f64"][:, 0],
                                  decode_attention(cache, 0, [0, 1], q1)["out_f64"])
    q5 = bf16_round(rng.standard_normal((2, 5, 4, 64)).astype(np.float32))
    out = extend_attention(cache, 0, [0, 1], q5)["out_f64"]
    assert np.all(out[1, :3] == 0) and np.all(np.abs(out[1, 3:]).max(axis=-1) > 0)   # L = 2 < T = 5
    assert np.all(np.abs(out[0]).max(axis=-1) > 0)


# ---- rotations folded into the caller's projections

def test_folded_rotations_reduce_to_the_default_path():
    # q_rotated with q' = bf16(H q) is the default path on q; out_rotated is the
    # default output taken back into the rotated basis (H symmetric, H H = I)
    cfg = _cfg(D=128, Bh=64, W=16, Hkv=1, Hq=4)
    rng = np.random.default_rng(14)
    L = 60
    k = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    v = bf16_round(rng.standard_normal((L, 1, 128)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0], [0, L], k, v)
    q = bf16_round(rng.standard_normal((1, 4, 128)).astype(np.float32))
    H = block_diag_hadamard(128, 64)
    base = decode_attention(cache, 0, [0], q)
    qr = base["q_rot"]
    np.testing.assert_array_equal(decode_attention(cache, 0, [0], qr, q_rotated=True)["out_f64"], base["out_f64"])
    rot = decode_attention(cache, 0, [0], q, out_rotated=True)["out_f64"]
    np.testing.assert_allclose(rot, base["out_f64"] @ H, atol=1e-12)
    np.testing.assert_allclose(rot @ H, base["out_f64"], atol=1e-12)
    both = extend_attention(cache, 0, [0], qr[:, None], q_rotated=True, out_rotated=True)["out_f64"][:, 0]
    np.testing.assert_allclose(both, rot, atol=1e-15)


def test_folded_rotations_are_the_identity_without_rotation():
    cfg = _cfg(D=64, Bh=1, W=8)
    rng = np.random.default_rng(15)
    k = bf16_round(rng.standard_normal((20, 1, 64)).astype(np.float32))
    cache = OracleKV4Cache(cfg, _table())
    cache.append(0, [0], [0, 20], k, k)
    q = bf16_round(rng.standard_normal((1, 4, 64)).astype(np.float32))
    ref = decode_attention(cache, 0, [0], q)["out_f64"]
    for qr in (False, True):
        for orot in (False, True):
            np.testing.assert_array_equal(decode_attention(cache, 0, [0], q, q_rotated=qr, out_rotated=orot)["out_f64"],
                                          ref)

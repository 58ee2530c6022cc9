"""Pins of the oracle's paged cache: placement, protection rules and the effective view."""

import numpy as np
import pytest

from oracle import OracleKV4Cache, OracleBF16Cache, fwht_fp32, quantize_groups, dequantize_groups, bf16_round
from oracle.cache import prot_slot, is_protected, n_prot_tiles


def _cfg(D=64, Hkv=2, P=16, S=4, W=32, Bh=64, pages=64, mpps=16, seqs=3, layers=2):
    return dict(num_layers=layers, max_seqs=seqs, num_q_heads=4 * Hkv, num_kv_heads=Hkv, head_dim=D,
                page_size=P, num_pages=pages, max_pages_per_seq=mpps, hadamard_block=Bh,
                sink_tokens=S, recent_window=W)


def _table(cfg, seed=0):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(cfg["num_pages"])
    t = np.full((cfg["max_seqs"], cfg["max_pages_per_seq"]), -1, np.int32)
    k = 0
    for s in range(cfg["max_seqs"]):
        n = min(cfg["max_pages_per_seq"], (cfg["num_pages"] - k))
        t[s, :n] = perm[k:k + n]
        k += n
    return t


def _kv(n, Hkv, D, seed):
    rng = np.random.default_rng(seed)
    k = bf16_round(rng.standard_normal((n, Hkv, D)).astype(np.float32) * 2)
    v = bf16_round(rng.standard_normal((n, Hkv, D)).astype(np.float32))
    return k, v


def _direct_view(x, Bh, L, S, W, protected=True):
    """Independent construction: each position quantized with the bits its position calls for."""
    xr = fwht_fp32(x[:L], Bh)
    out = np.zeros_like(xr)
    for p in range(L):
        bits = 8 if protected and is_protected(p, L, S, W) else 4
        c, s, z = quantize_groups(xr[p:p + 1], bits)
        out[p] = dequantize_groups(c, s, z)[0]
    return out


def test_slot_rules():
    S, W = 4, 32
    assert [prot_slot(p, S, W) for p in range(4)] == [0, 1, 2, 3]
    assert prot_slot(4, S, W) == 4 and prot_slot(35, S, W) == 35 and prot_slot(36, S, W) == 4
    assert n_prot_tiles(4, 32) == 3 and n_prot_tiles(4, 128) == 9 and n_prot_tiles(0, 16) == 1
    for L in range(1, 200):
        slots = sorted(prot_slot(p, S, W) for p in range(L) if is_protected(p, L, S, W))
        assert slots == list(range(min(L, S + W)))   # the protected slots are a prefix of the store


@pytest.mark.parametrize("chunks", [[1] * 120, [50, 1, 1, 37, 31], [120], [3, 80, 2, 35]])
def test_effective_view_equals_direct_construction(chunks):
    cfg = _cfg()
    cache = OracleKV4Cache(cfg, _table(cfg))
    total = sum(chunks)
    k, v = _kv(total, 2, 64, 1)
    pos = 0
    for n in chunks:
        cache.append(1, [2], [0, n], k[pos:pos + n], v[pos:pos + n])
        pos += n
        L = pos
        kh, vh = cache.view(1, 2)
        np.testing.assert_array_equal(kh, _direct_view(k, 64, L, 4, 32))
        np.testing.assert_array_equal(vh, _direct_view(v, 64, L, 4, 32))
        kh4, vh4 = cache.view(1, 2, protected=False)
        np.testing.assert_array_equal(kh4, _direct_view(k, 64, L, 4, 32, protected=False))
    assert cache.seq_lens[1, 2] == total and cache.seq_lens[0, 2] == 0


def test_bulk_and_incremental_appends_store_identical_bytes():
    cfg = _cfg(D=128, Hkv=1, Bh=128, W=32)
    k, v = _kv(150, 1, 128, 2)
    a = OracleKV4Cache(cfg, _table(cfg))
    b = OracleKV4Cache(cfg, _table(cfg))
    a.append(0, [0], [0, 150], k, v)
    for i in range(150):
        b.append(0, [0], [0, 1], k[i:i + 1], v[i:i + 1])
    assert a.pages.keys() == b.pages.keys()
    for key in a.pages:
        np.testing.assert_array_equal(a.pages[key], b.pages[key])
    # the protected store agrees on every slot of the effective view
    for p in range(150):
        if is_protected(p, 150, 4, 32):
            s = prot_slot(p, 4, 32)
            np.testing.assert_array_equal(a.prot[(0, 0)][s // 16], b.prot[(0, 0)][s // 16])
    np.testing.assert_array_equal(a.view(0, 0)[0], b.view(0, 0)[0])


def test_multi_sequence_append_and_placement():
    cfg = _cfg()
    t = _table(cfg, 3)
    cache = OracleKV4Cache(cfg, t)
    k, v = _kv(40, 2, 64, 4)
    cache.append(0, [2, 0], [0, 25, 40], k, v)
    assert cache.seq_lens[0, 2] == 25 and cache.seq_lens[0, 0] == 15
    # token 17 of seq 2 lives on page t[2, 1], slot 1 of that page's only tile
    assert (0, int(t[2, 1])) in cache.pages and (0, int(t[0, 0])) in cache.pages
    np.testing.assert_array_equal(cache.view(0, 0)[0], _direct_view(k[25:], 64, 15, 4, 32))


def test_page_size_64_and_ragged_tail():
    cfg = _cfg(P=64, mpps=4, W=16)
    cache = OracleKV4Cache(cfg, _table(cfg))
    k, v = _kv(131, 2, 64, 5)
    cache.append(0, [1], [0, 131], k, v)
    np.testing.assert_array_equal(cache.view(0, 1)[1], _direct_view(v, 64, 131, 4, 16))


def test_capacity_and_unmapped_pages():
    cfg = _cfg(mpps=2)
    cache = OracleKV4Cache(cfg, _table(cfg))
    k, v = _kv(33, 2, 64, 6)
    with pytest.raises(ValueError):
        cache.append(0, [0], [0, 33], k, v)
    t = _table(cfg)
    t[1, 0] = -1
    cache = OracleKV4Cache(cfg, t)
    with pytest.raises(ValueError):
        cache.append(0, [1], [0, 1], k[:1], v[:1])


def test_no_sinks_and_window_larger_than_context():
    cfg = _cfg(S=0, W=64)
    cache = OracleKV4Cache(cfg, _table(cfg))
    k, v = _kv(40, 2, 64, 7)
    cache.append(0, [0], [0, 40], k, v)
    np.testing.assert_array_equal(cache.view(0, 0)[0], _direct_view(k, 64, 40, 0, 64))


def test_bf16_cache_round_trip():
    cfg = _cfg(D=128)
    cache = OracleBF16Cache(cfg, _table(cfg))
    k, v = _kv(70, 2, 128, 8)
    cache.append(0, [1], [0, 30], k[:30], v[:30])
    cache.append(0, [1], [0, 40], k[30:], v[30:])
    kk, vv = cache.view(0, 1)
    np.testing.assert_array_equal(kk, k)
    np.testing.assert_array_equal(vv, v)


def test_largest_page_and_protected_window():
    """The largest shapes the library accepts: 1024-token pages and S + W = 4096 protected positions. The
    effective view after ragged appends equals the per-position construction, the protected slots fill the
    store's prefix, and the window wraps once the sequence passes S + W."""
    S, W = 96, 4000
    cfg = _cfg(D=64, Hkv=1, P=1024, S=S, W=W, Bh=64, pages=6, mpps=6, seqs=1, layers=1)
    cache = OracleKV4Cache(cfg, _table(cfg))
    k, v = _kv(4300, 1, 64, 7)
    pos = 0
    for n in (3000, 1, 1095, 204):                      # crosses S + W = 4096 and four page boundaries
        cache.append(0, [0], [0, n], k[pos:pos + n], v[pos:pos + n])
        pos += n
    assert pos == 4300 and cache.seq_lens[0, 0] == 4300
    kh, vh = cache.view(0, 0)
    np.testing.assert_array_equal(kh, _direct_view(k, 64, pos, S, W))
    np.testing.assert_array_equal(vh, _direct_view(v, 64, pos, S, W))
    assert n_prot_tiles(S, W) == 256
    slots = sorted(prot_slot(p, S, W) for p in range(pos) if is_protected(p, pos, S, W))
    assert slots == list(range(S + W))

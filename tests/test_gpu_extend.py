"""GPU parity of the multi-token query path (kv4_extend_attention): the last T
positions of every sequence attend causally over the cache, each query token
over the positions up to its own.  Compared with the oracle's extend_attention
on the same seeded inputs: every (query token, head) ratio that fits one
8-column operand, more query rows than that (several passes), lengths below T, empty sequences, a recent window shorter
than T (the causal tail then reaches INT4 pages), the INT4-only view, one long
sequence split over every CTA, and T = 1 against decode attention."""

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, REL_L2, MAX_ABS, f32
from oracle import extend_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _populate(pair, rng, seqs, lens, Hkv, D, chunk=256):
    done = np.zeros(len(seqs), np.int64)
    lens = np.asarray(lens, np.int64)
    while np.any(done < lens):
        counts = np.minimum(lens - done, rng.integers(1, chunk + 1, len(seqs)))
        counts[done >= lens] = 0
        n = int(counts.sum())
        k = bf16_values((n, Hkv, D), rng, 2.0, outlier_ch=[1, D // 2 + 3], outlier=10.0)
        v = bf16_values((n, Hkv, D), rng)
        pair.append(0, seqs, [int(c) for c in counts], k, v)
        done += counts


def _extend(pair, seqs, q, mode=0):
    ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    return pair.gpu.extend_attention(0, ids, q.cuda().contiguous(), mode=mode)


def _check(kv4, pair, seqs, q, mode=0):
    protected = not (mode & kv4.KV4_MODE_INT4_ONLY)
    ref = extend_attention(pair.orc, 0, seqs, f32(q), protected=protected)
    out = _extend(pair, seqs, q, mode)
    out32 = _extend(pair, seqs, q, mode | kv4.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)
    return out, ref


@pytest.mark.parametrize("Hq,Hkv,T", [(32, 8, 2), (16, 8, 2), (16, 8, 4), (8, 8, 8), (8, 8, 4), (24, 8, 2),
                                      (8, 8, 2), (16, 4, 2)])
def test_extend_matches_oracle(kv4, Hq, Hkv, T):
    rng = np.random.default_rng(100 * Hq + 10 * Hkv + T)
    D, n = 128, 7
    mpps = 1500 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=64, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    lens = [1, 1500, 67, 0, 333, T, 131]          # below T, empty, exactly T, ring wrapped, ring partly filled
    _populate(pair, rng, list(range(n)), lens, Hkv, D)
    seqs = [5, 1, 0, 3, 4, 2, 6]
    q = bf16_values((n, T, Hq, D), rng)
    out, _ = _check(kv4, pair, seqs, q)
    _check(kv4, pair, seqs, q, mode=kv4.KV4_MODE_INT4_ONLY)
    assert torch.all(out[seqs.index(3)] == 0)                      # empty sequence
    assert torch.all(out[seqs.index(0), :T - 1] == 0)              # L = 1: only the last token sees a position


@pytest.mark.parametrize("T", [4, 8])
def test_extend_window_shorter_than_query(kv4, T):
    """W = 4 < T: the causal tail of the query tokens lies partly in the INT4 pages."""
    rng = np.random.default_rng(T)
    D, Hkv, Hq, n = 64, 4, 4, 5
    mpps = 400 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=64, S=2, W=4, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, list(range(n)), [400, 37, 8, 3, 17], Hkv, D, chunk=64)
    _check(kv4, pair, list(range(n)), bf16_values((n, T, Hq, D), rng))


def test_extend_one_long_sequence_over_every_cta(kv4):
    rng = np.random.default_rng(77)
    D, Hkv, Hq, L, T = 128, 8, 32, 5000, 2
    mpps = L // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=mpps + 4, mpps=mpps, max_seqs=2)
    pair = Pair(cfg, random_table(2, mpps, mpps + 4, rng))
    _populate(pair, rng, [0], [L], Hkv, D, chunk=2048)
    q = bf16_values((1, T, Hq, D), rng)
    _check(kv4, pair, [0], q)
    _check(kv4, pair, [0], q, mode=kv4.KV4_MODE_INT4_ONLY)


def test_extend_one_token_is_decode(kv4):
    rng = np.random.default_rng(78)
    D, Hkv, Hq, n = 128, 8, 32, 4
    mpps = 900 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, list(range(n)), [900, 17, 450, 0], Hkv, D)
    q = bf16_values((n, Hq, D), rng)
    dec = pair.attention(0, [0, 1, 2, 3], q)
    ext = _extend(pair, [0, 1, 2, 3], q[:, None])
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    d = (ext[:, 0].float() - dec.float()).abs()
    assert torch.equal(ext[:, 0], dec), (d.max().item(), torch.nonzero(d).tolist()[:16])


@pytest.mark.parametrize("Hq,Hkv,T", [(32, 8, 3), (32, 8, 4), (64, 8, 2), (16, 8, 7)])
def test_extend_in_several_passes(kv4, Hq, Hkv, T):
    """More query rows than one 8-column operand: passes of 8 / G tokens, each with its causal offset."""
    rng = np.random.default_rng(1000 * Hq + T)
    D, n = 128, 5
    mpps = 700 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=64, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    lens = [700, 2, 0, T, 90]
    _populate(pair, rng, list(range(n)), lens, Hkv, D)
    seqs = [4, 0, 2, 1, 3]
    q = bf16_values((n, T, Hq, D), rng)
    out, _ = _check(kv4, pair, seqs, q)
    _check(kv4, pair, seqs, q, mode=kv4.KV4_MODE_INT4_ONLY)
    assert torch.all(out[seqs.index(2)] == 0)


@pytest.mark.parametrize("Hq,Hkv,T", [(4, 1, 2), (8, 2, 2), (6, 2, 3), (3, 3, 2)])
def test_extend_head_groups_of_one_and_two(kv4, Hq, Hkv, T):
    """KV-head counts that are not a multiple of 4 run in groups of 2 or 1 KV heads."""
    rng = np.random.default_rng(500 + 10 * Hkv + T)
    D, n = 64, 4
    mpps = 700 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=64, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, list(range(n)), [700, 1, 0, 45], Hkv, D, chunk=128)
    q = bf16_values((n, T, Hq, D), rng)
    out, _ = _check(kv4, pair, [3, 0, 2, 1], q)
    _check(kv4, pair, [3, 0, 2, 1], q, mode=kv4.KV4_MODE_INT4_ONLY)
    assert torch.all(out[2] == 0)


def test_extend_rejects_bad_arguments(kv4):
    rng = np.random.default_rng(79)
    cfg2 = cfg_dict(D=64, Hq=4, Hkv=2, P=16, Bh=64, S=4, W=32, num_pages=8, mpps=4, max_seqs=2)
    pair2 = Pair(cfg2, random_table(2, 4, 8, rng))
    with pytest.raises(kv4.KV4Error):                              # q_len < 1
        _extend(pair2, [0, 1], bf16_values((2, 0, 4, 64), rng))

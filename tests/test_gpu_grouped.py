"""GPU parity of the page-major attention path (KV heads a multiple of 4) in the
situations its single-launch plan has to get right: more head groups than one
planning chunk, runs of empty sequences, one sequence spread over every CTA,
every query-head ratio, and repeated calls (the merge counters of one call must
not leak into the next)."""

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, REL_L2, MAX_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _check(pair, seqs, q, mode=0):
    import int4_kv_cache_paged_b200 as m
    protected = not (mode & m.KV4_MODE_INT4_ONLY)
    ref = pair.oracle_attention(0, seqs, q, protected=protected)
    out = pair.attention(0, seqs, q, mode=mode)
    out32 = pair.attention(0, seqs, q, mode=mode | m.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)
    assert pair.gpu.status() == 0
    return out


def _populate(pair, rng, seqs, lens, Hkv, D, chunk=64):
    """Append `lens[i]` tokens to seqs[i], in a few ragged rounds."""
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


def test_many_groups_and_runs_of_empty_sequences(kv4):
    """600 head groups (four planning chunks of the 160-thread CTA), 40 consecutive
    empty sequences owned by one CTA, many groups split between CTAs."""
    rng = np.random.default_rng(21)
    n, D, Hkv, Hq, mpps = 300, 64, 8, 16, 8
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=64, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    lens = rng.integers(1, 120, n)
    lens[rng.random(n) < 0.3] = 0
    lens[100:140] = 0
    seqs = list(range(n))
    _populate(pair, rng, seqs, lens, Hkv, D)
    order = list(rng.permutation(n))
    out = _check(pair, order, bf16_values((n, Hq, D), rng))
    empty = [i for i, s in enumerate(order) if lens[s] == 0]
    assert torch.all(out[empty] == 0)


@pytest.mark.parametrize("Hq", [8, 16, 32, 64])
def test_one_long_sequence_over_every_cta(kv4, Hq):
    """One 5000-token sequence: its stages spread over every CTA, merged from ~150 partials."""
    rng = np.random.default_rng(Hq)
    D, Hkv, L = 128, 8, 5000
    mpps = L // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=mpps + 4, mpps=mpps, max_seqs=2)
    pair = Pair(cfg, random_table(2, mpps, mpps + 4, rng))
    _populate(pair, rng, [0], [L], Hkv, D, chunk=2048)   # sequence 0 owns the first mpps pages
    q = bf16_values((1, Hq, D), rng)
    _check(pair, [0], q)
    _check(pair, [0], q, mode=kv4.KV4_MODE_INT4_ONLY)


@pytest.mark.parametrize("Hq,Hkv", [(64, 8), (16, 8), (48, 16), (24, 8)])
def test_query_head_ratios_mixed_lengths(kv4, Hq, Hkv):
    """G = 8, 2, 3 and 3 with 16 KV heads (two groups per sequence), lengths from 1 to 1500."""
    rng = np.random.default_rng(Hq * 100 + Hkv)
    D, n = 128, 6
    mpps = 1500 // 32 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=32, Bh=128, S=4, W=64, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    lens = [1, 1500, 67, 0, 333, 68]
    _populate(pair, rng, list(range(n)), lens, Hkv, D, chunk=512)
    _check(pair, [5, 1, 0, 3, 4, 2], bf16_values((n, Hq, D), rng))


def test_repeated_calls_are_identical(kv4):
    """Identical calls in a row give the same bits (the split and the merge order depend only on
    the lengths; the merge counters are re-armed by the epoch)."""
    rng = np.random.default_rng(5)
    D, Hkv, Hq, n = 128, 8, 32, 4
    mpps = 900 // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, list(range(n)), [900, 17, 450, 300], Hkv, D, chunk=300)
    q = bf16_values((n, Hq, D), rng)
    first = _check(pair, [0, 1, 2, 3], q)
    for _ in range(3):
        again = pair.attention(0, [0, 1, 2, 3], q)
        assert torch.equal(again, first)
    # a subset in another order (another split of the stages), then the full batch again
    _check(pair, [2, 0], q[[2, 0]])
    assert torch.equal(pair.attention(0, [0, 1, 2, 3], q), first)


def test_more_sequences_than_max_seqs_is_rejected(kv4):
    rng = np.random.default_rng(6)
    cfg = cfg_dict(D=64, Hq=16, Hkv=8, P=16, Bh=64, S=4, W=32, num_pages=8, mpps=4, max_seqs=2)
    pair = Pair(cfg, random_table(2, 4, 8, rng))
    with pytest.raises(kv4.KV4Error):
        pair.attention(0, [0, 1, 0], bf16_values((3, 16, 64), rng))

"""GPU parity of the fused decode step (kv4_decode_step): appending one token
per sequence and attending in one call gives the same bytes in the cache, the
same lengths and the same outputs, bit for bit, as kv4_rotate_quantize_append
followed by kv4_decode_attention, and matches the oracle; several steps in a
row cross page boundaries and wrap the INT8 ring; empty sequences start; with
RoPE the new keys and the queries are turned at their positions."""

import numpy as np
import pytest
import torch

import workloads
from kvhelpers import (Pair, cfg_dict, random_table, bf16_values, check_bf16_out, compare_int4_pages,
                       compare_int8_store, REL_L2, f32)
from oracle import decode_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _twins(Hq, Hkv, D, Bh, lens, seed, rope=None):
    """Two GPU caches (and one oracle) with identical contents."""
    rng = np.random.default_rng(seed)
    n = len(lens)
    mpps = (max(lens) + 40) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=Bh, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    table = random_table(n, mpps, n * mpps, rng)
    a, b = Pair(cfg, table), Pair(cfg, table)
    cs = None
    if rope is not None:
        cs = workloads.rope_cos_sin(4096, rope[0])
        for p in (a, b):
            p.gpu.set_rope(torch.from_numpy(cs), rope[0], rope[1])
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0, outlier_ch=[2], outlier=9.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    for p in (a, b):
        p.gpu.append(0, torch.arange(n, dtype=torch.int32, device="cuda"), torch.from_numpy(cu).cuda(), k.cuda(),
                     v.cuda(), total_new=int(cu[-1]), rope=rope is not None)
    a.orc.append(0, list(range(n)), cu, f32(k), f32(v), rope=None if rope is None else (cs, rope[0], rope[1]))
    return a, b, rng, cs


@pytest.mark.parametrize("Hq,Hkv,D,Bh,rope", [(32, 8, 128, 128, None), (16, 4, 64, 64, None),
                                              (32, 8, 128, 128, (128, 0)), (8, 8, 64, 32, (32, 1)),
                                              (4, 1, 64, 64, None), (8, 2, 128, 128, None), (6, 6, 64, 64, None),
                                              (4, 2, 64, 64, (64, 0))])
def test_step_equals_append_then_attention(kv4, Hq, Hkv, D, Bh, rope):
    lens = [300, 0, 15, 31, 47, 1]
    a, b, rng, cs = _twins(Hq, Hkv, D, Bh, lens, Hq + D + (0 if rope is None else rope[1] + 1), rope)
    n = len(lens)
    order = [3, 0, 5, 1, 4, 2]
    ids = torch.tensor(order, dtype=torch.int32, device="cuda")
    mode = kv4.KV4_MODE_ROPE_Q if rope is not None else 0
    for step in range(20):                                   # crosses page boundaries, wraps the W = 32 ring
        k = bf16_values((n, Hkv, D), rng, 2.0)
        v = bf16_values((n, Hkv, D), rng)
        q = bf16_values((n, Hq, D), rng)
        a.gpu.append(0, ids, torch.arange(n + 1, dtype=torch.int32, device="cuda"), k.cuda(), v.cuda(), total_new=n,
                     rope=rope is not None)
        out_a = a.gpu.attention(0, ids, q.cuda(), mode=mode)
        out_b = b.gpu.decode_step(0, ids, k.cuda(), v.cuda(), q.cuda(), mode=mode)
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b), step
        a.orc.append(0, order, np.arange(n + 1), f32(k), f32(v),
                     rope=None if rope is None else (cs, rope[0], rope[1]))
        if step in (0, 19):
            ref = decode_attention(a.orc, 0, order, f32(q), rope=None if rope is None else (cs, rope[0], rope[1]))
            rel, excess = check_bf16_out(out_b, ref)
            assert rel <= REL_L2 and excess <= 0, (step, rel, excess)
    assert a.gpu.status() == 0 and b.gpu.status() == 0
    assert torch.equal(a.gpu.seq_lens(), b.gpu.seq_lens())
    # every written byte of both caches against the oracle (slots never written hold whatever the buffer held)
    b.orc = a.orc
    for pair in (a, b):
        assert compare_int4_pages(pair, 0, list(range(n))) == []
        assert compare_int8_store(pair, 0, list(range(n))) == []


def test_step_flags_an_unmapped_page_and_rejects_too_many_kv_heads(kv4):
    rng = np.random.default_rng(90)
    cfg = cfg_dict(D=64, Hq=8, Hkv=4, P=16, Bh=64, S=4, W=16, num_pages=4, mpps=4, max_seqs=2)
    table = np.full((2, 4), -1, np.int32)
    table[0, :2] = [0, 1]
    pair = Pair(cfg, table)
    ids = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    k, v, q = (bf16_values((2, 4, 64), rng).cuda(), bf16_values((2, 4, 64), rng).cuda(),
               bf16_values((2, 8, 64), rng).cuda())
    pair.gpu.decode_step(0, ids, k, v, q)
    torch.cuda.synchronize()
    assert pair.gpu.status() & kv4.KV4_DEV_BAD_PAGE          # sequence 1 has no page
    # the step kernel runs two warps per KV head in one block: at most 16 KV heads
    cfg2 = cfg_dict(D=64, Hq=32, Hkv=32, P=16, Bh=64, S=4, W=16, num_pages=8, mpps=4, max_seqs=2)
    pair2 = Pair(cfg2, random_table(2, 4, 8, rng))
    k2, v2, q2 = (bf16_values((2, 32, 64), rng).cuda(), bf16_values((2, 32, 64), rng).cuda(),
                  bf16_values((2, 32, 64), rng).cuda())
    with pytest.raises(kv4.KV4Error) as e:
        pair2.gpu.decode_step(0, ids, k2, v2, q2)
    assert e.value.code == kv4.KV4_ERR_UNSUPPORTED

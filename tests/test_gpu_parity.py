"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on identical seeded inputs.

Codes, scales and their placement must match bit for bit; dequantized values
bit for bit; attention within the stated tolerances (see kvhelpers)."""

import numpy as np
import pytest
import torch

import workloads
from kvhelpers import (Pair, cfg_dict, random_table, bf16_values, f32, compare_int4_pages, compare_int8_store,
                       compare_bf16_pages, check_bf16_out, check_f32_out, REL_L2, MAX_ABS, BF16_REL_L2, BF16_MAX_ABS)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _assert_attention(pair, layer, seq_ids, q, scale=0.0, protected=True):
    import int4_kv_cache_paged_b200 as m
    mode = 0 if protected else m.KV4_MODE_INT4_ONLY
    ref = pair.oracle_attention(layer, seq_ids, q, scale, protected=protected)
    out = pair.attention(layer, seq_ids, q, scale=scale, mode=mode)
    out32 = pair.attention(layer, seq_ids, q, scale=scale, mode=mode | m.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)
    assert pair.gpu.status() == 0


def test_tiny_workload_decode_steps(kv4):
    """The tiny workload: bulk-populate L-1 tokens, then 4 decode steps of append + attention."""
    w = workloads.workload("tiny")
    L = workloads.context_lengths(w)
    table, num_pages, mpps = workloads.block_table(w, L)
    cfg = workloads.cache_config(w, num_pages, mpps)
    pair = Pair(cfg, table)
    seqs = list(range(w["batch"]))
    kv = [workloads.kv_sequence(w, 0, s, int(L[s]) - 1 + w["steps"], device="cuda") for s in seqs]
    k0 = torch.cat([kv[s][0][:L[s] - 1] for s in seqs]).cpu()
    v0 = torch.cat([kv[s][1][:L[s] - 1] for s in seqs]).cpu()
    pair.append(0, seqs, [int(L[s]) - 1 for s in seqs], k0, v0)
    assert compare_int4_pages(pair, 0, seqs) == []
    assert compare_int8_store(pair, 0, seqs) == []
    for step in range(w["steps"]):
        pos = [int(L[s]) - 1 + step for s in seqs]
        k1 = torch.stack([kv[s][0][pos[s]] for s in seqs]).cpu()
        v1 = torch.stack([kv[s][1][pos[s]] for s in seqs]).cpu()
        pair.append(0, seqs, [1] * len(seqs), k1, v1)
        lens = pair.gpu.seq_lens()[0, :len(seqs)].cpu().numpy()
        np.testing.assert_array_equal(lens, [p + 1 for p in pos])
        assert compare_int4_pages(pair, 0, seqs) == []
        assert compare_int8_store(pair, 0, seqs) == []
        q = workloads.queries(w, 0, step, device="cpu")
        _assert_attention(pair, 0, seqs, q)


VARIANTS = [
    # D, Hq, Hkv, P, Bh, S, W
    (128, 32, 8, 16, 128, 4, 128),
    (128, 8, 8, 32, 64, 0, 16),
    (128, 16, 2, 64, 128, 4, 256),
    (64, 8, 1, 16, 64, 4, 32),
    (64, 16, 2, 32, 16, 7, 21),
    (128, 4, 4, 16, 1, 2, 16),
    (64, 8, 4, 64, 32, 1, 1),
]


@pytest.mark.parametrize("D,Hq,Hkv,P,Bh,S,W", VARIANTS)
def test_ragged_appends_and_attention(kv4, D, Hq, Hkv, P, Bh, S, W):
    rng = np.random.default_rng(hash((D, Hq, Hkv, P, Bh, S, W)) % 2 ** 32)
    max_seqs, mpps = 4, 40 // (P // 16) + 2
    num_pages = max_seqs * mpps
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=P, Bh=Bh, S=S, W=W, num_pages=num_pages, mpps=mpps, max_seqs=max_seqs)
    table = random_table(max_seqs, mpps, num_pages, rng)
    pair = Pair(cfg, table)
    seqs = [3, 0, 2]
    # ragged rounds: bulk, zero-length, single tokens, a round longer than W
    rounds = [[37, 0, 150], [1, 1, 1], [0, 290, 2], [17, 3, 0], [1, 1, 1]]
    for counts in rounds:
        n = sum(counts)
        k = bf16_values((n, Hkv, D), rng, 2.0, outlier_ch=[3, D // 2], outlier=12.0)
        v = bf16_values((n, Hkv, D), rng)
        pair.append(0, seqs, counts, k, v)
        assert compare_int4_pages(pair, 0, seqs) == []
        assert compare_int8_store(pair, 0, seqs) == []
        q = bf16_values((len(seqs), Hq, D), rng)
        _assert_attention(pair, 0, seqs, q)
    _assert_attention(pair, 0, seqs, bf16_values((3, Hq, D), rng), protected=False)
    _assert_attention(pair, 0, seqs[::-1], bf16_values((3, Hq, D), rng), scale=0.3)


@pytest.mark.parametrize("L", [1, 3, 4, 5, 16, 17, 35, 36, 37, 48, 131, 132, 133, 200, 321])
def test_edge_lengths(kv4, L):
    rng = np.random.default_rng(L)
    cfg = cfg_dict(D=64, Hq=8, Hkv=2, P=16, Bh=64, S=4, W=32, num_pages=64, mpps=32, max_seqs=2)
    pair = Pair(cfg, random_table(2, 32, 64, rng))
    k = bf16_values((L, 2, 64), rng, 3.0)
    v = bf16_values((L, 2, 64), rng)
    pair.append(0, [1], [L], k, v)
    assert compare_int4_pages(pair, 0, [1]) == [] and compare_int8_store(pair, 0, [1]) == []
    _assert_attention(pair, 0, [1], bf16_values((1, 8, 64), rng))
    _assert_attention(pair, 0, [1], bf16_values((1, 8, 64), rng), protected=False)


def test_dequantize_debug_bitexact(kv4):
    rng = np.random.default_rng(7)
    cfg = cfg_dict(D=128, Hq=8, Hkv=2, P=32, Bh=128, S=4, W=32, num_pages=40, mpps=10, max_seqs=2)
    pair = Pair(cfg, random_table(2, 10, 40, rng))
    k = bf16_values((250, 2, 128), rng, 4.0, outlier_ch=[9], outlier=15.0)
    v = bf16_values((250, 2, 128), rng)
    pair.append(0, [0], [250], k, v)
    for view, protected in ((kv4.KV4_VIEW_EFFECTIVE, True), (kv4.KV4_VIEW_INT4, False)):
        for start, count in ((0, 250), (3, 7), (200, 50)):
            kg, vg = pair.gpu.dequantize(0, 0, start, count, view)
            ko, vo = pair.orc.view(0, 0, protected=protected, start=start, count=count)
            np.testing.assert_array_equal(kg.cpu().numpy(), ko)
            np.testing.assert_array_equal(vg.cpu().numpy(), vo)


def test_empty_and_short_sequences(kv4):
    rng = np.random.default_rng(8)
    cfg = cfg_dict(D=128, Hq=8, Hkv=2, P=16, Bh=128, S=4, W=16, num_pages=32, mpps=8, max_seqs=3)
    pair = Pair(cfg, random_table(3, 8, 32, rng))
    pair.append(0, [1], [2], bf16_values((2, 2, 128), rng), bf16_values((2, 2, 128), rng))
    q = bf16_values((3, 8, 128), rng)
    out = pair.attention(0, [0, 1, 2], q, mode=kv4.KV4_MODE_OUT_F32).cpu().numpy()
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    ref = pair.oracle_attention(0, [1], q[1:2])
    assert np.max(np.abs(out[1] - ref["out_f64"][0])) <= MAX_ABS


def test_seq_reset_and_reuse(kv4):
    rng = np.random.default_rng(9)
    cfg = cfg_dict(D=64, Hq=4, Hkv=1, P=16, Bh=64, S=4, W=32, num_pages=32, mpps=8, max_seqs=2, layers=2)
    pair = Pair(cfg, random_table(2, 8, 32, rng))
    pair.append(1, [0], [70], bf16_values((70, 1, 64), rng), bf16_values((70, 1, 64), rng))
    pair.gpu.reset(0)
    assert pair.gpu.seq_lens()[:, 0].cpu().tolist() == [0, 0]
    from oracle import OracleKV4Cache
    pair.orc = OracleKV4Cache(cfg, pair.table)
    pair.append(1, [0], [40], bf16_values((40, 1, 64), rng), bf16_values((40, 1, 64), rng))
    assert compare_int4_pages(pair, 1, [0]) == [] and compare_int8_store(pair, 1, [0]) == []
    _assert_attention(pair, 1, [0], bf16_values((1, 4, 64), rng))


@pytest.mark.parametrize("D,P", [(128, 16), (64, 32), (128, 64)])
def test_bf16_baseline(kv4, D, P):
    rng = np.random.default_rng(D + P)
    mpps = 30 // (P // 16) + 1
    cfg = cfg_dict(D=D, Hq=16, Hkv=4, P=P, num_pages=3 * mpps, mpps=mpps, max_seqs=3)
    pair = Pair(cfg, random_table(3, mpps, 3 * mpps, rng), bf16=True)
    for counts in ([100, 0, 33], [1, 1, 1], [0, 200, 7]):
        n = sum(counts)
        pair.append(0, [0, 1, 2], counts, bf16_values((n, 4, D), rng, 2.0), bf16_values((n, 4, D), rng))
        assert compare_bf16_pages(pair, 0, [0, 1, 2]) == []
        q = bf16_values((3, 16, D), rng)
        ref = pair.oracle_attention(0, [0, 1, 2], q)
        out32 = pair.attention(0, [0, 1, 2], q, mode=kv4.KV4_MODE_OUT_F32)
        rel, mx = check_f32_out(out32, ref)
        assert rel <= BF16_REL_L2 and mx <= BF16_MAX_ABS, (rel, mx)
    assert pair.gpu.status() == 0


def test_device_faults_set_status_bits(kv4):
    rng = np.random.default_rng(10)
    cfg = cfg_dict(D=64, Hq=4, Hkv=1, P=16, Bh=64, S=4, W=32, num_pages=8, mpps=4, max_seqs=2)
    table = random_table(2, 4, 8, rng)
    table[1, 2] = -1
    pair = Pair(cfg, table)
    k, v = bf16_values((40, 1, 64), rng), bf16_values((40, 1, 64), rng)
    pair.append(0, [1], [40], k, v, oracle=False)            # positions 32..39 map to an unmapped page
    assert pair.gpu.status() & kv4.KV4_DEV_BAD_PAGE
    assert pair.gpu.status() == 0                            # reading clears the word
    big = bf16_values((65, 1, 64), rng)
    pair.append(0, [0], [65], big, big, oracle=False)        # capacity is 4 pages * 16 = 64 tokens
    assert pair.gpu.status() & kv4.KV4_DEV_OVERFLOW
    assert int(pair.gpu.seq_lens()[0, 0]) == 0               # the sequence was skipped
    pair.append(0, [5], [1], big[:1], big[:1], oracle=False)  # sequence id out of range
    assert pair.gpu.status() & kv4.KV4_DEV_BAD_SEQ
    nan = big[:1].clone()
    nan[0, 0, 3] = float("nan")
    pair.append(0, [0], [1], nan, big[:1], oracle=False)
    assert pair.gpu.status() & kv4.KV4_DEV_RANGE
    # the context is still usable
    pair.append(0, [0], [3], big[:3], big[:3], oracle=False)
    assert pair.gpu.status() == 0

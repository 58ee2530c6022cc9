"""GPU parity of the fused RoPE path: kv4_rope_rotate_quantize_append (RoPE of
each key at its position, then rotation and quantization) against the oracle
byte for byte, and attention with KV4_MODE_ROPE_Q (RoPE of each query at its
position) against the oracle, for both pair layouts, partial rotary dims,
groups of 4, 2 and 1 KV heads, decode and multi-token queries; a key past
the table is flagged and not written."""

import numpy as np
import pytest
import torch

import workloads
from kvhelpers import (Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, compare_int4_pages,
                       compare_int8_store, REL_L2, MAX_ABS, f32)
from oracle import decode_attention, extend_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _append(pair, rope, seqs, counts, k, v):
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    pair.gpu.append(0, torch.tensor(seqs, dtype=torch.int32, device="cuda"), torch.from_numpy(cu).cuda(),
                    k.cuda().contiguous(), v.cuda().contiguous(), total_new=int(cu[-1]), rope=True)
    pair.orc.append(0, list(seqs), cu, f32(k), f32(v), rope=rope)


def _build(kv4, Hq, Hkv, D, Bh, R, style, lens, seed, max_pos=40000):
    rng = np.random.default_rng(seed)
    n = len(lens)
    mpps = max(lens) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=Bh, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    cs = workloads.rope_cos_sin(max_pos, R)
    pair.gpu.set_rope(torch.from_numpy(cs), R, style)
    rope = (cs, R, style)
    done = np.zeros(n, np.int64)
    lens = np.asarray(lens, np.int64)
    while np.any(done < lens):                        # ragged rounds: positions continue across calls
        counts = np.minimum(lens - done, rng.integers(1, 200, n))
        counts[done >= lens] = 0
        tot = int(counts.sum())
        k = bf16_values((tot, Hkv, D), rng, 2.0, outlier_ch=[1, D // 2 + 3], outlier=10.0)
        v = bf16_values((tot, Hkv, D), rng)
        _append(pair, rope, list(range(n)), [int(c) for c in counts], k, v)
        done += counts
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    return pair, rope, rng


CASES = [(32, 8, 128, 128, 128, 0), (32, 8, 128, 128, 64, 1), (16, 8, 64, 64, 32, 0), (8, 2, 128, 64, 128, 1),
         (8, 2, 64, 32, 64, 0)]


@pytest.mark.parametrize("Hq,Hkv,D,Bh,R,style", CASES)
def test_rope_append_codes_and_attention(kv4, Hq, Hkv, D, Bh, R, style):
    lens = [900, 1, 250, 0, 37]
    pair, rope, rng = _build(kv4, Hq, Hkv, D, Bh, R, style, lens, Hq + R + style)
    seqs = [0, 1, 2, 3, 4]
    assert compare_int4_pages(pair, 0, seqs) == []
    assert compare_int8_store(pair, 0, seqs) == []
    q = bf16_values((5, Hq, D), rng)
    order = [2, 0, 4, 3, 1]
    ref = decode_attention(pair.orc, 0, order, f32(q), rope=rope)
    out = pair.attention(0, order, q, mode=kv4.KV4_MODE_ROPE_Q)
    out32 = pair.attention(0, order, q, mode=kv4.KV4_MODE_ROPE_Q | kv4.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)


@pytest.mark.parametrize("style", [0, 1])
def test_rope_multi_token_queries(kv4, style):
    pair, rope, rng = _build(kv4, 16, 8, 128, 128, 128, style, [700, 2, 90], 50 + style)
    q = bf16_values((3, 4, 16, 128), rng)
    ids = torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda")
    ref = extend_attention(pair.orc, 0, [0, 1, 2], f32(q), rope=rope)
    out = pair.gpu.extend_attention(0, ids, q.cuda(), mode=kv4.KV4_MODE_ROPE_Q)
    out32 = pair.gpu.extend_attention(0, ids, q.cuda(), mode=kv4.KV4_MODE_ROPE_Q | kv4.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)


def test_key_past_the_table_is_flagged(kv4):
    rng = np.random.default_rng(60)
    cfg = cfg_dict(D=64, Hq=8, Hkv=4, P=16, Bh=64, S=4, W=16, num_pages=8, mpps=8, max_seqs=1)
    pair = Pair(cfg, random_table(1, 8, 8, rng))
    pair.gpu.set_rope(torch.from_numpy(workloads.rope_cos_sin(40, 64)), 64, 0)
    k, v = bf16_values((50, 4, 64), rng), bf16_values((50, 4, 64), rng)
    pair.gpu.append(0, torch.zeros(1, dtype=torch.int32, device="cuda"),
                    torch.tensor([0, 50], dtype=torch.int32, device="cuda"), k.cuda(), v.cuda(), rope=True)
    torch.cuda.synchronize()
    assert pair.gpu.status() & kv4.KV4_DEV_ROPE_POS


def test_rope_arguments_are_checked(kv4):
    rng = np.random.default_rng(61)
    cfg = cfg_dict(D=64, Hq=8, Hkv=4, P=16, Bh=64, S=4, W=16, num_pages=8, mpps=8, max_seqs=1)
    pair = Pair(cfg, random_table(1, 8, 8, rng))
    q = bf16_values((1, 8, 64), rng)
    with pytest.raises(kv4.KV4Error):                              # no table registered
        pair.attention(0, [0], q, mode=kv4.KV4_MODE_ROPE_Q)
    cs = torch.from_numpy(workloads.rope_cos_sin(16, 64))
    for R, style in ((48, 0), (16, 0), (128, 0), (64, 2)):         # not a power of two, < 32, > D, bad style
        with pytest.raises(kv4.KV4Error):
            pair.gpu.set_rope(cs, R, style)
    pair.gpu.set_rope(cs, 64, 0)
    with pytest.raises(kv4.KV4Error):                              # RoPE of an already rotated query
        pair.attention(0, [0], q, mode=kv4.KV4_MODE_ROPE_Q | kv4.KV4_MODE_Q_ROTATED)

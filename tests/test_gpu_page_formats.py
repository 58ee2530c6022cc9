"""GPU parity of the alternative page formats (kv4_config.page_format): the CUDA
path against the oracle on identical seeded inputs.

* KV4_FORMAT_NVFP4 -- "KV Cache Quantization" topic page, item 3 (SGLang's NVFP4
  paged KV cache); the block quantizer's readings are the library's (E2M1
  codes, one E4M3 scale per 16 dims, per-tensor scale 1).
* KV4_FORMAT_INT2 -- the same page, item 2 (INT2 KV with folded scale and
  offset): the method's token-wise quantizer with 2-bit codes.

Codes and scales must match bit for bit -- for NVFP4 including each token's
nibble of the V bytes it shares with its neighbour, written by different warps
or different calls; the INT8 store of the protected positions is the INT4
cache's; attention, the multi-token query, the fused step and the debug view
within the tolerances of the INT4 format."""

import numpy as np
import pytest
import torch

from kvhelpers import (Pair, cfg_dict, random_table, bf16_values, f32, compare_page_copy, compare_int8_store,
                       check_bf16_out, check_f32_out, REL_L2, MAX_ABS)
from oracle import extend_attention

pytestmark = pytest.mark.gpu

FORMATS = [1, 2]   # KV4_FORMAT_NVFP4, KV4_FORMAT_INT2


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _populate(pair, rng, seqs, lens, Hkv, D, chunk=200, fill=True):
    """Ragged appends in pieces of random size (so the two tokens of a V byte arrive both in one call and in
    different calls), over a pool pre-filled with 0xFF (NaN scales in every unwritten slot)."""
    if fill:
        pair.gpu.pages(0).fill_(0xFF)
        pair.gpu.protected(0).fill_(0xFF)
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


def _check(kv4, pair, seqs, q, protected=True):
    mode = 0 if protected else kv4.KV4_MODE_INT4_ONLY
    ref = pair.oracle_attention(0, seqs, q, protected=protected)
    out = pair.attention(0, seqs, q, mode=mode)
    out32 = pair.attention(0, seqs, q, mode=mode | kv4.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)


CASES = [
    # D, Hq, Hkv, P, Bh, S, W, lens
    (128, 32, 8, 16, 128, 4, 128, [900, 17, 0, 450, 1, 3000]),
    (128, 16, 2, 32, 64, 4, 32, [700, 33, 129]),
    (64, 8, 1, 16, 64, 4, 32, [300, 2, 61]),
    (64, 16, 4, 64, 16, 2, 21, [1000, 250]),
    (128, 8, 8, 16, 128, 0, 16, [512, 511, 16]),
]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("D,Hq,Hkv,P,Bh,S,W,lens", CASES)
def test_codes_scales_and_attention(kv4, fmt, D, Hq, Hkv, P, Bh, S, W, lens):
    rng = np.random.default_rng(sum(lens) + D + Hkv)
    n = len(lens)
    mpps = max(lens) // P + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=P, Bh=Bh, S=S, W=W, num_pages=n * mpps, mpps=mpps, max_seqs=n, fmt=fmt)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    seqs = list(range(n))
    _populate(pair, rng, seqs, lens, Hkv, D)
    np.testing.assert_array_equal(pair.gpu.seq_lens()[0, :n].cpu().numpy(), lens)
    assert compare_page_copy(pair, 0, seqs) == []
    assert compare_int8_store(pair, 0, seqs) == []
    q = bf16_values((n, Hq, D), rng)
    order = seqs[::-1]
    _check(kv4, pair, order, q[order])
    _check(kv4, pair, order, q[order], protected=False)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("D", [64, 128])
def test_debug_view_is_the_oracle_view(kv4, fmt, D):
    rng = np.random.default_rng(11)
    Hkv, n = 4, 2
    lens = [300, 40]
    cfg = cfg_dict(D=D, Hq=16, Hkv=Hkv, P=32, Bh=D, S=4, W=32, num_pages=24, mpps=12, max_seqs=n, fmt=fmt)
    pair = Pair(cfg, random_table(n, 12, 24, rng))
    _populate(pair, rng, [0, 1], lens, Hkv, D)
    for s, L in enumerate(lens):
        for view, prot in ((kv4.KV4_VIEW_EFFECTIVE, True), (kv4.KV4_VIEW_INT4, False)):
            k, v = pair.gpu.dequantize(0, s, 0, L, view=view)
            ko, vo = pair.orc.view(0, s, protected=prot)
            np.testing.assert_array_equal(k.cpu().numpy(), ko)
            np.testing.assert_array_equal(v.cpu().numpy(), vo)


@pytest.mark.parametrize("fmt", FORMATS)
def test_decode_steps_fused_and_two_calls(kv4, fmt):
    """kv4_decode_step on these pages equals append + attention bit for bit over 12 steps (for NVFP4 the
    tokens of a shared V byte arrive in consecutive steps), and matches the oracle."""
    rng = np.random.default_rng(12)
    D, Hq, Hkv = 128, 32, 8
    lens = [500, 33, 1000, 0]
    n = len(lens)
    mpps = (max(lens) + 20) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n, fmt=fmt)
    table = random_table(n, mpps, n * mpps, rng)
    a, b = Pair(cfg, table), Pair(cfg, table)
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    for pr in (a, b):
        pr.gpu.pages(0).fill_(0xFF)
        pr.append(0, list(range(n)), lens, k, v, oracle=pr is a)
    ids = torch.tensor([2, 0, 3, 1], dtype=torch.int32, device="cuda")
    for step in range(12):
        kn, vn, q = (bf16_values((n, Hkv, D), rng, 2.0), bf16_values((n, Hkv, D), rng), bf16_values((n, Hq, D), rng))
        a.gpu.append(0, ids, torch.arange(n + 1, dtype=torch.int32, device="cuda"), kn.cuda(), vn.cuda(), total_new=n)
        out_a = a.gpu.attention(0, ids, q.cuda())
        out_b = b.gpu.decode_step(0, ids, kn.cuda(), vn.cuda(), q.cuda())
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b), step
        a.orc.append(0, [2, 0, 3, 1], np.arange(n + 1), f32(kn), f32(vn))
    assert compare_page_copy(a, 0, list(range(n))) == []
    torch.cuda.synchronize()
    assert torch.equal(a.gpu.pages(0), b.gpu.pages(0))
    rel, excess = check_bf16_out(out_b, a.oracle_attention(0, [2, 0, 3, 1], q))
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    assert a.gpu.status() == 0 and b.gpu.status() == 0


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("Hq,Hkv,T", [(32, 8, 2), (16, 8, 4), (32, 8, 5)])
def test_multi_token_queries(kv4, fmt, Hq, Hkv, T):
    rng = np.random.default_rng(13 + T)
    D = 128
    lens = [700, 3, 0, 140]
    n = len(lens)
    mpps = max(lens) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=64, num_pages=n * mpps, mpps=mpps, max_seqs=n, fmt=fmt)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, list(range(n)), lens, Hkv, D)
    q = bf16_values((n, T, Hq, D), rng)
    seqs = [3, 1, 0, 2]
    for protected in (True, False):
        mode = 0 if protected else kv4.KV4_MODE_INT4_ONLY
        ref = extend_attention(pair.orc, 0, seqs, f32(q[seqs]), protected=protected)
        ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
        out = pair.gpu.extend_attention(0, ids, q[seqs].cuda().contiguous(), mode=mode)
        out32 = pair.gpu.extend_attention(0, ids, q[seqs].cuda().contiguous(), mode=mode | kv4.KV4_MODE_OUT_F32)
        torch.cuda.synchronize()
        assert pair.gpu.status() == 0
        rel, excess = check_bf16_out(out, ref)
        assert rel <= REL_L2 and excess <= 0, (rel, excess)
        rel32, mx32 = check_f32_out(out32, ref)
        assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)


@pytest.mark.parametrize("fmt", FORMATS)
def test_one_long_sequence_over_every_cta(kv4, fmt):
    rng = np.random.default_rng(14)
    D, Hq, Hkv = 128, 32, 8
    L = 40000
    mpps = L // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=mpps, mpps=mpps, max_seqs=1, fmt=fmt)
    pair = Pair(cfg, random_table(1, mpps, mpps, rng))
    _populate(pair, rng, [0], [L], Hkv, D, chunk=4096, fill=False)
    q = bf16_values((1, Hq, D), rng)
    _check(kv4, pair, [0], q)

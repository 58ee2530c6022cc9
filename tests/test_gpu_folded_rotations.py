"""GPU parity of the folded-rotation modes: KV4_MODE_Q_ROTATED (the query
arrives as H q and is used as given) and KV4_MODE_OUT_ROTATED (the output
stays in the rotated basis), alone and together, on the page-major path
(decode and multi-token) with groups of 4, 2 and 1 KV heads, against the
oracle with the same options."""

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, REL_L2, MAX_ABS, f32
from oracle import decode_attention, extend_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _build(Hq, Hkv, D, Bh, lens, seed):
    rng = np.random.default_rng(seed)
    n = len(lens)
    mpps = max(lens) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=Bh, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0, outlier_ch=[3], outlier=8.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    pair.append(0, list(range(n)), lens, k, v)
    return pair, rng


def _modes(kv4):
    return [(kv4.KV4_MODE_Q_ROTATED, True, False), (kv4.KV4_MODE_OUT_ROTATED, False, True),
            (kv4.KV4_MODE_Q_ROTATED | kv4.KV4_MODE_OUT_ROTATED, True, True)]


def _check_out(out, out32, ref):
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)


@pytest.mark.parametrize("Hq,Hkv,D,Bh", [(32, 8, 128, 128), (16, 8, 64, 32), (8, 2, 128, 64)])
def test_decode_folded_rotations(kv4, Hq, Hkv, D, Bh):
    pair, rng = _build(Hq, Hkv, D, Bh, [700, 1, 90, 0, 260], Hq + D)
    seqs = [2, 0, 4, 3, 1]
    q = bf16_values((5, Hq, D), rng)            # any bf16 tensor is a valid rotated query
    for mode, qr, orot in _modes(kv4):
        ref = decode_attention(pair.orc, 0, seqs, f32(q), q_rotated=qr, out_rotated=orot)
        out = pair.attention(0, seqs, q, mode=mode)
        out32 = pair.attention(0, seqs, q, mode=mode | kv4.KV4_MODE_OUT_F32)
        torch.cuda.synchronize()
        assert pair.gpu.status() == 0
        _check_out(out, out32, ref)


def test_extend_folded_rotations(kv4):
    pair, rng = _build(16, 8, 128, 128, [500, 3, 77], 5)
    seqs = [0, 1, 2]
    q = bf16_values((3, 4, 16, 128), rng)
    ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    for mode, qr, orot in _modes(kv4):
        ref = extend_attention(pair.orc, 0, seqs, f32(q), q_rotated=qr, out_rotated=orot)
        out = pair.gpu.extend_attention(0, ids, q.cuda(), mode=mode)
        out32 = pair.gpu.extend_attention(0, ids, q.cuda(), mode=mode | kv4.KV4_MODE_OUT_F32)
        torch.cuda.synchronize()
        assert pair.gpu.status() == 0
        _check_out(out, out32, ref)

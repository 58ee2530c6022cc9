"""The two one-token attention kernels of 4-KV-head groups at D = 128 -- the
mma.sync kernel (the default) and the tensor-memory kernel (tcgen05
multiplies, KV4_ATTENTION_KERNEL=tc when the cache is created) -- against the
oracle on the same caches.  The inputs make the tensor-memory kernel move its running
max late (a large-norm key at the last positions and at the sink, which it
reads last) and its fixed-point scale (V magnitudes growing along the
sequence), so its accumulator is folded several times within one segment."""

import os

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, REL_L2, MAX_ABS, f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _pair(cfg, table, kernel):
    old = os.environ.get("KV4_ATTENTION_KERNEL")
    try:
        if kernel == "tc":
            os.environ["KV4_ATTENTION_KERNEL"] = "tc"
        else:
            os.environ.pop("KV4_ATTENTION_KERNEL", None)
        return Pair(cfg, table)
    finally:
        if old is None:
            os.environ.pop("KV4_ATTENTION_KERNEL", None)
        else:
            os.environ["KV4_ATTENTION_KERNEL"] = old


@pytest.mark.parametrize("lens", [[3000, 17, 0, 700, 129, 4096], [20000], [1, 2, 16, 128, 133, 300]])
def test_both_kernels_match_the_oracle(kv4, lens):
    rng = np.random.default_rng(sum(lens) % 9973)
    D, Hq, Hkv, n = 128, 32, 8, len(lens)
    mpps = max(lens) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    table = random_table(n, mpps, n * mpps, rng)
    tot = int(sum(lens))
    k = bf16_values((tot, Hkv, D), rng, 2.0, outlier_ch=[5, 70], outlier=12.0).float()
    v = bf16_values((tot, Hkv, D), rng).float()
    off = 0
    for L in lens:
        if L:
            ramp = torch.linspace(0.3, 4.0, L)[:, None, None]   # V magnitudes grow along the sequence
            v[off:off + L] *= ramp
            k[off] *= 9.0                                       # large-norm sink at position 0
            k[off + max(L - 3, 1):off + L] *= 3.0               # and large keys among the last positions
        off += L
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    pairs = {name: _pair(cfg, table, name) for name in ("tc", "mma")}
    for pr in pairs.values():
        pr.gpu.pages(0).fill_(0xFF)          # unwritten slots hold NaN scales and codes
        pr.gpu.protected(0).fill_(0xFF)
        pr.append(0, list(range(n)), list(lens), k, v)
    seqs = list(range(n))[::-1]
    q = bf16_values((n, Hq, D), rng)
    outs = {}
    for name, pr in pairs.items():
        ref = pr.oracle_attention(0, seqs, q)
        out = pr.attention(0, seqs, q)
        out32 = pr.attention(0, seqs, q, mode=kv4.KV4_MODE_OUT_F32)
        torch.cuda.synchronize()
        assert pr.gpu.status() == 0, name
        rel, excess = check_bf16_out(out, ref)
        assert rel <= REL_L2 and excess <= 0, (name, rel, excess)
        rel32, mx32 = check_f32_out(out32, ref)
        assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (name, rel32, mx32)
        outs[name] = out32
        for s, L in zip(seqs, [lens[i] for i in seqs]):
            if L == 0:
                assert torch.all(out[seqs.index(s)] == 0)
    d = (outs["tc"] - outs["mma"]).abs().max().item()
    assert d <= 2 * MAX_ABS, d


def test_step_through_both_kernels(kv4):
    """kv4_decode_step (append + attention) on the tensor-memory kernel equals the two calls, 10 steps."""
    rng = np.random.default_rng(41)
    D, Hq, Hkv = 128, 32, 8
    lens = [500, 33, 1000]
    n = len(lens)
    mpps = (max(lens) + 20) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    table = random_table(n, mpps, n * mpps, rng)
    a, b = _pair(cfg, table, "tc"), _pair(cfg, table, "tc")
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    for pr in (a, b):
        pr.append(0, list(range(n)), lens, k, v, oracle=pr is a)
    ids = torch.tensor([2, 0, 1], dtype=torch.int32, device="cuda")
    for step in range(10):
        kn, vn, q = (bf16_values((n, Hkv, D), rng, 2.0), bf16_values((n, Hkv, D), rng), bf16_values((n, Hq, D), rng))
        a.gpu.append(0, ids, torch.arange(n + 1, dtype=torch.int32, device="cuda"), kn.cuda(), vn.cuda(), total_new=n)
        out_a = a.gpu.attention(0, ids, q.cuda())
        out_b = b.gpu.decode_step(0, ids, kn.cuda(), vn.cuda(), q.cuda())
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b), step
        a.orc.append(0, [2, 0, 1], np.arange(n + 1), f32(kn), f32(vn))
    rel, excess = check_bf16_out(out_b, a.oracle_attention(0, [2, 0, 1], q))
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    assert a.gpu.status() == 0 and b.gpu.status() == 0

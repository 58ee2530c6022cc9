"""The bounded waits of the attention kernel, exercised without a device fault.

kv4_test_stall_next_attention makes the first CTA of the next attention call
leave one of its shared-memory stages unfilled: a flag that nothing sets.  Its
consumer warps then wait on that stage until the wait gives up (about a
second), set KV4_DEV_TIMEOUT and leave; the producer lets every copy it issued
land before it leaves.  The test checks that the call returns with the status
bit set, and that the next ordinary call on the same cache (the plain
attention call and the fused decode step) again matches the oracle."""

import time

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, REL_L2, f32
from oracle import decode_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _pair(rng, Hq=32, Hkv=8, D=128, lens=(3000, 40, 700)):
    n = len(lens)
    mpps = (max(lens) + 8) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=D, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0, outlier_ch=[3], outlier=8.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    pair.append(0, list(range(n)), list(lens), k, v)
    return pair


@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (4, 1, 64)])
def test_stalled_stage_times_out_then_attention_is_correct(kv4, Hq, Hkv, D):
    rng = np.random.default_rng(11 + Hkv)
    pair = _pair(rng, Hq, Hkv, D)
    seqs = [2, 0, 1]
    q = bf16_values((3, Hq, D), rng)
    assert pair.gpu.status() == 0
    pair.gpu.stall_next_attention(3)
    t0 = time.time()
    pair.attention(0, seqs, q)
    torch.cuda.synchronize()
    waited = time.time() - t0
    status = pair.gpu.status()
    assert status & kv4.KV4_DEV_TIMEOUT, status
    assert 0.5 < waited < 60, waited                   # gave up after about a second, did not hang
    # the hook applied to one call only: the next call on the same cache is correct and clean
    out = pair.attention(0, seqs, q)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, pair.oracle_attention(0, seqs, q))
    assert rel <= REL_L2 and excess <= 0, (rel, excess)


def test_stalled_decode_step_times_out_then_steps_are_correct(kv4):
    rng = np.random.default_rng(23)
    Hq, Hkv, D = 32, 8, 128
    pair = _pair(rng, Hq, Hkv, D)
    seqs = [1, 2, 0]
    ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    for step in range(2):
        k = bf16_values((3, Hkv, D), rng, 2.0)
        v = bf16_values((3, Hkv, D), rng)
        q = bf16_values((3, Hq, D), rng)
        if step == 0:
            pair.gpu.stall_next_attention(5)
        out = pair.gpu.decode_step(0, ids, k.cuda(), v.cuda(), q.cuda())
        torch.cuda.synchronize()
        pair.orc.append(0, seqs, np.arange(4), f32(k), f32(v))   # the append of a stalled step still happened
        status = pair.gpu.status()
        if step == 0:
            assert status & kv4.KV4_DEV_TIMEOUT, status
            continue
        assert status == 0
        rel, excess = check_bf16_out(out, decode_attention(pair.orc, 0, seqs, f32(q)))
        assert rel <= REL_L2 and excess <= 0, (rel, excess)

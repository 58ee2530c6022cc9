"""The integer query planes of one-token attention at their range limits.

With one query token and at most 4 query heads per KV head the kernel holds
each rotated query as q = 256 hi + lo with both bytes signed, after scaling
the KV head's queries by 2^e so that their largest magnitude lies in
[2^14, 2^15).  Two signed bytes reach 32639, so the one scaled bf16 value
above it, 32640 (an all-ones mantissa, 1.9921875 * 2^k), makes the operand
take one bit less.  The queries arrive already rotated (KV4_MODE_Q_ROTATED),
so the values below are q_rot exactly: per KV head, a largest element of
+1.9921875 (the narrower operand), -1.9921875 (the same, by magnitude),
1.984375 (32512: the full width), 1.9921875 * 2^-7, a head group of zeros
(uniform weights: the mean of the values), and plain random values.  Each is
checked against the oracle run with the same rotated queries."""

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, check_bf16_out, check_f32_out, REL_L2, MAX_ABS, f32
from oracle import decode_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (16, 8, 64), (8, 4, 128)])
def test_query_planes_at_their_limits(kv4, Hq, Hkv, D):
    rng = np.random.default_rng(97 + D + Hq)
    lens = [700, 33, 2000]
    n = len(lens)
    mpps = max(lens) // 16 + 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=D, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    k = bf16_values((sum(lens), Hkv, D), rng, 2.0, outlier_ch=[5], outlier=10.0)
    v = bf16_values((sum(lens), Hkv, D), rng)
    pair.append(0, list(range(n)), lens, k, v)

    G = Hq // Hkv
    q = np.clip(rng.standard_normal((n, Hq, D)).astype(np.float32) * 0.4, -1.5, 1.5)
    specials = [1.9921875, -1.9921875, 1.984375, 1.9921875 * 2.0 ** -7, 0.0]
    for b in range(n):
        for h in range(Hkv):
            kind = (h + b) % (len(specials) + 1)
            blk = q[b, h * G:(h + 1) * G]
            if kind == len(specials):
                continue                                    # plain random values
            s = specials[kind]
            if s == 0.0:
                blk[:] = 0.0                                 # the whole head group is zero
                continue
            if abs(s) < 1.0:
                blk *= 2.0 ** -8                             # keep the special value the largest
            blk[(b + h) % G, (7 * h + b) % D] = s
    q = torch.from_numpy(q).to(torch.bfloat16)
    assert set(np.abs(f32(q)).max(axis=2).ravel()) >= {1.9921875, 1.984375}   # the values survive bf16

    seqs = [2, 0, 1]
    mode = kv4.KV4_MODE_Q_ROTATED
    ref = decode_attention(pair.orc, 0, seqs, f32(q), q_rotated=True)
    out = pair.attention(0, seqs, q, mode=mode)
    out32 = pair.attention(0, seqs, q, mode=mode | kv4.KV4_MODE_OUT_F32)
    torch.cuda.synchronize()
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out, ref)
    assert rel <= REL_L2 and excess <= 0, (rel, excess)
    rel32, mx32 = check_f32_out(out32, ref)
    assert rel32 <= REL_L2 and mx32 <= MAX_ABS, (rel32, mx32)
    # the fused step builds the same operands: one more token through kv4_decode_step
    ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    kn, vn = bf16_values((n, Hkv, D), rng, 2.0), bf16_values((n, Hkv, D), rng)
    out_s = pair.gpu.decode_step(0, ids, kn.cuda(), vn.cuda(), q.cuda(), mode=mode)
    torch.cuda.synchronize()
    pair.orc.append(0, seqs, np.arange(n + 1), f32(kn), f32(vn))
    assert pair.gpu.status() == 0
    rel, excess = check_bf16_out(out_s, decode_attention(pair.orc, 0, seqs, f32(q), q_rotated=True))
    assert rel <= REL_L2 and excess <= 0, (rel, excess)

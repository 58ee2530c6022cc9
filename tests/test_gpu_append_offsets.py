"""Append row offsets that do not run 0 = cu[0] <= cu[1] <= ... <= cu[n] = total_new.

The append kernel checks the offsets against the host's total_new before any
row is placed: a mismatch sets KV4_DEV_BAD_CU and nothing is written -- no
page code or scale, no INT8 slot, no sequence length -- so a row can never
land past its sequence's new length in another sequence's page or in a live
recent-window slot.  Three kinds of bad offsets are tried (a last offset
below total_new, a decreasing pair, a first offset above 0); every byte of
the pages and of the INT8 store and every length must be unchanged, and a
valid append afterwards must still match the oracle."""

import numpy as np
import pytest
import torch

from kvhelpers import (Pair, cfg_dict, random_table, bf16_values, compare_int4_pages, check_bf16_out, REL_L2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def test_bad_row_offsets_write_nothing(kv4):
    rng = np.random.default_rng(404)
    D, Hq, Hkv = 64, 8, 2
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=64, S=4, W=16, num_pages=12, mpps=4, max_seqs=3)
    pair = Pair(cfg, random_table(3, 4, 12, rng))
    lens = [20, 33, 7]
    pair.append(0, [0, 1, 2], lens, bf16_values((sum(lens), Hkv, D), rng, 2.0), bf16_values((sum(lens), Hkv, D), rng))
    assert pair.gpu.status() == 0
    pages0 = pair.gpu.pages(0).clone()
    prot0 = pair.gpu.protected(0).clone()
    lens0 = pair.gpu.seq_lens().clone()

    k = bf16_values((8, Hkv, D), rng).cuda()
    v = bf16_values((8, Hkv, D), rng).cuda()
    for seqs, cu in (([0, 1], [0, 3, 5]),          # cu[n] = 5, total_new = 8
                     ([0, 1, 2], [0, 5, 3, 8]),    # decreasing
                     ([0, 1], [1, 4, 8])):         # cu[0] = 1
        pair.gpu.append(0, torch.tensor(seqs, dtype=torch.int32, device="cuda"),
                        torch.tensor(cu, dtype=torch.int32, device="cuda"), k, v, total_new=8)
        status = pair.gpu.status()
        assert status & kv4.KV4_DEV_BAD_CU, (cu, status)
        assert pair.gpu.status() == 0                  # reading cleared it
        torch.cuda.synchronize()
        assert torch.equal(pair.gpu.seq_lens(), lens0), cu
        assert torch.equal(pair.gpu.pages(0), pages0), cu
        assert torch.equal(pair.gpu.protected(0), prot0), cu

    # the cache is still usable: a valid append, then codes and attention against the oracle
    pair.append(0, [1, 0], [5, 2], bf16_values((7, Hkv, D), rng, 2.0), bf16_values((7, Hkv, D), rng))
    assert pair.gpu.status() == 0
    assert compare_int4_pages(pair, 0, [0, 1, 2]) == []
    q = bf16_values((3, Hq, D), rng)
    out = pair.attention(0, [0, 1, 2], q)
    torch.cuda.synchronize()
    rel, excess = check_bf16_out(out, pair.oracle_attention(0, [0, 1, 2], q))
    assert rel <= REL_L2 and excess <= 0, (rel, excess)

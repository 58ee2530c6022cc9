"""kv4_decode_attention_noalloc (static device scratch instead of a workspace)
against kv4_decode_attention on the same cache, two calls in a row.

The file name sorts last so that it also runs after every other GPU test (the
scratch array is shared by all caches of the process on a device)."""

import numpy as np
import pytest
import torch

from kvhelpers import Pair, cfg_dict, random_table, bf16_values, bf16_ulp, REL_L2, MAX_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


def _populate(pair, rng, lens, Hkv, D):
    n = int(sum(lens))
    pair.append(0, list(range(len(lens))), list(lens), bf16_values((n, Hkv, D), rng, 2.0),
                bf16_values((n, Hkv, D), rng), oracle=False)


def test_noalloc_equals_workspace_call_grouped_path(kv4):
    """8 KV heads (page-major kernel, deterministic split): same bits as the workspace call."""
    rng = np.random.default_rng(31)
    D, Hq, Hkv, n, mpps = 128, 32, 8, 6, 40
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, [600, 17, 0, 333, 129, 640], Hkv, D)
    ids = torch.tensor([5, 0, 2, 3, 1, 4], dtype=torch.int32, device="cuda")
    for _ in range(2):
        q = bf16_values((n, Hq, D), rng).cuda()
        ref = pair.gpu.attention(0, ids, q)
        got = pair.gpu.attention_noalloc(0, ids, q, torch.empty_like(ref))
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        assert torch.all(got[2] == 0)
    assert pair.gpu.status() == 0


def test_noalloc_equals_workspace_call_two_head_groups(kv4):
    """2 KV heads (the page-major kernel in groups of 2 heads): equal to the workspace call within the
    attention tolerance, in bf16 and fp32 output."""
    rng = np.random.default_rng(32)
    D, Hq, Hkv, n, mpps = 64, 8, 2, 3, 20
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=64, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n)
    pair = Pair(cfg, random_table(n, mpps, n * mpps, rng))
    _populate(pair, rng, [300, 45, 1], Hkv, D)
    ids = torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda")
    for mode in (0, kv4.KV4_MODE_OUT_F32):
        q = bf16_values((n, Hq, D), rng).cuda()
        ref = pair.gpu.attention(0, ids, q, mode=mode)
        for _ in range(2):
            got = pair.gpu.attention_noalloc(0, ids, q, torch.empty_like(ref), mode=mode)
            torch.cuda.synchronize()
            g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
            rel = np.linalg.norm(g - r) / np.linalg.norm(r)
            allowed = MAX_ABS if mode else np.maximum(MAX_ABS, bf16_ulp(r))   # bf16: one ulp of rounding
            assert rel <= REL_L2 and np.all(np.abs(g - r) <= allowed)
    assert pair.gpu.status() == 0


def test_noalloc_rejects_what_does_not_fit(kv4):
    """A batch whose scratch exceeds the static array is refused before any launch."""
    D, Hq, Hkv, n = 128, 32, 8, 1024
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=16, Bh=128, S=4, W=128, num_pages=n, mpps=1, max_seqs=n)
    import int4_kv_cache_paged_b200 as m
    cache = m.KV4Cache(cfg, torch.full((n, 1), -1, dtype=torch.int32), "cuda")
    need = cache._ws_bytes(cache.handle, n, 0)
    assert need > m.KV4_NOALLOC_SCRATCH_BYTES
    ids = torch.arange(n, dtype=torch.int32, device="cuda")
    q = torch.zeros((n, Hq, D), dtype=torch.bfloat16, device="cuda")
    out = torch.full((n, Hq, D), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.KV4Error) as e:
        cache.attention_noalloc(0, ids, q, out)
    assert e.value.code == m.KV4_ERR_SCRATCH
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)          # nothing ran
    small = ids[:64]
    assert cache._ws_bytes(cache.handle, 64, 0) <= m.KV4_NOALLOC_SCRATCH_BYTES
    cache.attention_noalloc(0, small, q[:64], out[:64])   # all sequences empty: zero rows
    torch.cuda.synchronize()
    assert torch.all(out[:64] == 0) and torch.all(out[64:] == 7.0)

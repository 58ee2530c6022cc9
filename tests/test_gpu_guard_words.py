"""Guard words around every buffer the kernels write.

The cache buffer, the attention workspace and the outputs are carved from
larger device allocations whose margins hold a fixed pattern.  The test runs
the library's writers on them -- bulk appends of ragged sequences (an empty one
and one filled exactly to its capacity), decode attention (bf16 and fp32
output), fused decode steps up to and past the capacity (the step past it
must be refused with KV4_DEV_OVERFLOW) and multi-token queries -- on every page
format and on groups of 4 and of 1 KV heads, then checks that no margin byte
changed: a write outside a buffer would show there."""

import numpy as np
import pytest
import torch

from kvhelpers import cfg_dict, random_table, bf16_values

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of margin on each side (a multiple of 256, so the carved buffers stay aligned)
PATTERN = 0xA5


@pytest.fixture(scope="module")
def kv4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int4_kv_cache_paged_b200 as m
    return m


class Guarded:
    """A device byte buffer with PATTERN margins; .inner is the usable part."""

    def __init__(self, nbytes):
        self.n = int(nbytes)
        self.full = torch.full((self.n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.inner = self.full[GUARD:GUARD + self.n]

    def view(self, dtype, shape):
        return self.inner.view(dtype).view(*shape)

    def intact(self):
        torch.cuda.synchronize()
        head, tail = self.full[:GUARD], self.full[GUARD + self.n:]
        return bool(torch.all(head == PATTERN)) and bool(torch.all(tail == PATTERN))


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (4, 1, 64)])
def test_writes_stay_inside_their_buffers(kv4, fmt, Hq, Hkv, D):
    rng = np.random.default_rng(3 + fmt + Hkv)
    P, mpps = 16, 12                                   # capacity 192 tokens per sequence
    cap = P * mpps
    lens = [150, 0, cap - 3, 17]                        # the third reaches exactly the capacity after 3 steps
    n = len(lens)
    cfg = cfg_dict(D=D, Hq=Hq, Hkv=Hkv, P=P, Bh=D, S=4, W=32, num_pages=n * mpps, mpps=mpps, max_seqs=n, fmt=fmt)
    c = kv4.make_config(**cfg)
    cache_buf = Guarded(kv4.kv4_cache_required_bytes(c))
    table = torch.from_numpy(random_table(n, mpps, n * mpps, rng)).cuda()
    h = kv4.kv4_cache_create(c, cache_buf.inner, table)
    try:
        ids = torch.arange(n, dtype=torch.int32, device="cuda")
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
        tot = int(sum(lens))
        k = bf16_values((tot, Hkv, D), rng, 2.0).cuda()
        v = bf16_values((tot, Hkv, D), rng).cuda()
        kv4.kv4_rotate_quantize_append(h, 0, ids, cu, n, tot, k, v)

        ws = Guarded(max(kv4.kv4_attention_workspace_bytes(h, n, 0), kv4.kv4_extend_workspace_bytes(h, n, 3)))
        out_b = Guarded(n * Hq * D * 2)
        out_f = Guarded(n * Hq * D * 4)
        q = bf16_values((n, Hq, D), rng).cuda()
        kv4.kv4_decode_attention(h, 0, ids, n, q, out_b.view(torch.bfloat16, (n, Hq, D)), 0.0, 0, ws.inner)
        kv4.kv4_decode_attention(h, 0, ids, n, q, out_f.view(torch.float32, (n, Hq, D)), 0.0,
                                 kv4.KV4_MODE_OUT_F32, ws.inner)
        assert kv4.kv4_get_status(h) == 0

        # fused steps: three fill the third sequence to its capacity, the fourth must be refused for it
        for step in range(4):
            kn = bf16_values((n, Hkv, D), rng, 2.0).cuda()
            vn = bf16_values((n, Hkv, D), rng).cuda()
            qn = bf16_values((n, Hq, D), rng).cuda()
            kv4.kv4_decode_step(h, 0, ids, n, kn, vn, qn, out_b.view(torch.bfloat16, (n, Hq, D)), 0.0, 0, ws.inner)
            status = kv4.kv4_get_status(h)
            assert status == (kv4.KV4_DEV_OVERFLOW if step == 3 else 0), (step, status)

        # multi-token queries over the same cache (three tokens per sequence)
        out_e = Guarded(n * 3 * Hq * D * 2)
        qe = bf16_values((n, 3, Hq, D), rng).cuda()
        kv4.kv4_extend_attention(h, 0, ids, n, 3, qe, out_e.view(torch.bfloat16, (n, 3, Hq, D)), 0.0, 0, ws.inner)
        assert kv4.kv4_get_status(h) == 0
        assert torch.isfinite(out_e.view(torch.bfloat16, (n, 3, Hq, D)).float()).all()

        for name, g in (("cache", cache_buf), ("workspace", ws), ("bf16 output", out_b), ("fp32 output", out_f),
                        ("multi-token output", out_e)):
            assert g.intact(), name
    finally:
        kv4.kv4_cache_destroy(h)

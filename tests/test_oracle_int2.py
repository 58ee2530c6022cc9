"""Pins of the INT2 page format in the oracle (the folded-scale 2-bit variant of the
"KV Cache Quantization" topic page, item 2, with the method's token-wise groups):
the tile layout (bijection, byte ownership, the operand order the kernels read)
and the cache's page copy.  The 2-bit quantizer itself is pinned with the 4- and
8-bit ones in test_oracle_quant.py (worked example, error bound, definition)."""

import numpy as np
import pytest

from oracle import layout as L
from oracle.layout import TILE
from oracle.hadamard import fwht_fp32
from oracle.quant import bf16_round, quantize_groups, dequantize_groups
from oracle import OracleKV4Cache


@pytest.mark.parametrize("D", [64, 128])
def test_int2_bijection_and_ownership(D):
    for fn in (L.int2_k_crumb, L.int2_v_crumb):
        seen = {}
        for r in range(TILE):
            for d in range(D):
                pos = fn(D, r, d)
                assert 0 <= pos[0] < 4 * D and pos[1] in (0, 1, 2, 3)
                assert pos not in seen
                seen[pos] = r
        assert len(seen) == 16 * D
        for byte in range(4 * D):           # the four crumbs of a byte belong to one token
            assert len({seen[(byte, c)] for c in range(4)}) == 1
    assert L.int2_tile_bytes(D) == 8 * D + 128


@pytest.mark.parametrize("D", [64, 128])
def test_int2_operand_order(D):
    """K: lane 4g + t reads token g's word (t, kq); (word >> 2c) & 0x03030303 holds dims 4t..4t+3 of 16-dim
    block 4kq + c, byte j = dim 4t + j (the integer multiply's A registers, as in the INT4 layout).
    V: the word of lane 4g + t and dim-block pair mp holds, for m = 2mp + mb, the codes of (dim g | g + 8) x
    (tokens 2t, 2t+1 | 2t+8, 2t+9) with tokens 2t and 2t+1 at bits b and b + 16."""
    for lane in range(32):
        g, t = divmod(lane, 4)
        for tok in (g, g + 8):
            for kq in range(D // 64):
                w = tok * (D // 4) + t * (D // 16) + 4 * kq
                for c in range(4):
                    for j in range(4):
                        assert L.int2_k_crumb(D, tok, 64 * kq + 16 * c + 4 * t + j) == (w + j, c)
        for m in range(D // 16):
            mp, mb = divmod(m, 2)
            w = (D // 8) * lane + 4 * mp
            for (dim, th, base) in ((g, 0, 4 * mb), (g + 8, 0, 4 * mb + 2), (g, 1, 4 * mb + 8), (g + 8, 1, 4 * mb + 10)):
                for e in (0, 1):
                    bit = base + 16 * e
                    assert L.int2_v_crumb(D, 8 * th + 2 * t + e, 16 * m + dim) == (w + bit // 8, (bit % 8) // 2)


def _cfg(fmt, D):
    return dict(num_layers=1, max_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=D, page_size=32,
                num_pages=12, max_pages_per_seq=4, hadamard_block=D, sink_tokens=4, recent_window=16,
                page_format=fmt)


@pytest.mark.parametrize("D", [64, 128])
def test_cache_pages_hold_the_two_bit_rotation(D):
    """Ragged appends: the page view is the 2-bit round trip of the rotated inputs, the protected view is
    the INT8 path of the INT4 cache."""
    rng = np.random.default_rng(8)
    bt = rng.permutation(12).reshape(3, 4)
    a, b = OracleKV4Cache(_cfg(2, D), bt), OracleKV4Cache(_cfg(0, D), bt)
    rows = {s: ([], []) for s in range(3)}
    for step in range(6):
        n = rng.integers(0, 9, 3)
        tot = int(n.sum())
        k = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32) * 2)
        v = bf16_round(rng.standard_normal((tot, 2, D)).astype(np.float32))
        cu = np.concatenate([[0], np.cumsum(n)])
        for c in (a, b):
            c.append(0, [0, 1, 2], cu, k, v)
        for s in range(3):
            rows[s][0].append(k[cu[s]:cu[s + 1]])
            rows[s][1].append(v[cu[s]:cu[s + 1]])
    np.testing.assert_array_equal(a.seq_lens, b.seq_lens)
    for s in range(3):
        L_ = int(a.seq_lens[0, s])
        if L_ == 0:
            continue
        kr, vr = fwht_fp32(np.concatenate(rows[s][0]), D), fwht_fp32(np.concatenate(rows[s][1]), D)
        kp, vp = a.view(0, s, protected=False)
        np.testing.assert_array_equal(kp, dequantize_groups(*quantize_groups(kr, 2)))
        np.testing.assert_array_equal(vp, dequantize_groups(*quantize_groups(vr, 2)))
        ke, ve = a.view(0, s)
        kb, vb = b.view(0, s)
        prot = np.array([p < 4 or p >= L_ - 16 for p in range(L_)])
        np.testing.assert_array_equal(ke[prot], kb[prot])
        np.testing.assert_array_equal(ve[prot], vb[prot])

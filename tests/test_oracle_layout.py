"""Pins of the tile layout: bijections, byte ownership, and the tensor-core operand order it serves.

Scores use the 16x8x32 integer multiply (row-major A, 16 x 32 bytes): lane = 4*g + t
holds A[g][4t..4t+3] (register 0), A[g+8][4t..4t+3] (1), A[g][16+4t..16+4t+3] (2),
A[g+8][16+4t..16+4t+3] (3); the A matrix of k-block kk is K[token][32kk + col].
P.V uses the 16x8x16 fp16 multiply (row-major A, 16 x 16): lane holds
A[g][2t, 2t+1] (a0a1), A[g+8][2t, 2t+1] (a2a3), A[g][2t+8, 2t+9] (a4a5),
A[g+8][2t+8, 2t+9] (a6a7), with A = V^T[16m + row][token].
"""

import numpy as np
import pytest

from oracle import layout as L
from oracle.layout import TILE


@pytest.mark.parametrize("D", [64, 128])
def test_int4_bijection_and_ownership(D):
    for fn in (L.int4_k_nibble, L.int4_v_nibble):
        seen = {}
        for r in range(TILE):
            for d in range(D):
                pos = fn(D, r, d)
                assert 0 <= pos[0] < 8 * D and pos[1] in (0, 1)
                assert pos not in seen
                seen[pos] = r
        assert len(seen) == 16 * D
        for byte in range(8 * D):           # both nibbles of a byte belong to one token
            assert seen[(byte, 0)] == seen[(byte, 1)]
    t = L.tables("int4", D)
    for r in range(TILE):                   # a token's K codes are its natural row
        np.testing.assert_array_equal(np.sort(t.k_byte[r]), np.arange(r * D // 2, (r + 1) * D // 2))


@pytest.mark.parametrize("D", [64, 128])
def test_int8_and_bf16_bijection(D):
    for fn, n in ((L.int8_k_byte, 16 * D), (L.int8_v_byte, 16 * D), (L.bf16_k_elem, 16 * D), (L.bf16_v_elem, 16 * D)):
        pos = {fn(D, r, d) for r in range(TILE) for d in range(D)}
        assert pos == set(range(n))


def test_scale_offsets():
    offs = [L.scale_offset(r, T) for r in range(TILE) for T in (0, 1)]
    assert sorted(offs) == list(range(0, 128, 4))
    # lane group g reads one 16-byte run: K(g), K(g+8), V(g), V(g+8)
    for g in range(8):
        assert [L.scale_offset(g, 0), L.scale_offset(g + 8, 0), L.scale_offset(g, 1), L.scale_offset(g + 8, 1)] == \
            [16 * g, 16 * g + 4, 16 * g + 8, 16 * g + 12]


def _pack_int4(D, codes, fn):
    blk = np.zeros(8 * D, np.uint8)
    for r in range(TILE):
        for d in range(D):
            b, h = fn(D, r, d)
            blk[b] |= np.uint8(codes[r, d] << (4 * h))
    return blk


def _word(blk, off):
    return int(blk[off]) | int(blk[off + 1]) << 8 | int(blk[off + 2]) << 16 | int(blk[off + 3]) << 24


def _nib_pairs(w):
    """The four (low half, high half) code pairs the kernel extracts from one 32-bit word."""
    return [((w >> (4 * j)) & 15, (w >> (16 + 4 * j)) & 15) for j in range(4)]


def _byte_pairs(w):
    return [(w & 255, (w >> 16) & 255), ((w >> 8) & 255, (w >> 24) & 255)]


def _nib_bytes(w, hf):
    """The four byte-wide codes the kernel extracts from one word: (w >> 4*hf) & 0x0F0F0F0F."""
    return [(w >> (8 * j + 4 * hf)) & 15 for j in range(4)]


@pytest.mark.parametrize("D", [64, 128])
def test_int4_k_words_are_qk_a_operands(D):
    rng = np.random.default_rng(0)
    K = rng.integers(0, 16, (TILE, D))
    blk = _pack_int4(D, K, L.int4_k_nibble)
    for lane in range(32):
        g, t = divmod(lane, 4)
        for rowhi in (0, 1):
            row = g + 8 * rowhi
            for kk in range(D // 32):
                w = _word(blk, rowhi * 4 * D + lane * (D // 8) + 4 * kk)
                A = K[:, 32 * kk:32 * kk + 32]
                assert _nib_bytes(w, 0) == list(A[row, 4 * t:4 * t + 4])           # register 0 / 1
                assert _nib_bytes(w, 1) == list(A[row, 16 + 4 * t:16 + 4 * t + 4])  # register 2 / 3


@pytest.mark.parametrize("D", [64, 128])
def test_int4_v_words_are_pv_a_operands(D):
    rng = np.random.default_rng(1)
    V = rng.integers(0, 16, (TILE, D))
    blk = _pack_int4(D, V, L.int4_v_nibble)
    for lane in range(32):
        g, t = divmod(lane, 4)
        for m in range(D // 16):
            u = _nib_pairs(_word(blk, 512 * (m // 4) + 16 * lane + 4 * (m % 4)))
            AT = V[:, 16 * m:16 * m + 16].T          # rows = dims, cols = tokens
            assert u[0] == (AT[g, 2 * t], AT[g, 2 * t + 1])
            assert u[1] == (AT[g + 8, 2 * t], AT[g + 8, 2 * t + 1])
            assert u[2] == (AT[g, 2 * t + 8], AT[g, 2 * t + 9])
            assert u[3] == (AT[g + 8, 2 * t + 8], AT[g + 8, 2 * t + 9])


@pytest.mark.parametrize("D", [64, 128])
def test_int8_words_are_a_operands(D):
    rng = np.random.default_rng(2)
    K = rng.integers(0, 256, (TILE, D))
    V = rng.integers(0, 256, (TILE, D))
    kb = np.zeros(16 * D, np.uint8)
    vb = np.zeros(16 * D, np.uint8)
    for r in range(TILE):
        for d in range(D):
            kb[L.int8_k_byte(D, r, d)] = K[r, d]
            vb[L.int8_v_byte(D, r, d)] = V[r, d]
    for lane in range(32):
        g, t = divmod(lane, 4)
        for rowhi in (0, 1):
            row = g + 8 * rowhi
            for kk in range(D // 32):
                A = K[:, 32 * kk:32 * kk + 32]
                for hf in (0, 1):
                    w = _word(kb, rowhi * 8 * D + (D // 4) * lane + 4 * (2 * kk + hf))
                    assert [(w >> (8 * j)) & 255 for j in range(4)] == list(A[row, 16 * hf + 4 * t:16 * hf + 4 * t + 4])
        for m in range(D // 16):
            AT = V[:, 16 * m:16 * m + 16].T
            for th in (0, 1):
                w = 2 * m + th
                u = _byte_pairs(_word(vb, 16 * (32 * (w // 4) + lane) + 4 * (w % 4)))
                c = 2 * t + 8 * th
                assert u[0] == (AT[g, c], AT[g, c + 1])
                assert u[1] == (AT[g + 8, c], AT[g + 8, c + 1])


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_elements_are_a_operands(D):
    rng = np.random.default_rng(3)
    K = rng.integers(0, 60000, (TILE, D))
    V = rng.integers(0, 60000, (TILE, D))
    kb = np.zeros(16 * D, np.int64)
    vb = np.zeros(16 * D, np.int64)
    for r in range(TILE):
        for d in range(D):
            kb[L.bf16_k_elem(D, r, d)] = K[r, d]
            vb[L.bf16_v_elem(D, r, d)] = V[r, d]
    for lane in range(32):
        g, t = divmod(lane, 4)
        for k in range(D // 16):
            regs = kb[8 * (32 * k + lane): 8 * (32 * k + lane) + 8].reshape(4, 2)
            A = K[:, 16 * k:16 * k + 16]
            want = [(A[g, 2 * t], A[g, 2 * t + 1]), (A[g + 8, 2 * t], A[g + 8, 2 * t + 1]),
                    (A[g, 2 * t + 8], A[g, 2 * t + 9]), (A[g + 8, 2 * t + 8], A[g + 8, 2 * t + 9])]
            assert [tuple(x) for x in regs] == want
            regs = vb[8 * (32 * k + lane): 8 * (32 * k + lane) + 8].reshape(4, 2)
            AT = V[:, 16 * k:16 * k + 16].T
            want = [(AT[g, 2 * t], AT[g, 2 * t + 1]), (AT[g + 8, 2 * t], AT[g + 8, 2 * t + 1]),
                    (AT[g, 2 * t + 8], AT[g, 2 * t + 9]), (AT[g + 8, 2 * t + 8], AT[g + 8, 2 * t + 9])]
            assert [tuple(x) for x in regs] == want

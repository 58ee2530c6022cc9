"""Byte placement of codes and scales inside a 16-token tile (oracle; test infrastructure only).

The pages ask for a quantized cache that keeps "paged memory layouts, regular
memory access, and fused attention execution" ("SAW-INT4: System-Aware 4-Bit
KV-Cache Quantization for Real-World LLM Serving", Abstract) but print no
layout.  This module DEFINES the one this library uses; the CUDA path must
place every byte where these functions say.

Unit of storage: a tile of 16 consecutive token slots of one KV head.

INT4 tile (16*D + 128 bytes):   [K codes 8*D][V codes 8*D][scales 128]
INT8 tile (32*D + 128 bytes):   [K codes 16*D][V codes 16*D][scales 128]
NVFP4 tile (18*D bytes):        [K codes 8*D][V codes 8*D][K scales D][V scales D]
INT2 tile (8*D + 128 bytes):    [K codes 4*D][V codes 4*D][scales 128]
BF16 tile (64*D bytes):         [K 16*D bf16][V 16*D bf16]      (baseline cache)

Inside the code blocks the order of nibbles/bytes follows the operand order
of the tensor-core multiplies the decode kernel feeds from them (K: the
16x8x32 integer multiply, V: the 16x8x16 fp16 multiply); the functions below
state each placement in closed form.  Properties that the
tests check: every (token, dim) owns exactly one nibble (or byte, or bf16
element), and every byte of a code block belongs to exactly one token (so a
token can be written without reading its neighbours).

Scales: a 128-byte block of 32 half2 (s, z) entries.  Entry for token r of
tensor T (K = 0, V = 1) sits at byte 16*(r % 8) + 4*(2*T + r // 8); the half
at +0 is the scale s, the half at +2 the zero point z.

The NVFP4 tile (the alternative page format, see nvfp4.py) feeds 16x8x16 fp16
multiplies for both products.  Its K bytes belong to one token each; each V
byte holds one dim of two neighbouring tokens (2i, 2i + 1), the pair that one
fp16x2 operand register of the P.V multiply takes, so a token's V codes are
written nibble by nibble.  One E4M3 scale byte per (token, 16-dim block).
"""

import numpy as np

TILE = 16


def int4_tile_bytes(D):
    return 16 * D + 128


def int8_tile_bytes(D):
    return 32 * D + 128


def bf16_tile_bytes(D):
    return 64 * D


def fp4_tile_bytes(D):
    return 18 * D


def int2_tile_bytes(D):
    return 8 * D + 128


def int4_k_nibble(D, r, d):
    """(byte offset inside the K code block, nibble: 0 = low, 1 = high) of token r, dim d.

    Token r owns the D/2 bytes [r*D/2, (r+1)*D/2).  With d = 32*kk + 16*hf + 4*t + j
    (kk < D/32, hf < 2, t < 4, j < 4), the code is nibble hf of byte j of the
    32-bit word at byte r*D/2 + t*D/8 + 4*kk: masking the word with 0x0F0F0F0F
    gives the four dims 4t..4t+3 of the 32-dim block as bytes, shifting it right
    by 4 first gives dims 16+4t..16+4t+3.
    """
    kk, dd = divmod(d, 32)
    hf, rem = divmod(dd, 16)
    t, j = divmod(rem, 4)
    return r * (D // 2) + t * (D // 8) + 4 * kk + j, hf


def int4_v_nibble(D, r, d):
    """(byte offset inside the V code block, nibble) of token r, dim d.

    With d = 16*m + 8*dh + g (g < 8, dh < 2) and r = 8*th + 2*t + e
    (t < 4, e < 2, th < 2), the nibble is number i = dh + 2*th + 4*e of the
    32-bit word at byte 512*(m // 4) + 16*(4*g + t) + 4*(m % 4).
    """
    m, rr = divmod(d, 16)
    dh, g = divmod(rr, 8)
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    i = dh + 2 * th + 4 * e
    return 512 * (m // 4) + 16 * (4 * g + t) + 4 * (m % 4) + i // 2, i % 2


def int8_k_byte(D, r, d):
    """Byte offset inside the INT8 K code block of token r, dim d.

    Token r owns the D bytes [r*D, (r+1)*D).  With d = 32*kk + 16*hf + 4*t + j,
    the code is byte j of the word at r*D + (D/4)*t + 4*(2*kk + hf): one word
    holds the dims 4t..4t+3 (hf = 0) or 16+4t..16+4t+3 (hf = 1) of a 32-dim block.
    """
    kk, dd = divmod(d, 32)
    hf, rem = divmod(dd, 16)
    t, j = divmod(rem, 4)
    return r * D + (D // 4) * t + 4 * (2 * kk + hf) + j


def int8_v_byte(D, r, d):
    """Byte offset inside the INT8 V code block of token r, dim d.

    With d = 16*m + 8*dh + g and r = 8*th + 2*t + e: word w = 2*m + th, byte
    dh + 2*e of the word at 16*(32*(w//4) + 4*g + t) + 4*(w % 4).
    """
    m, rr = divmod(d, 16)
    dh, g = divmod(rr, 8)
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    w = 2 * m + th
    return 16 * (32 * (w // 4) + 4 * g + t) + 4 * (w % 4) + dh + 2 * e


def bf16_k_elem(D, r, d):
    """Element index (bf16 units) inside the BF16 K block of token r, dim d."""
    rowhi, g = divmod(r, 8)
    k, c = divmod(d, 16)
    h8, c2 = divmod(c, 8)
    t, e = divmod(c2, 2)
    reg = rowhi + 2 * h8
    return 8 * (32 * k + 4 * g + t) + 2 * reg + e


def bf16_v_elem(D, r, d):
    """Element index (bf16 units) inside the BF16 V block of token r, dim d."""
    m, rr = divmod(d, 16)
    dh, g = divmod(rr, 8)
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    reg = dh + 2 * th
    return 8 * (32 * m + 4 * g + t) + 2 * reg + e


def int2_k_crumb(D, r, d):
    """(byte offset inside the INT2 K code block, crumb 0..3 = bits 2c, 2c+1) of token r, dim d.

    Token r owns the D/4 bytes [r*D/4, (r+1)*D/4).  With d = 64*kq + 16*c + 4*t + j
    (kq < D/64, c < 4, t < 4, j < 4), the code is crumb c of byte j of the 32-bit
    word at r*D/4 + t*D/16 + 4*kq: shifting the word right by 2c and masking it
    with 0x03030303 gives the four dims 4t..4t+3 of 16-dim block 4kq + c as bytes
    (the INT4 layout's integer-multiply operand order, two bits a code).
    """
    kq, rem = divmod(d, 64)
    c, rem = divmod(rem, 16)
    t, j = divmod(rem, 4)
    return r * (D // 4) + t * (D // 16) + 4 * kq + j, c


def int2_v_crumb(D, r, d):
    """(byte offset inside the INT2 V code block, crumb) of token r, dim d.

    With d = 16*m + 8*dh + g (m = 2*mp + mb) and r = 8*th + 2*t + e, the code is
    crumb i % 4 of byte i // 4 of the word at (D/8)*(4*g + t) + 4*mp, where
    i = dh + 2*mb + 4*th + 8*e: a byte holds four dims of one token, and the
    codes of tokens 2t and 2t+1 (e = 0, 1) sit 16 bits apart, the two halves of
    one fp16x2 operand register.
    """
    m, rr = divmod(d, 16)
    mp, mb = divmod(m, 2)
    dh, g = divmod(rr, 8)
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    i = dh + 2 * mb + 4 * th + 8 * e
    return (D // 8) * (4 * g + t) + 4 * mp + i // 4, i % 4


def fp4_k_nibble(D, r, d):
    """(byte offset inside the NVFP4 K code block, nibble) of token r, dim d.

    With r = 8*rh + g (g < 8) and d = 16*b + 4*t + 2*j + e (b < D/16, t < 4,
    j < 2, e < 2), the code is nibble e of byte rh + 2*j of the 32-bit word at
    16*(4*g + t) + 4*(b % 4) + 512*(b // 4): lane 4g + t of a warp reads, per
    16-dim block b, one word whose four bytes are the E2M1 pairs of its four
    16x8x16 A-operand registers (tokens g, g + 8; dims 4t, 4t+1 and 4t+2, 4t+3).
    """
    rh, g = divmod(r, 8)
    b, rem = divmod(d, 16)
    t, rem = divmod(rem, 4)
    j, e = divmod(rem, 2)
    return 16 * (4 * g + t) + 4 * (b % 4) + 512 * (b // 4) + rh + 2 * j, e


def fp4_v_nibble(D, r, d):
    """(byte offset inside the NVFP4 V code block, nibble) of token r, dim d.

    With d = 16*m + 8*dh + g and r = 8*th + 2*t + e, the code is nibble e of
    byte dh + 2*th of the word at 16*(4*g + t) + 4*(m % 4) + 512*(m // 4): the
    word of lane 4g + t and dim block m holds the four A-operand pairs (dims g,
    g + 8; tokens 2t, 2t+1 and 2t+8, 2t+9) of the transposed P.V multiply.
    """
    m, rr = divmod(d, 16)
    dh, g = divmod(rr, 8)
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    return 16 * (4 * g + t) + 4 * (m % 4) + 512 * (m // 4) + dh + 2 * th, e


def fp4_k_scale_byte(D, r, b):
    """Byte offset inside the tile of the E4M3 scale of token r, K block b: 16*D + (D/8)*g + 2*b + rh."""
    rh, g = divmod(r, 8)
    return 16 * D + (D // 8) * g + 2 * b + rh


def fp4_v_scale_byte(D, r, m):
    """Byte offset inside the tile of the E4M3 scale of token r, V block m: 17*D + (D/4)*t + 4*m + 2*th + e."""
    th, tt = divmod(r, 8)
    t, e = divmod(tt, 2)
    return 17 * D + (D // 4) * t + 4 * m + 2 * th + e


def scale_offset(r, tensor):
    """Byte offset of the half2 (s, z) of token r inside the 128-byte scale block; tensor 0 = K, 1 = V."""
    return 16 * (r % 8) + 4 * (2 * tensor + r // 8)


# ---------------------------------------------------------------------------
# Tables used by the oracle cache.  For a token slot r they list, per byte of
# the code block that the token owns, which dims go into the byte.

class Int4Tables:
    """For token slot r: byte offsets (D/2,) and the dims in the low / high nibble."""

    def __init__(self, D):
        self.D = D
        self.k_byte = np.zeros((TILE, D // 2), np.int64)
        self.k_lo = np.zeros((TILE, D // 2), np.int64)
        self.k_hi = np.zeros((TILE, D // 2), np.int64)
        self.v_byte = np.zeros((TILE, D // 2), np.int64)
        self.v_lo = np.zeros((TILE, D // 2), np.int64)
        self.v_hi = np.zeros((TILE, D // 2), np.int64)
        for which, fn, tb, tlo, thi in (("k", int4_k_nibble, self.k_byte, self.k_lo, self.k_hi),
                                        ("v", int4_v_nibble, self.v_byte, self.v_lo, self.v_hi)):
            for r in range(TILE):
                owned = {}
                for d in range(D):
                    byte, half = fn(D, r, d)
                    owned.setdefault(byte, [None, None])[half] = d
                if len(owned) != D // 2 or any(None in v for v in owned.values()):
                    raise AssertionError("INT4 %s layout: token %d does not own whole bytes" % (which, r))
                for n, byte in enumerate(sorted(owned)):
                    tb[r, n] = byte
                    tlo[r, n], thi[r, n] = owned[byte]


class Int8Tables:
    """For token slot r: byte offset of each dim (D,) in the K and V code blocks."""

    def __init__(self, D):
        self.D = D
        self.k_byte = np.array([[int8_k_byte(D, r, d) for d in range(D)] for r in range(TILE)], np.int64)
        self.v_byte = np.array([[int8_v_byte(D, r, d) for d in range(D)] for r in range(TILE)], np.int64)


class BF16Tables:
    """For token slot r: bf16 element index of each dim (D,) in the K and V blocks."""

    def __init__(self, D):
        self.D = D
        self.k_elem = np.array([[bf16_k_elem(D, r, d) for d in range(D)] for r in range(TILE)], np.int64)
        self.v_elem = np.array([[bf16_v_elem(D, r, d) for d in range(D)] for r in range(TILE)], np.int64)


class Int2Tables:
    """For token slot r: the K and V bytes it owns (D/4 each) and, per byte, the dims of its four crumbs."""

    def __init__(self, D):
        self.D = D
        for which, fn in (("k", int2_k_crumb), ("v", int2_v_crumb)):
            byte = np.zeros((TILE, D // 4), np.int64)
            dims = np.zeros((TILE, D // 4, 4), np.int64)
            for r in range(TILE):
                owned = {}
                for d in range(D):
                    b, c = fn(D, r, d)
                    owned.setdefault(b, [None] * 4)[c] = d
                if len(owned) != D // 4 or any(None in v for v in owned.values()):
                    raise AssertionError("INT2 %s layout: token %d does not own whole bytes" % (which, r))
                for n, b in enumerate(sorted(owned)):
                    byte[r, n] = b
                    dims[r, n] = owned[b]
            setattr(self, which + "_byte", byte)
            setattr(self, which + "_dims", dims)


class Fp4Tables:
    """For token slot r: the K bytes it owns (D/2) with their low / high dims; per dim its V byte and
    nibble (D); its scale bytes per 16-dim block (D/16) for K and V."""

    def __init__(self, D):
        self.D = D
        self.k_byte = np.zeros((TILE, D // 2), np.int64)
        self.k_lo = np.zeros((TILE, D // 2), np.int64)
        self.k_hi = np.zeros((TILE, D // 2), np.int64)
        for r in range(TILE):
            owned = {}
            for d in range(D):
                byte, half = fp4_k_nibble(D, r, d)
                owned.setdefault(byte, [None, None])[half] = d
            if len(owned) != D // 2 or any(None in v for v in owned.values()):
                raise AssertionError("NVFP4 K layout: token %d does not own whole bytes" % r)
            for n, byte in enumerate(sorted(owned)):
                self.k_byte[r, n] = byte
                self.k_lo[r, n], self.k_hi[r, n] = owned[byte]
        vb = [[fp4_v_nibble(D, r, d) for d in range(D)] for r in range(TILE)]
        self.v_byte = np.array([[x[0] for x in row] for row in vb], np.int64)
        self.v_nib = np.array([[x[1] for x in row] for row in vb], np.int64)
        self.ks_byte = np.array([[fp4_k_scale_byte(D, r, b) for b in range(D // 16)] for r in range(TILE)], np.int64)
        self.vs_byte = np.array([[fp4_v_scale_byte(D, r, m) for m in range(D // 16)] for r in range(TILE)], np.int64)


_cache = {}


def tables(kind, D):
    key = (kind, D)
    if key not in _cache:
        _cache[key] = {"int4": Int4Tables, "int8": Int8Tables, "bf16": BF16Tables, "nvfp4": Fp4Tables,
                       "int2": Int2Tables}[kind](D)
    return _cache[key]

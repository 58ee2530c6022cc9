"""Paged KV cache with INT4 pages and an INT8 sink/recent store (oracle; test infrastructure only).

Sources:
* "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
  Serving", Abstract -- rotate, quantize token-wise and write straight into a
  paged KV-cache layout (block table of pages per sequence).
* "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache
  Quantization", Abstract -- INT4 for the full context, INT8 protection of
  attention sinks and recent context, for a bounded number of positions.

Readings of this library (the pages give none of these details):

* Dual store.  Every appended token at position p is INT4-encoded into page
  block_table[seq][p // P], slot p % P.  It is also INT8-encoded into the
  per-sequence protected store: slot p when p < S (sinks), otherwise ring slot
  S + ((p - S) mod W).  In a multi-token append only tokens with
  p >= L_new - W write the ring, so each ring slot is written once per append.
* Effective view at length L: p < S -> INT8 sink slot; p >= S and p >= L - W
  -> INT8 ring slot; otherwise the INT4 page.  The protected count is
  min(L, S + W) and those slots are exactly the prefix [0, min(L, S+W)) of the
  store.  A token that leaves the window needs no re-quantization: its INT4
  copy was made from the original values.  The "INT4-only" view reads the
  pages for every position.
* K and V are quantized separately, each with its own (s, z), each after the
  same block-diagonal Hadamard rotation.
* Keys arrive post-RoPE; RoPE is not part of this cache.
"""

import numpy as np

from .hadamard import fwht_fp32
from .quant import quantize_groups, dequantize_groups
from .layout import TILE, tables, int4_tile_bytes, int8_tile_bytes, bf16_tile_bytes, scale_offset

CONFIG_FIELDS = ("num_layers", "max_seqs", "num_q_heads", "num_kv_heads", "head_dim",
                 "page_size", "num_pages", "max_pages_per_seq", "hadamard_block",
                 "sink_tokens", "recent_window")


def prot_slot(p, S, W):
    """Protected-store slot of position p: p for sinks, S + (p - S) mod W for the ring."""
    return p if p < S else S + (p - S) % W


def n_prot_tiles(S, W):
    return -(-(S + W) // TILE)


def is_protected(p, L, S, W):
    """Whether position p reads the INT8 store in the effective view at length L."""
    return p < S or p >= L - W


def _write_half2(buf, off, s16, z16):
    buf[off:off + 2] = np.frombuffer(np.float16(s16).tobytes(), np.uint8)
    buf[off + 2:off + 4] = np.frombuffer(np.float16(z16).tobytes(), np.uint8)


def _read_half2(buf, off):
    s = np.frombuffer(buf[off:off + 2].tobytes(), np.float16)[0]
    z = np.frombuffer(buf[off + 2:off + 4].tobytes(), np.float16)[0]
    return s, z


class OracleKV4Cache:
    """The cache state: per-layer INT4 pages, per-(layer, seq) INT8 store, sequence lengths.

    Pages are held sparsely: pages[(layer, page)] is uint8 [Hkv, P/16, int4 tile];
    prot[(layer, seq)] is uint8 [Hkv, n_prot_tiles, int8 tile].  Bytes never
    written are zero here and undefined on the device.
    """

    def __init__(self, cfg, block_table):
        self.cfg = dict(cfg)
        for f in CONFIG_FIELDS:
            if f not in self.cfg:
                raise KeyError(f)
        c = self.cfg
        if c["page_size"] % TILE:
            raise ValueError("page_size must be a multiple of 16")
        self.D = c["head_dim"]
        self.Hkv = c["num_kv_heads"]
        self.P = c["page_size"]
        self.S = c["sink_tokens"]
        self.W = c["recent_window"]
        self.Bh = c["hadamard_block"]
        self.block_table = np.asarray(block_table, dtype=np.int64)
        self.seq_lens = np.zeros((c["num_layers"], c["max_seqs"]), np.int64)
        self.pages = {}
        self.prot = {}
        self.t4 = tables("int4", self.D)
        self.t8 = tables("int8", self.D)

    # -- storage helpers -------------------------------------------------
    def _page_tile(self, layer, seq, p):
        page = int(self.block_table[seq, p // self.P])
        if page < 0 or page >= self.cfg["num_pages"]:
            raise ValueError("block table entry %d for seq %d page %d is unmapped" % (page, seq, p // self.P))
        key = (layer, page)
        if key not in self.pages:
            self.pages[key] = np.zeros((self.Hkv, self.P // TILE, int4_tile_bytes(self.D)), np.uint8)
        return self.pages[key][:, (p % self.P) // TILE, :], p % TILE

    def _prot_tile(self, layer, seq, slot):
        key = (layer, seq)
        if key not in self.prot:
            self.prot[key] = np.zeros((self.Hkv, n_prot_tiles(self.S, self.W), int8_tile_bytes(self.D)), np.uint8)
        return self.prot[key][:, slot // TILE, :], slot % TILE

    def _put_int4(self, tiles_h, r, codes, s16, z16, tensor):
        """tiles_h: [Hkv, tile bytes] view; codes [Hkv, D]; s16/z16 [Hkv]."""
        D = self.D
        base = 0 if tensor == 0 else 8 * D
        if tensor == 0:
            byte, lo, hi = self.t4.k_byte[r], self.t4.k_lo[r], self.t4.k_hi[r]
        else:
            byte, lo, hi = self.t4.v_byte[r], self.t4.v_lo[r], self.t4.v_hi[r]
        tiles_h[:, base + byte] = codes[:, lo] | (codes[:, hi] << 4)
        off = 16 * D + scale_offset(r, tensor)
        for h in range(self.Hkv):
            _write_half2(tiles_h[h], off, s16[h], z16[h])

    def _put_int8(self, tiles_h, r, codes, s16, z16, tensor):
        D = self.D
        base = 0 if tensor == 0 else 16 * D
        byte = self.t8.k_byte[r] if tensor == 0 else self.t8.v_byte[r]
        tiles_h[:, base + byte] = codes
        off = 32 * D + scale_offset(r, tensor)
        for h in range(self.Hkv):
            _write_half2(tiles_h[h], off, s16[h], z16[h])

    def _get_int4(self, tiles_h, r, tensor):
        D = self.D
        base = 0 if tensor == 0 else 8 * D
        if tensor == 0:
            byte, lo, hi = self.t4.k_byte[r], self.t4.k_lo[r], self.t4.k_hi[r]
        else:
            byte, lo, hi = self.t4.v_byte[r], self.t4.v_lo[r], self.t4.v_hi[r]
        b = tiles_h[:, base + byte]
        codes = np.zeros((self.Hkv, D), np.uint8)
        codes[:, lo] = b & 15
        codes[:, hi] = b >> 4
        off = 16 * D + scale_offset(r, tensor)
        sz = [_read_half2(tiles_h[h], off) for h in range(self.Hkv)]
        s16 = np.array([a for a, _ in sz], np.float16)
        z16 = np.array([b_ for _, b_ in sz], np.float16)
        return codes, s16, z16

    def _get_int8(self, tiles_h, r, tensor):
        D = self.D
        base = 0 if tensor == 0 else 16 * D
        byte = self.t8.k_byte[r] if tensor == 0 else self.t8.v_byte[r]
        codes = tiles_h[:, base + byte].astype(np.uint8)
        off = 32 * D + scale_offset(r, tensor)
        sz = [_read_half2(tiles_h[h], off) for h in range(self.Hkv)]
        s16 = np.array([a for a, _ in sz], np.float16)
        z16 = np.array([b_ for _, b_ in sz], np.float16)
        return codes, s16, z16

    # -- the method --------------------------------------------------------
    def rotate_quantize(self, x):
        """x: [n, Hkv, D] values (bf16 held in fp32).  Returns the rotation and both encodings."""
        xr = fwht_fp32(x, self.Bh)
        return xr, quantize_groups(xr, 4), quantize_groups(xr, 8)

    def append(self, layer, seq_ids, cu_new, k_new, v_new):
        """Append new tokens: seq_ids[i] receives rows cu_new[i]:cu_new[i+1] of k_new / v_new.

        k_new, v_new: [total_new, Hkv, D] bf16 values (as fp32 or bf16-exact floats).
        """
        k_new = np.asarray(k_new, np.float32)
        v_new = np.asarray(v_new, np.float32)
        cap = self.cfg["max_pages_per_seq"] * self.P
        for i, seq in enumerate(seq_ids):
            a, b = int(cu_new[i]), int(cu_new[i + 1])
            n = b - a
            if n <= 0:
                continue
            L_old = int(self.seq_lens[layer, seq])
            L_new = L_old + n
            if L_new > cap:
                raise ValueError("sequence %d would exceed its capacity of %d tokens" % (seq, cap))
            enc = [self.rotate_quantize(k_new[a:b]), self.rotate_quantize(v_new[a:b])]
            for j in range(n):
                p = L_old + j
                tiles_h, r = self._page_tile(layer, seq, p)
                for tensor in (0, 1):
                    _, (c4, s4, z4), _ = enc[tensor]
                    self._put_int4(tiles_h, r, c4[j], s4[j], z4[j], tensor)
                if p < self.S or p >= L_new - self.W:
                    ptiles, r8 = self._prot_tile(layer, seq, prot_slot(p, self.S, self.W))
                    for tensor in (0, 1):
                        _, _, (c8, s8, z8) = enc[tensor]
                        self._put_int8(ptiles, r8, c8[j], s8[j], z8[j], tensor)
            self.seq_lens[layer, seq] = L_new

    def view(self, layer, seq, protected=True, start=0, count=None):
        """Dequantized K^, V^ [count, Hkv, D] fp32 in the rotated basis.

        protected=True gives the effective view (INT8 for protected positions),
        protected=False reads the INT4 pages for every position.
        """
        L = int(self.seq_lens[layer, seq])
        if count is None:
            count = L - start
        if start < 0 or start + count > L:
            raise ValueError("range outside the sequence")
        out = [np.zeros((count, self.Hkv, self.D), np.float32) for _ in range(2)]
        for j in range(count):
            p = start + j
            if protected and is_protected(p, L, self.S, self.W):
                tiles_h, r = self._prot_tile(layer, seq, prot_slot(p, self.S, self.W))
                for tensor in (0, 1):
                    c, s, z = self._get_int8(tiles_h, r, tensor)
                    out[tensor][j] = dequantize_groups(c, s, z)
            else:
                tiles_h, r = self._page_tile(layer, seq, p)
                for tensor in (0, 1):
                    c, s, z = self._get_int4(tiles_h, r, tensor)
                    out[tensor][j] = dequantize_groups(c, s, z)
        return out[0], out[1]


class OracleBF16Cache:
    """The BF16 baseline cache: same block table and page placement, bf16 values, no rotation."""

    def __init__(self, cfg, block_table):
        self.cfg = dict(cfg)
        self.D = cfg["head_dim"]
        self.Hkv = cfg["num_kv_heads"]
        self.P = cfg["page_size"]
        self.block_table = np.asarray(block_table, dtype=np.int64)
        self.seq_lens = np.zeros((cfg["num_layers"], cfg["max_seqs"]), np.int64)
        self.pages = {}
        self.tb = tables("bf16", self.D)

    def _page_tile(self, layer, seq, p):
        page = int(self.block_table[seq, p // self.P])
        if page < 0 or page >= self.cfg["num_pages"]:
            raise ValueError("unmapped page")
        key = (layer, page)
        if key not in self.pages:
            self.pages[key] = np.zeros((self.Hkv, self.P // TILE, bf16_tile_bytes(self.D) // 2), np.uint16)
        return self.pages[key][:, (p % self.P) // TILE, :], p % TILE

    def append(self, layer, seq_ids, cu_new, k_new, v_new):
        k_bits = _bf16_bits(k_new)
        v_bits = _bf16_bits(v_new)
        D = self.D
        for i, seq in enumerate(seq_ids):
            a, b = int(cu_new[i]), int(cu_new[i + 1])
            L_old = int(self.seq_lens[layer, seq])
            for j in range(b - a):
                tiles_h, r = self._page_tile(layer, seq, L_old + j)
                tiles_h[:, self.tb.k_elem[r]] = k_bits[a + j]
                tiles_h[:, 16 * D + self.tb.v_elem[r]] = v_bits[a + j]
            self.seq_lens[layer, seq] = L_old + (b - a)

    def view(self, layer, seq):
        L = int(self.seq_lens[layer, seq])
        D = self.D
        k = np.zeros((L, self.Hkv, D), np.uint16)
        v = np.zeros((L, self.Hkv, D), np.uint16)
        for p in range(L):
            tiles_h, r = self._page_tile(layer, seq, p)
            k[p] = tiles_h[:, self.tb.k_elem[r]]
            v[p] = tiles_h[:, 16 * D + self.tb.v_elem[r]]
        return _bits_bf16(k), _bits_bf16(v)


def _bf16_bits(x):
    """fp32 array holding bf16-representable values -> uint16 bf16 bit patterns."""
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    u = x.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-representable")
    return (u >> 16).astype(np.uint16)


def _bits_bf16(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32)

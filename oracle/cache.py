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
* Keys arrive post-RoPE, or get RoPE at their positions on the way in when a
  table is given (append(..., rope=...), see rope.py).
* Page format (config key "page_format"): 0 = INT4 (the method), 1 = NVFP4,
  the alternative format of the "KV Cache Quantization" topic page, item 3
  (see nvfp4.py), 2 = INT2, the folded-scale 2-bit variant of the same page's
  item 2 (the token-wise quantizer of quant.py with Q = 3).  The format
  changes only what the pages hold; the rotation, the INT8 store of the
  protected positions and the effective view are the same.  Below, "INT4
  page" means the page copy in any format.
* Device byte order (head-innermost, so that the tiles of all KV heads at one
  page position are contiguous):
    INT4 pool of a layer   uint8 [num_pages][P/16][Hkv][16*D + 128]
    NVFP4 pool of a layer  uint8 [num_pages][P/16][Hkv][18*D]
    INT2 pool of a layer   uint8 [num_pages][P/16][Hkv][8*D + 128]
    INT8 store of a layer  uint8 [max_seqs][ceil((S+W)/16)][Hkv][32*D + 128]
    BF16 pool of a layer   bf16  [num_pages][P/16][Hkv][32*D]
  The arrays below use the same order per page / per sequence.
"""

import numpy as np

from .hadamard import fwht_fp32
from .rope import rope_fp32
from .quant import quantize_groups, dequantize_groups
from .nvfp4 import quantize_nvfp4, dequantize_nvfp4
from .layout import (TILE, tables, int4_tile_bytes, int8_tile_bytes, bf16_tile_bytes, fp4_tile_bytes,
                     int2_tile_bytes, scale_offset)

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


class OracleKV4Cache:
    """The cache state: per-layer INT4 pages, per-(layer, seq) INT8 store, sequence lengths.

    Pages are held sparsely: pages[(layer, page)] is uint8 [P/16, Hkv, int4 tile];
    prot[(layer, seq)] is uint8 [n_prot_tiles, Hkv, int8 tile].  Bytes never
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
        self.fmt = int(c.get("page_format", 0))
        if self.fmt not in (0, 1, 2):
            raise ValueError("page_format must be 0 (INT4), 1 (NVFP4) or 2 (INT2)")
        self.block_table = np.asarray(block_table, dtype=np.int64)
        self.seq_lens = np.zeros((c["num_layers"], c["max_seqs"]), np.int64)
        self.pages = {}
        self.prot = {}
        self.t4 = tables("int4", self.D)
        self.t8 = tables("int8", self.D)
        self.tf = tables("nvfp4", self.D)
        self.t2 = tables("int2", self.D)
        self.page_tile_bytes = {0: int4_tile_bytes, 1: fp4_tile_bytes, 2: int2_tile_bytes}[self.fmt](self.D)

    # -- storage helpers -------------------------------------------------
    def _page_tiles(self, layer, page):
        key = (layer, page)
        if key not in self.pages:
            self.pages[key] = np.zeros((self.P // TILE, self.Hkv, self.page_tile_bytes), np.uint8)
        return self.pages[key]

    def _prot_tiles(self, layer, seq):
        key = (layer, seq)
        if key not in self.prot:
            self.prot[key] = np.zeros((n_prot_tiles(self.S, self.W), self.Hkv, int8_tile_bytes(self.D)), np.uint8)
        return self.prot[key]

    def _pages_of(self, seq, pos):
        """Physical page of every position (raises on an unmapped entry)."""
        page = self.block_table[seq, pos // self.P]
        if np.any((page < 0) | (page >= self.cfg["num_pages"])):
            raise ValueError("block table entry of sequence %d is unmapped" % seq)
        return page

    @staticmethod
    def _sz_bytes(s16, z16):
        """[m, Hkv] fp16 scale / zero -> [m, Hkv, 4] bytes (s low, s high, z low, z high)."""
        sb = np.ascontiguousarray(s16, np.float16).view(np.uint8).reshape(s16.shape + (2,))
        zb = np.ascontiguousarray(z16, np.float16).view(np.uint8).reshape(z16.shape + (2,))
        return np.concatenate([sb, zb], axis=-1)

    @staticmethod
    def _sz_values(b):
        """[..., 4] bytes -> (s16, z16)."""
        b = np.ascontiguousarray(b)
        s16 = b[..., 0:2].copy().view(np.float16)[..., 0]
        z16 = b[..., 2:4].copy().view(np.float16)[..., 0]
        return s16, z16

    def _scatter(self, tiles, ti, byte_idx, vals):
        """tiles [T, Hkv, bytes]; ti [m]; byte_idx [m, k]; vals [m, Hkv, k] -> tiles[ti_j, h, byte_idx_j] = vals[j, h]."""
        for h in range(self.Hkv):
            tiles[ti[:, None], h, byte_idx] = vals[:, h, :]

    def _gather(self, tiles, ti, byte_idx):
        """Inverse of _scatter: returns [m, Hkv, k]."""
        return np.stack([tiles[ti[:, None], h, byte_idx] for h in range(self.Hkv)], axis=1)

    def _write_int4(self, layer, seq, pos, enc_k, enc_v):
        """INT4 codes and scales of positions `pos` (enc_*: codes [m, Hkv, D], s16, z16 [m, Hkv])."""
        D, t4 = self.D, self.t4
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        for pg in np.unique(page):
            sel = page == pg
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            for tensor, (codes, s16, z16) in enumerate((enc_k, enc_v)):
                if tensor == 0:
                    byte, lo, hi, base = t4.k_byte[rs], t4.k_lo[rs], t4.k_hi[rs], 0
                else:
                    byte, lo, hi, base = t4.v_byte[rs], t4.v_lo[rs], t4.v_hi[rs], 8 * D
                c = codes[sel]                                            # [m, Hkv, D]
                lo_c = np.take_along_axis(c, lo[:, None, :], axis=2)      # low-nibble dims of each byte
                hi_c = np.take_along_axis(c, hi[:, None, :], axis=2)
                self._scatter(tiles, ts, base + byte, lo_c | (hi_c << 4))
                off = 16 * D + np.array([scale_offset(int(x), tensor) for x in rs])
                self._scatter(tiles, ts, off[:, None] + np.arange(4), self._sz_bytes(s16[sel], z16[sel]))

    def _write_fp4(self, layer, seq, pos, enc_k, enc_v):
        """NVFP4 codes and block scales of positions `pos` (enc_*: codes [m, Hkv, D], scales [m, Hkv, D/16]).

        A V byte holds one dim of two tokens: only this token's nibble of it changes."""
        D, tf = self.D, self.tf
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        for pg in np.unique(page):
            sel = page == pg
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            kc, ks = enc_k[0][sel], enc_k[1][sel]
            lo_c = np.take_along_axis(kc, tf.k_lo[rs][:, None, :], axis=2)
            hi_c = np.take_along_axis(kc, tf.k_hi[rs][:, None, :], axis=2)
            self._scatter(tiles, ts, tf.k_byte[rs], lo_c | (hi_c << 4))
            self._scatter(tiles, ts, tf.ks_byte[rs], ks)
            self._scatter(tiles, ts, tf.vs_byte[rs], enc_v[1][sel])
            vc = enc_v[0][sel]                                            # [m, Hkv, D]
            for j in range(len(rs)):
                byte = 8 * D + tf.v_byte[rs[j]]                           # [D]
                shift = 4 * tf.v_nib[rs[j]]
                for h in range(self.Hkv):
                    old = tiles[ts[j], h, byte].astype(np.int64)
                    new = (old & ~(15 << shift)) | (vc[j, h].astype(np.int64) << shift)
                    tiles[ts[j], h, byte] = new.astype(np.uint8)

    def _read_fp4(self, layer, seq, pos):
        """Dequantized K^, V^ [m, Hkv, D] of positions `pos` from NVFP4 pages."""
        D, tf = self.D, self.tf
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        out = [np.zeros((len(pos), self.Hkv, D), np.float32) for _ in range(2)]
        for pg in np.unique(page):
            sel = np.nonzero(page == pg)[0]
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            b = self._gather(tiles, ts, tf.k_byte[rs])                       # [m, Hkv, D/2]
            kc = np.zeros((len(sel), self.Hkv, D), np.uint8)
            np.put_along_axis(kc, tf.k_lo[rs][:, None, :], b & 15, axis=2)
            np.put_along_axis(kc, tf.k_hi[rs][:, None, :], b >> 4, axis=2)
            out[0][sel] = dequantize_nvfp4(kc, self._gather(tiles, ts, tf.ks_byte[rs]))
            vb = self._gather(tiles, ts, 8 * D + tf.v_byte[rs])               # [m, Hkv, D]
            vc = ((vb >> (4 * tf.v_nib[rs])[:, None, :]) & 15).astype(np.uint8)
            out[1][sel] = dequantize_nvfp4(vc, self._gather(tiles, ts, tf.vs_byte[rs]))
        return out

    def _write_int2(self, layer, seq, pos, enc_k, enc_v):
        """INT2 codes (four a byte, token-owned bytes) and the half2 (s, z) of positions `pos`."""
        D, t2 = self.D, self.t2
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        for pg in np.unique(page):
            sel = page == pg
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            for tensor, (codes, s16, z16) in enumerate((enc_k, enc_v)):
                byte = (t2.k_byte if tensor == 0 else 4 * D + t2.v_byte)[rs]              # [m, D/4]
                dims = (t2.k_dims if tensor == 0 else t2.v_dims)[rs]                      # [m, D/4, 4]
                c = codes[sel].astype(np.uint32)                                          # [m, Hkv, D]
                packed = np.zeros(c.shape[:2] + (D // 4,), np.uint32)
                for k in range(4):
                    packed |= np.take_along_axis(c, dims[:, None, :, k], axis=2) << (2 * k)
                self._scatter(tiles, ts, byte, packed.astype(np.uint8))
                off = 8 * D + np.array([scale_offset(int(x), tensor) for x in rs])
                self._scatter(tiles, ts, off[:, None] + np.arange(4), self._sz_bytes(s16[sel], z16[sel]))

    def _read_int2(self, layer, seq, pos):
        """Dequantized K^, V^ [m, Hkv, D] of positions `pos` from INT2 pages."""
        D, t2 = self.D, self.t2
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        out = [np.zeros((len(pos), self.Hkv, D), np.float32) for _ in range(2)]
        for pg in np.unique(page):
            sel = np.nonzero(page == pg)[0]
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            for tensor in (0, 1):
                byte = (t2.k_byte if tensor == 0 else 4 * D + t2.v_byte)[rs]
                dims = (t2.k_dims if tensor == 0 else t2.v_dims)[rs]
                b = self._gather(tiles, ts, byte)                                         # [m, Hkv, D/4]
                codes = np.zeros((len(sel), self.Hkv, D), np.uint8)
                for k in range(4):
                    np.put_along_axis(codes, dims[:, None, :, k], (b >> (2 * k)) & 3, axis=2)
                off = 8 * D + np.array([scale_offset(int(x), tensor) for x in rs])
                s16, z16 = self._sz_values(self._gather(tiles, ts, off[:, None] + np.arange(4)))
                out[tensor][sel] = dequantize_groups(codes, s16, z16)
        return out

    def _write_int8(self, layer, seq, slots, enc_k, enc_v):
        D, t8 = self.D, self.t8
        tiles = self._prot_tiles(layer, seq)
        r, ti = slots % TILE, slots // TILE
        for tensor, (codes, s16, z16) in enumerate((enc_k, enc_v)):
            byte = (t8.k_byte if tensor == 0 else 16 * D + t8.v_byte)[r]     # [m, D]: byte of each dim
            self._scatter(tiles, ti, byte, codes)
            off = 32 * D + np.array([scale_offset(int(x), tensor) for x in r])
            self._scatter(tiles, ti, off[:, None] + np.arange(4), self._sz_bytes(s16, z16))

    def _read_int4(self, layer, seq, pos):
        """Dequantized K^, V^ [m, Hkv, D] of positions `pos` from the pages."""
        D, t4 = self.D, self.t4
        page = self._pages_of(seq, pos)
        r = pos % TILE
        ti = (pos % self.P) // TILE
        out = [np.zeros((len(pos), self.Hkv, D), np.float32) for _ in range(2)]
        for pg in np.unique(page):
            sel = np.nonzero(page == pg)[0]
            tiles = self._page_tiles(layer, int(pg))
            rs, ts = r[sel], ti[sel]
            for tensor in (0, 1):
                if tensor == 0:
                    byte, lo, hi, base = t4.k_byte[rs], t4.k_lo[rs], t4.k_hi[rs], 0
                else:
                    byte, lo, hi, base = t4.v_byte[rs], t4.v_lo[rs], t4.v_hi[rs], 8 * D
                b = self._gather(tiles, ts, base + byte)                      # [m, Hkv, D/2]
                codes = np.zeros((len(sel), self.Hkv, D), np.uint8)
                np.put_along_axis(codes, lo[:, None, :], b & 15, axis=2)
                np.put_along_axis(codes, hi[:, None, :], b >> 4, axis=2)
                off = 16 * D + np.array([scale_offset(int(x), tensor) for x in rs])
                s16, z16 = self._sz_values(self._gather(tiles, ts, off[:, None] + np.arange(4)))
                out[tensor][sel] = dequantize_groups(codes, s16, z16)
        return out

    def _read_int8(self, layer, seq, slots):
        D, t8 = self.D, self.t8
        tiles = self._prot_tiles(layer, seq)
        r, ti = slots % TILE, slots // TILE
        out = []
        for tensor in (0, 1):
            byte = (t8.k_byte if tensor == 0 else 16 * D + t8.v_byte)[r]
            codes = self._gather(tiles, ti, byte)
            off = 32 * D + np.array([scale_offset(int(x), tensor) for x in r])
            s16, z16 = self._sz_values(self._gather(tiles, ti, off[:, None] + np.arange(4)))
            out.append(dequantize_groups(codes, s16, z16))
        return out

    # -- the method --------------------------------------------------------
    def rotate_quantize(self, x):
        """x: [n, Hkv, D] values (bf16 held in fp32).  Returns the rotation, the page encoding (INT4 or
        INT2 (codes, s16, z16), NVFP4 (codes, scales)) and the INT8 encoding."""
        xr = fwht_fp32(x, self.Bh)
        page = quantize_nvfp4(xr) if self.fmt == 1 else quantize_groups(xr, 2 if self.fmt == 2 else 4)
        return xr, page, quantize_groups(xr, 8)

    def append(self, layer, seq_ids, cu_new, k_new, v_new, rope=None):
        """Append new tokens: seq_ids[i] receives rows cu_new[i]:cu_new[i+1] of k_new / v_new.

        k_new, v_new: [total_new, Hkv, D] bf16 values (as fp32 or bf16-exact floats).
        rope: None, or (cos_sin, R, style): each new key first gets RoPE at its position.
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
            pos = L_old + np.arange(n)
            kx = k_new[a:b]
            if rope is not None:
                kx = rope_fp32(kx, pos[:, None], *rope)
            _, k4, k8 = self.rotate_quantize(kx)
            _, v4, v8 = self.rotate_quantize(v_new[a:b])
            if self.fmt == 1:                                    # every position: the page copy
                self._write_fp4(layer, seq, pos, k4, v4)
            elif self.fmt == 2:
                self._write_int2(layer, seq, pos, k4, v4)
            else:
                self._write_int4(layer, seq, pos, k4, v4)
            prot = (pos < self.S) | (pos >= L_new - self.W)      # sinks, and the last W of this append
            if np.any(prot):
                j = np.nonzero(prot)[0]
                slots = np.array([prot_slot(int(p), self.S, self.W) for p in pos[j]])
                self._write_int8(layer, seq, slots, tuple(x[j] for x in k8), tuple(x[j] for x in v8))
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
        if count == 0:
            return out[0], out[1]
        pos = start + np.arange(count)
        from_int8 = np.array([protected and is_protected(int(p), L, self.S, self.W) for p in pos])
        for src, sel in ((False, ~from_int8), (True, from_int8)):
            if not np.any(sel):
                continue
            if src:
                slots = np.array([prot_slot(int(p), self.S, self.W) for p in pos[sel]])
                kv = self._read_int8(layer, seq, slots)
            elif self.fmt == 1:
                kv = self._read_fp4(layer, seq, pos[sel])
            elif self.fmt == 2:
                kv = self._read_int2(layer, seq, pos[sel])
            else:
                kv = self._read_int4(layer, seq, pos[sel])
            out[0][sel], out[1][sel] = kv
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
            self.pages[key] = np.zeros((self.P // TILE, self.Hkv, bf16_tile_bytes(self.D) // 2), np.uint16)
        return self.pages[key][(p % self.P) // TILE], p % TILE

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

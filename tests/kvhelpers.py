"""Shared helpers of the parity tests: build the same cache on the GPU (through the C ABI)
and in the oracle (on the CPU) from identical inputs, and compare them."""

import numpy as np
import torch

from oracle import OracleKV4Cache, OracleBF16Cache, decode_attention, decode_attention_bf16
from oracle.layout import tables, scale_offset, TILE

# Tolerances (attention):
#  * bf16 output: kernel bf16 vs oracle bf16 (both rounded from values that agree to ~1e-5),
#    rel-L2 <= 1e-3 and max-abs <= max(2e-3, one bf16 ulp of the oracle value);
#  * fp32 output: kernel fp32 vs oracle fp64, max-abs <= 2e-3 and rel-L2 <= 1e-3.
REL_L2 = 1e-3
MAX_ABS = 2e-3
# BF16 baseline (P rounded to bf16 before P.V, unit roundoff 2^-8): fp32 output vs fp64,
# rel-L2 <= 5e-3, max-abs <= 4 * 2^-8 (|v| <= ~4 for N(0,1) values).
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 4 * 2.0 ** -8


def cfg_dict(D=128, Hq=32, Hkv=8, P=16, Bh=128, S=4, W=128, num_pages=64, mpps=16, max_seqs=4, layers=1, fmt=0):
    return dict(num_layers=layers, max_seqs=max_seqs, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, page_size=P,
                num_pages=num_pages, max_pages_per_seq=mpps, hadamard_block=Bh, sink_tokens=S, recent_window=W,
                page_format=fmt)


def random_table(max_seqs, mpps, num_pages, rng):
    """Seeded permutation of pages handed to sequences in order; -1 where the pool runs out."""
    perm = rng.permutation(num_pages).astype(np.int32)
    t = np.full((max_seqs, mpps), -1, np.int32)
    k = 0
    for s in range(max_seqs):
        n = min(mpps, num_pages - k)
        t[s, :n] = perm[k:k + n]
        k += n
    return t


def bf16_values(shape, rng, scale=1.0, outlier_ch=None, outlier=1.0):
    x = rng.standard_normal(shape).astype(np.float32) * scale
    if outlier_ch is not None:
        x[..., outlier_ch] *= outlier
    return torch.from_numpy(x).to(torch.bfloat16)


def f32(t):
    """bf16 tensor -> fp32 numpy (exact)."""
    return t.float().cpu().numpy()


class Pair:
    """A GPU cache (KV4Cache or BF16Cache) and the oracle cache fed identical appends."""

    def __init__(self, cfg, table, bf16=False, device="cuda"):
        import int4_kv_cache_paged_b200 as kv4
        self.cfg = cfg
        self.table = np.asarray(table, np.int32)
        self.bf16 = bf16
        self.device = device
        self.gpu = (kv4.BF16Cache if bf16 else kv4.KV4Cache)(cfg, torch.from_numpy(self.table), device)
        self.orc = (OracleBF16Cache if bf16 else OracleKV4Cache)(cfg, self.table)

    def append(self, layer, seq_ids, counts, k, v, oracle=True):
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        dev = self.device
        self.gpu.append(layer, torch.tensor(seq_ids, dtype=torch.int32, device=dev),
                        torch.from_numpy(cu).to(dev), k.to(dev).contiguous(), v.to(dev).contiguous(),
                        total_new=int(cu[-1]))
        if oracle:
            self.orc.append(layer, list(seq_ids), cu, f32(k), f32(v))

    def attention(self, layer, seq_ids, q, scale=0.0, mode=0):
        dev = self.device
        return self.gpu.attention(layer, torch.tensor(seq_ids, dtype=torch.int32, device=dev), q.to(dev).contiguous(),
                                  scale=scale, mode=mode)

    def oracle_attention(self, layer, seq_ids, q, scale=0.0, protected=True):
        if self.bf16:
            return decode_attention_bf16(self.orc, layer, seq_ids, f32(q), scale)
        return decode_attention(self.orc, layer, seq_ids, f32(q), scale, protected=protected)


def compare_int4_pages(pair, layer, seqs):
    """Bit-exact comparison of every INT4 byte owned by a written position of `seqs`."""
    c = pair.cfg
    D, P = c["head_dim"], c["page_size"]
    t4 = tables("int4", D)
    pages = pair.gpu.pages(layer).cpu().numpy()
    ar4 = np.arange(4)
    bad = []
    for seq in seqs:
        L = int(pair.orc.seq_lens[layer, seq])
        for p in range(L):
            page = int(pair.table[seq, p // P])
            ti, r = (p % P) // TILE, p % TILE
            idx = np.concatenate([t4.k_byte[r], 8 * D + t4.v_byte[r], 16 * D + scale_offset(r, 0) + ar4,
                                  16 * D + scale_offset(r, 1) + ar4])
            g = pages[page, ti][:, idx]
            o = pair.orc.pages[(layer, page)][ti][:, idx]
            if not np.array_equal(g, o):
                bad.append((seq, p, int(np.sum(g != o))))
    return bad


def compare_fp4_pages(pair, layer, seqs):
    """Bit-exact comparison of every NVFP4 code and scale owned by a written position of `seqs` (its K
    bytes and scale bytes, and its nibble of each shared V byte)."""
    c = pair.cfg
    D, P = c["head_dim"], c["page_size"]
    tf = tables("nvfp4", D)
    pages = pair.gpu.pages(layer).cpu().numpy()
    bad = []
    for seq in seqs:
        L = int(pair.orc.seq_lens[layer, seq])
        for p in range(L):
            page = int(pair.table[seq, p // P])
            ti, r = (p % P) // TILE, p % TILE
            idx = np.concatenate([tf.k_byte[r], tf.ks_byte[r], tf.vs_byte[r]])
            g = pages[page, ti][:, idx]
            o = pair.orc.pages[(layer, page)][ti][:, idx]
            vb = 8 * D + tf.v_byte[r]
            sh = 4 * tf.v_nib[r]
            gv = (pages[page, ti][:, vb] >> sh) & 15
            ov = (pair.orc.pages[(layer, page)][ti][:, vb] >> sh) & 15
            n = int(np.sum(g != o)) + int(np.sum(gv != ov))
            if n:
                bad.append((seq, p, n))
    return bad


def compare_int2_pages(pair, layer, seqs):
    """Bit-exact comparison of every INT2 byte owned by a written position of `seqs` (K and V code bytes,
    its half2 scale entries)."""
    c = pair.cfg
    D, P = c["head_dim"], c["page_size"]
    t2 = tables("int2", D)
    pages = pair.gpu.pages(layer).cpu().numpy()
    ar4 = np.arange(4)
    bad = []
    for seq in seqs:
        L = int(pair.orc.seq_lens[layer, seq])
        for p in range(L):
            page = int(pair.table[seq, p // P])
            ti, r = (p % P) // TILE, p % TILE
            idx = np.concatenate([t2.k_byte[r], 4 * D + t2.v_byte[r], 8 * D + scale_offset(r, 0) + ar4,
                                  8 * D + scale_offset(r, 1) + ar4])
            g = pages[page, ti][:, idx]
            o = pair.orc.pages[(layer, page)][ti][:, idx]
            if not np.array_equal(g, o):
                bad.append((seq, p, int(np.sum(g != o))))
    return bad


def compare_page_copy(pair, layer, seqs):
    """The page comparison of the cache's page format."""
    fmt = pair.cfg.get("page_format", 0)
    return {0: compare_int4_pages, 1: compare_fp4_pages, 2: compare_int2_pages}[fmt](pair, layer, seqs)


def compare_int8_store(pair, layer, seqs):
    """Bit-exact comparison of the protected slots [0, min(L, S+W)) of `seqs`."""
    c = pair.cfg
    D, S, W = c["head_dim"], c["sink_tokens"], c["recent_window"]
    t8 = tables("int8", D)
    prot = pair.gpu.protected(layer).cpu().numpy()
    ar4 = np.arange(4)
    bad = []
    for seq in seqs:
        L = int(pair.orc.seq_lens[layer, seq])
        for slot in range(min(L, S + W)):
            ti, r = slot // TILE, slot % TILE
            idx = np.concatenate([t8.k_byte[r], 16 * D + t8.v_byte[r], 32 * D + scale_offset(r, 0) + ar4,
                                  32 * D + scale_offset(r, 1) + ar4])
            g = prot[seq, ti][:, idx]
            o = pair.orc.prot[(layer, seq)][ti][:, idx]
            if not np.array_equal(g, o):
                bad.append((seq, slot, int(np.sum(g != o))))
    return bad


def compare_bf16_pages(pair, layer, seqs):
    c = pair.cfg
    D, P = c["head_dim"], c["page_size"]
    tb = tables("bf16", D)
    pages = pair.gpu.pages(layer).cpu().numpy().view(np.uint16)
    bad = []
    for seq in seqs:
        L = int(pair.orc.seq_lens[layer, seq])
        for p in range(L):
            page = int(pair.table[seq, p // P])
            ti, r = (p % P) // TILE, p % TILE
            idx = np.concatenate([tb.k_elem[r], 16 * D + tb.v_elem[r]])
            if not np.array_equal(pages[page, ti][:, idx], pair.orc.pages[(layer, page)][ti][:, idx]):
                bad.append((seq, p))
    return bad


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (x holds bf16 values)."""
    a = np.abs(np.asarray(x, np.float32))
    a = np.where(a == 0, np.float32(2.0 ** -126), a)
    e = np.floor(np.log2(a))
    return np.float32(2.0) ** (e - 7)


def check_bf16_out(got_bf16, ref):
    """got_bf16: kernel output (bf16 tensor); ref: oracle dict. Returns (rel_l2, max_excess)."""
    g = f32(got_bf16).astype(np.float64)
    r = ref["out_bf16"].astype(np.float64)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    allowed = np.maximum(MAX_ABS, bf16_ulp(ref["out_bf16"]))
    excess = float(np.max(np.abs(g - r) - allowed))
    return rel, excess


def check_f32_out(got_f32, ref, rel_tol=REL_L2, abs_tol=MAX_ABS):
    g = got_f32.cpu().numpy().astype(np.float64)
    r = ref["out_f64"]
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    mx = float(np.max(np.abs(g - r)))
    return rel, mx

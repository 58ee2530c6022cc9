"""fp64 GQA decode attention over the effective view (oracle; test infrastructure only).

Source: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
Serving", Abstract -- fused attention over the quantized paged cache; the
query gets the same block-diagonal Hadamard rotation as the keys, so the
scores of the rotated problem equal those of the original one.

Readings of this library:

* q_rot = bf16_round(fwht_fp32(q)): queries are bf16 and stay bf16 after the
  rotation (the kernel can then use 16-bit tensor-core inputs without extra
  error).
* scores s_p = sigma * <q_rot, k^_p> with sigma = 1/sqrt(D) unless the caller
  passes another scale (textbook scaled dot-product attention).
* a = softmax(s) over every cached position 0..L-1 (including the token the
  same decode step appended); o_rot = sum_p a_p v^_p; o = H_blk o_rot (H is
  symmetric and orthonormal, so it is its own inverse); out = bf16(o).
* GQA grouping is contiguous: query head j uses KV head j // (Hq / Hkv).
* A sequence with no cached position gives an all-zero output row (the
  library's convention; softmax over an empty set is undefined).
* Folded rotations (a library option for callers that fold H into W_q and
  o_proj): with q_rotated the given bf16 query is q_rot itself; with
  out_rotated the output is o_rot, not H o_rot.  The attention between them
  is unchanged.
* The bf16 output is rounded fp64 -> fp32 -> bf16 (two round-to-nearest-even
  steps); the tests allow one bf16 ulp between two bf16 outputs for this
  reason.
"""

import numpy as np

from .hadamard import fwht_fp32, block_diag_hadamard
from .quant import bf16_round
from .rope import rope_fp32


def attention_fp64(q, k, v, scale):
    """Textbook GQA attention for one query token.

    q: [Hq, D]; k, v: [L, Hkv, D]; returns o [Hq, D] in fp64:
    o[j] = sum_p softmax_p(scale * <q[j], k[p, j // G]>) v[p, j // G].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Hq, D = q.shape
    L, Hkv, _ = k.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    o = np.zeros((Hq, D), np.float64)
    for j in range(Hq):
        h = j // G
        s = scale * (k[:, h, :] @ q[j])
        a = np.exp(s - s.max())
        a /= a.sum()
        o[j] = a @ v[:, h, :]
    return o


def _bf16_of_f64(x):
    return bf16_round(np.asarray(x, np.float64).astype(np.float32))


def rotate_query(q, Bh):
    """q_rot = bf16_round(fwht_fp32(q)) for bf16 queries q [..., D]."""
    return bf16_round(fwht_fp32(q, Bh))


def _query_and_output_rotation(cache, q, q_rotated, out_rotated, rope=None, qpos=None):
    """q_rot and the matrix that takes o_rot to the output basis.

    q_rotated: the caller passes H q itself (H folded into its query
    projection), used as given.  out_rotated: the output stays in the rotated
    basis (H folded into the output projection), so the map is the identity.
    rope = (cos_sin, R, style): q first gets RoPE at positions qpos (fp32,
    no bf16 rounding before the rotation)."""
    if rope is not None:
        q = rope_fp32(np.asarray(q, np.float32), qpos, *rope)
    q_rot = np.asarray(q, np.float32) if q_rotated else rotate_query(q, cache.Bh)
    back = np.eye(cache.D) if out_rotated else block_diag_hadamard(cache.D, cache.Bh).T
    return q_rot, back


def decode_attention(cache, layer, seq_ids, q, scale=None, protected=True, q_rotated=False, out_rotated=False,
                     rope=None):
    """Decode attention of one query token per sequence over an OracleKV4Cache.

    q: [n, Hq, D] bf16 values (already H q when q_rotated; the output stays
    in the rotated basis when out_rotated; rope: RoPE of q at position L - 1
    first, L the sequence's length).  Returns dict with
      out_f64  [n, Hq, D]  fp64 output in the original (unrotated) basis,
      out_bf16 [n, Hq, D]  the same rounded to bf16 (held in fp32),
      q_rot    [n, Hq, D]  the rotated bf16 queries.
    """
    q = np.asarray(q, np.float32)
    D = cache.D
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    n = len(seq_ids)
    out = np.zeros((n,) + q.shape[1:], np.float64)
    lens = np.array([int(cache.seq_lens[layer, int(s)]) for s in seq_ids], np.int64)
    qpos = np.maximum(lens - 1, 0)[:, None]
    q_rot, back = _query_and_output_rotation(cache, q, q_rotated, out_rotated, rope, qpos)
    for i, seq in enumerate(seq_ids):
        kh, vh = cache.view(layer, int(seq), protected=protected)
        if kh.shape[0] == 0:
            continue                      # an empty sequence has an all-zero output row
        o_rot = attention_fp64(q_rot[i], kh, vh, scale)
        out[i] = o_rot @ back
    return {"out_f64": out, "out_bf16": _bf16_of_f64(out), "q_rot": q_rot}


def extend_attention(cache, layer, seq_ids, q, scale=None, protected=True, q_rotated=False, out_rotated=False,
                     rope=None):
    """Attention of several query tokens per sequence: the last T positions.

    q: [n, T, Hq, D] bf16 values, token i (0 = oldest) of a sequence of length
    L standing at position L - T + i.  Textbook causal attention: token i sees
    positions 0 .. L - T + i.  Every token reads the same effective view, the
    one of length L (sinks and the last W positions of L from INT8; that the
    protected set follows the cache length, not the query position, is this
    library's reading: the cache holds one view at a time).  A token with no
    visible position (L - T + i < 0) gets an all-zero row.  q_rotated,
    out_rotated as in decode_attention; rope: RoPE of token i at L - T + i.

    Returns dict out_f64 / out_bf16 [n, T, Hq, D] and q_rot [n, T, Hq, D].
    """
    q = np.asarray(q, np.float32)
    D = cache.D
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    n, T = q.shape[0], q.shape[1]
    out = np.zeros(q.shape, np.float64)
    lens = np.array([int(cache.seq_lens[layer, int(s)]) for s in seq_ids], np.int64)
    qpos = np.maximum(lens[:, None] - T + np.arange(T)[None, :], 0)[:, :, None]
    q_rot, back = _query_and_output_rotation(cache, q, q_rotated, out_rotated, rope, qpos)
    for b, seq in enumerate(seq_ids):
        kh, vh = cache.view(layer, int(seq), protected=protected)
        L = kh.shape[0]
        for i in range(T):
            vis = L - T + i + 1           # positions 0 .. L - T + i
            if vis <= 0:
                continue
            out[b, i] = attention_fp64(q_rot[b, i], kh[:vis], vh[:vis], scale) @ back
    return {"out_f64": out, "out_bf16": _bf16_of_f64(out), "q_rot": q_rot}


def decode_attention_bf16(cache, layer, seq_ids, q, scale=None):
    """Plain decode attention over an OracleBF16Cache (no rotation, no quantization)."""
    q = np.asarray(q, np.float32)
    D = cache.D
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    n = len(seq_ids)
    out = np.zeros((n,) + q.shape[1:], np.float64)
    for i, seq in enumerate(seq_ids):
        k, v = cache.view(layer, int(seq))
        if k.shape[0]:
            out[i] = attention_fp64(q[i], k, v, scale)
    return {"out_f64": out, "out_bf16": _bf16_of_f64(out)}

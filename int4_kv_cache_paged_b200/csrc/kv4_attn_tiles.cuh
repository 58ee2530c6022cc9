// Tile routines of the split-K decode attention kernels: turn the codes of one
// 16-token tile in shared memory into 16x8x16 tensor-core operands, run the
// scores, the online softmax and P.V.  Used by the page-major INT4/INT8
// kernel and (the BF16 tile) by the per-head BF16 baseline kernel.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Abstract (fused attention over the rotated token-wise INT4 cache);
// scale and zero point are folded out of the inner products as in the
// folded-scale kernels of "KV Cache Quantization" (topic page), item 2:
//     q . k^  = s_k * (q . c_k) + z_k * sum(q)
//     sum_p a_p v^_p = sum_p (a_p s_p) (c_p - 8) + sum_p a_p (z_p + 8 s_p)     (INT4; 128 for INT8)
#pragma once

#include "kv4_common.cuh"

#include <math.h>

namespace kv4 {
namespace tiles {

constexpr float NEG_INF = -INFINITY;

// Partial of one item: per query head, o[D] (unnormalised, rotated basis), m, l,
// padded to D + 4 floats so every head row starts on a 16-byte boundary.
__host__ __device__ constexpr int head_stride(int D) { return D + 4; }
__host__ __device__ inline int partial_stride(int G, int D) { return G * head_stride(D); }

// ---------------------------------------------------------------------------
// per-warp online-softmax state

template <int D>
struct WarpState {
  float o[D / 16][4];  // o^T fragments: (dim 16m+g, head 2t), (16m+g, 2t+1), (16m+g+8, 2t), (16m+g+8, 2t+1)
  float m0, m1, l0, l1, z0, z1;
};

// Column split of the P.V weights (see pv_operands): part of each of the thread's two columns.
struct ColSplit {
  bool colsplit;
  int part0, part1;
};

// Query operand of the scores: q_rot * 2^e rounded to a 16-bit integer and split
// into a signed high byte and an unsigned low byte (q = 256 hi + lo).  b[kk] is
// the high-byte B fragment of 32-dim block kk, b[D/32 + kk] the low-byte one
// (16x8x32 layout: register 0 holds dims 4t..4t+3 of column g, register 1
// dims 16+4t..16+4t+3).  qs0/qs1: sum(q_rot) * scale_log2 of the thread's two
// columns; kscale = scale_log2 * 2^-e.
template <int D>
struct QFrag {
  uint32_t b[D / 16][2];
  float qs0, qs1, kscale;
};

// Integer scores of one 32-dim block: A = the K codes as bytes (rows g and g+8,
// dims 4t..4t+3 and 16+4t..16+4t+3), times both query planes.
template <int D>
__device__ __forceinline__ void qk_block(int (&hi)[4], int (&lo)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, const QFrag<D>& qf, int kk) {
  imma_u8s8(hi, a0, a1, a2, a3, qf.b[kk][0], qf.b[kk][1]);
  imma_u8u8(lo, a0, a1, a2, a3, qf.b[D / 32 + kk][0], qf.b[D / 32 + kk][1]);
}

template <int D, bool GUARD = false>
__device__ __forceinline__ void online_softmax_pv(WarpState<D>& ws, float x0, float x1, float x2, float x3,
                                                  float& p0, float& p1, float& p2, float& p3) {
  float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float n0 = fmaxf(ws.m0, mx0), n1 = fmaxf(ws.m1, mx1);
  if (__any_sync(0xffffffffu, n0 > ws.m0 || n1 > ws.m1)) {
    // GUARD: a column with no visible position so far keeps m = -inf and a zero state
    const float a0 = (GUARD && n0 == NEG_INF) ? 1.f : ex2(ws.m0 - n0);
    const float a1 = (GUARD && n1 == NEG_INF) ? 1.f : ex2(ws.m1 - n1);
    ws.l0 *= a0; ws.l1 *= a1; ws.z0 *= a0; ws.z1 *= a1;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      ws.o[m][0] *= a0; ws.o[m][1] *= a1; ws.o[m][2] *= a0; ws.o[m][3] *= a1;
    }
    ws.m0 = n0; ws.m1 = n1;
  }
  const float u0 = (GUARD && ws.m0 == NEG_INF) ? 0.f : ws.m0, u1 = (GUARD && ws.m1 == NEG_INF) ? 0.f : ws.m1;
  p0 = ex2(x0 - u0); p1 = ex2(x1 - u1); p2 = ex2(x2 - u0); p3 = ex2(x3 - u1);
}


// P.V weights of this thread's two columns (c0 = 2t, c1 = 2t+1) for tokens g and
// g+8.  With the column split (G = 1, 2, 4), column c carries part c / G of the
// weight of head c % G: part 0 = hi = fp16(P), part 1 = lo = fp16(P - hi),
// parts >= 2 are zero; one 16x8x16 multiply then accumulates both parts.
// Without it (other G) the hi parts go to (B0, B1) and the lo parts to (C0, C1).
__device__ __forceinline__ void pv_operands(float P0, float P1, float P2, float P3, int part0, int part1,
                                            bool colsplit, uint32_t& B0, uint32_t& B1, uint32_t& C0, uint32_t& C1) {
  const uint32_t h01 = pack_half2(P0, P1), h23 = pack_half2(P2, P3);
  const uint32_t l01 = pack_half2(P0 - half_lo(h01), P1 - half_hi(h01));
  const uint32_t l23 = pack_half2(P2 - half_lo(h23), P3 - half_hi(h23));
  if (colsplit) {
    const uint32_t m0 = part0 == 0 ? 0x0000FFFFu : 0u, m1 = part1 == 0 ? 0xFFFF0000u : 0u;
    const uint32_t n0 = part0 == 1 ? 0x0000FFFFu : 0u, n1 = part1 == 1 ? 0xFFFF0000u : 0u;
    B0 = movmatrix_trans((h01 & (m0 | m1)) | (l01 & (n0 | n1)));
    B1 = movmatrix_trans((h23 & (m0 | m1)) | (l23 & (n0 | n1)));
    C0 = C1 = 0u;
  } else {
    B0 = movmatrix_trans(h01);
    B1 = movmatrix_trans(h23);
    C0 = movmatrix_trans(l01);
    C1 = movmatrix_trans(l23);
  }
}

// The V code words a lane reads from a page tile: BITS = 4 (INT4 pages), D/16 words at 8D + 16 lane
// (+512), one per 16-dim block; BITS = 2 (INT2 pages), D/32 words at 4D + (D/8) lane, one per pair of
// blocks.
template <int D, int BITS>
__device__ __forceinline__ void load_v_words(uint32_t st, int lane, uint32_t (&vw)[D / 16]) {
  if constexpr (BITS == 4) {
    if constexpr (D == 128) {
      const uint4 v0 = lds128(st + 8 * D + lane * 16), v1 = lds128(st + 8 * D + 512 + lane * 16);
      vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
      vw[4] = v1.x; vw[5] = v1.y; vw[6] = v1.z; vw[7] = v1.w;
    } else {
      const uint4 v0 = lds128(st + 8 * D + lane * 16);
      vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
    }
  } else {
    if constexpr (D == 128) {
      const uint4 v0 = lds128(st + 4 * D + lane * 16);
      vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
    } else {
      const uint2 v0 = lds64(st + 4 * D + lane * 8);
      vw[0] = v0.x; vw[1] = v0.y;
    }
  }
}

// Crumbs at bits P, P+1 and 16+P, 17+P (P <= 8) as an fp16 pair, minus 2 (exact): under the magic
// exponent the crumb is the half 1024 + c 2^P, and one fma by 2^-P takes away 1024 2^-P + 2.
template <int P>
__device__ __forceinline__ uint32_t crumb_c(uint32_t w) {
  static_assert(P >= 0 && P <= 8, "crumb inside the fp16 mantissa");
  uint32_t x = lop3_and_or(w, 0x00030003u << P, 0x64006400u);
  const __half sc = __float2half_rn(1.f / static_cast<float>(1 << P));
  const __half b = __float2half_rn(-(1024.f / static_cast<float>(1 << P) + 2.f));
  __half2 h = __hfma2(*reinterpret_cast<__half2*>(&x), __half2(sc, sc), __half2(b, b));
  return *reinterpret_cast<uint32_t*>(&h);
}

// The four centred A registers of the P.V multiply of dim block m: (dim g | g+8) x (tokens 2t, 2t+1 |
// 2t+8, 2t+9), codes minus 8 (INT4) or minus 2 (INT2).
template <int BITS>
__device__ __forceinline__ void v_operands(const uint32_t* vw, int m, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                           uint32_t& a3) {
  if constexpr (BITS == 4) {
    const uint32_t w = vw[m], u = w >> 8;
    a0 = nib_lo_c(w); a1 = nib_hi_c(w); a2 = nib_lo_c(u); a3 = nib_hi_c(u);
  } else {
    // block m of the pair sits at bits 4 (m % 2) + {0, 2} (dims g, g+8) of the low byte of each half (tokens
    // 2t, 2t+1) and 8 further (tokens 2t+8, 2t+9); a crumb above bit 8 of a half takes one shift
    const uint32_t w = vw[m >> 1], u = w >> 8;
    if (m & 1) {
      a0 = crumb_c<4>(w); a1 = crumb_c<6>(w); a2 = crumb_c<4>(u); a3 = crumb_c<6>(u);
    } else {
      a0 = crumb_c<0>(w); a1 = crumb_c<2>(w); a2 = crumb_c<8>(w); a3 = crumb_c<2>(u);
    }
  }
}

// P.V of one INT4 (or INT2) tile: o^T[m] += V^T codes * (hi + lo) weights.
template <int D, int BITS = 4>
__device__ __forceinline__ void pv_int4(uint32_t st, WarpState<D>& ws, int lane, uint32_t B0, uint32_t B1,
                                        uint32_t C0, uint32_t C1, bool colsplit) {
  uint32_t vw[D / 16];
  load_v_words<D, BITS>(st, lane, vw);
#pragma unroll
  for (int m = 0; m < D / 16; ++m) {
    uint32_t a0, a1, a2, a3;
    v_operands<BITS>(vw, m, a0, a1, a2, a3);
    mma_f16(ws.o[m], a0, a1, a2, a3, B0, B1);
    if (!colsplit) mma_f16(ws.o[m], a0, a1, a2, a3, C0, C1);
  }
}

// One unit of NT INT4 tiles at shared addresses tile[0 .. NT-1]:
// scores, one online-softmax update for the NT*16 tokens, P.V.  valid[u] bits
// 0-3 (used when MASKED): token g of tile u is visible to the thread's column
// 2t / 2t+1, token g+8 to column 2t / 2t+1 (inside the range being read, and
// not after the column's query position).  Without CAUSAL the columns agree
// (bits 0 and 2 decide) and every column sees a token of the unit; with it a
// column may see none, and its state stays at m = -inf, l = 0.
// The stages are handed back (empty barriers eb[0 .. NT-1], each distinct one
// once) after the last shared-memory load.  BITS = 2: INT2 pages (the same
// folded form with 2-bit codes: four a byte, the half2 scales at 8D).
template <int D, int NT, bool MASKED, bool CAUSAL = false, int BITS = 4>
__device__ __forceinline__ void unit_int4(const uint32_t* tile, const QFrag<D>& qf, WarpState<D>& ws, int lane,
                                          const int* valid, const uint32_t* eb, const ColSplit& cs) {
  static_assert(BITS == 4 || BITS == 2, "code width");
  constexpr int SZOFF = BITS == 4 ? 16 * D : 8 * D;          // the half2 (s, z) block of the tile
  constexpr float VCENTRE = BITS == 4 ? 8.f : 2.f;          // P.V takes the codes minus this
  float x[NT][4];
  uint4 sz[NT];
  // Q.K^T of the NT tiles on the integer tensor cores: each tile's K codes are
  // unpacked to bytes with one mask per plane and multiplied by both query
  // planes (2*NT independent accumulator chains of D/32 multiplies).
  constexpr int NKK = D / 32;
  uint32_t kw[NT][2][NKK];   // INT2: the first NKK / 2 words of each row
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    if constexpr (BITS == 4 && D == 128) {
      const uint4 a = lds128(tile[u] + lane * 16), bq = lds128(tile[u] + 512 + lane * 16);
      kw[u][0][0] = a.x; kw[u][0][1] = a.y; kw[u][0][2] = a.z; kw[u][0][3] = a.w;
      kw[u][1][0] = bq.x; kw[u][1][1] = bq.y; kw[u][1][2] = bq.z; kw[u][1][3] = bq.w;
    } else if constexpr (BITS == 4 || D == 128) {   // INT4 at D = 64, INT2 at D = 128: 8 bytes per row
      const uint2 a = lds64(tile[u] + lane * 8), bq = lds64(tile[u] + 256 + lane * 8);   // rows g + 8
      kw[u][0][0] = a.x; kw[u][0][1] = a.y; kw[u][1][0] = bq.x; kw[u][1][1] = bq.y;
    } else {                                        // INT2 at D = 64: one word per row
      kw[u][0][0] = lds32(tile[u] + lane * 4);
      kw[u][1][0] = lds32(tile[u] + 128 + lane * 4);
    }
    sz[u] = lds128(tile[u] + SZOFF + (lane >> 2) * 16);
  }
  int ahi[NT][4], alo[NT][4];
#pragma unroll
  for (int u = 0; u < NT; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) ahi[u][i] = alo[u][i] = 0;
#pragma unroll
  for (int kk = 0; kk < NKK; ++kk) {
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      if constexpr (BITS == 4) {
        const uint32_t w0 = kw[u][0][kk], w1 = kw[u][1][kk];
        qk_block<D>(ahi[u], alo[u], w0 & 0x0F0F0F0Fu, w1 & 0x0F0F0F0Fu, (w0 >> 4) & 0x0F0F0F0Fu,
                    (w1 >> 4) & 0x0F0F0F0Fu, qf, kk);
      } else {   // crumbs 2(kk % 2) and 2(kk % 2) + 1 of word kk / 2: the two 16-dim halves of block kk
        const int sh = 4 * (kk & 1);
        const uint32_t w0 = kw[u][0][kk >> 1] >> sh, w1 = kw[u][1][kk >> 1] >> sh;
        qk_block<D>(ahi[u], alo[u], w0 & 0x03030303u, w1 & 0x03030303u, (w0 >> 2) & 0x03030303u,
                    (w1 >> 2) & 0x03030303u, qf, kk);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    float acc2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc2[i] = static_cast<float>(ahi[u][i] * 256 + alo[u][i]);
    const float sKg = half_lo(sz[u].x) * qf.kscale, zKg = half_hi(sz[u].x);
    const float sKg8 = half_lo(sz[u].y) * qf.kscale, zKg8 = half_hi(sz[u].y);
    x[u][0] = fmaf(acc2[0], sKg, zKg * qf.qs0);
    x[u][1] = fmaf(acc2[1], sKg, zKg * qf.qs1);
    x[u][2] = fmaf(acc2[2], sKg8, zKg8 * qf.qs0);
    x[u][3] = fmaf(acc2[3], sKg8, zKg8 * qf.qs1);
    if constexpr (MASKED && CAUSAL) {
      if (!(valid[u] & 1)) x[u][0] = NEG_INF;
      if (!(valid[u] & 2)) x[u][1] = NEG_INF;
      if (!(valid[u] & 4)) x[u][2] = NEG_INF;
      if (!(valid[u] & 8)) x[u][3] = NEG_INF;
    } else if constexpr (MASKED) {
      if (!(valid[u] & 1)) { x[u][0] = NEG_INF; x[u][1] = NEG_INF; }
      if (!(valid[u] & 4)) { x[u][2] = NEG_INF; x[u][3] = NEG_INF; }
    }
  }
  // online softmax over the unit.  The running max only moves when some score
  // exceeds it: vote first, and reduce over the 8 row groups and rescale only then.
  float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
  for (int u = 1; u < NT; ++u) {
    mx0 = fmaxf(mx0, fmaxf(x[u][0], x[u][2]));
    mx1 = fmaxf(mx1, fmaxf(x[u][1], x[u][3]));
  }
  if (__any_sync(0xffffffffu, mx0 > ws.m0 || mx1 > ws.m1)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float n0 = fmaxf(ws.m0, mx0), n1 = fmaxf(ws.m1, mx1);
    // causal: a column with no visible position so far keeps m = -inf and a zero state
    const float a0 = (CAUSAL && n0 == NEG_INF) ? 1.f : ex2(ws.m0 - n0);
    const float a1 = (CAUSAL && n1 == NEG_INF) ? 1.f : ex2(ws.m1 - n1);
    ws.l0 *= a0; ws.l1 *= a1; ws.z0 *= a0; ws.z1 *= a1;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      ws.o[m][0] *= a0; ws.o[m][1] *= a1; ws.o[m][2] *= a0; ws.o[m][3] *= a1;
    }
    ws.m0 = n0; ws.m1 = n1;
  }
  const float mu0 = (CAUSAL && ws.m0 == NEG_INF) ? 0.f : ws.m0;
  const float mu1 = (CAUSAL && ws.m1 == NEG_INF) ? 0.f : ws.m1;
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    const float p0 = ex2(x[u][0] - mu0), p1 = ex2(x[u][1] - mu1);
    const float p2 = ex2(x[u][2] - mu0), p3 = ex2(x[u][3] - mu1);
    const float sVg = half_lo(sz[u].z), sVg8 = half_lo(sz[u].w);
    const float zVg = fmaf(VCENTRE, sVg, half_hi(sz[u].z)), zVg8 = fmaf(VCENTRE, sVg8, half_hi(sz[u].w));   // centred
    float P0 = p0 * sVg, P1 = p1 * sVg, P2 = p2 * sVg8, P3 = p3 * sVg8;
    float zg0 = p0 * zVg, zg1 = p1 * zVg, zg80 = p2 * zVg8, zg81 = p3 * zVg8;
    if constexpr (MASKED && CAUSAL) {   // unwritten slots may hold non-finite scales
      if (!(valid[u] & 1)) { P0 = 0.f; zg0 = 0.f; }
      if (!(valid[u] & 2)) { P1 = 0.f; zg1 = 0.f; }
      if (!(valid[u] & 4)) { P2 = 0.f; zg80 = 0.f; }
      if (!(valid[u] & 8)) { P3 = 0.f; zg81 = 0.f; }
    } else if constexpr (MASKED) {
      if (!(valid[u] & 1)) { P0 = 0.f; P1 = 0.f; zg0 = 0.f; zg1 = 0.f; }
      if (!(valid[u] & 4)) { P2 = 0.f; P3 = 0.f; zg80 = 0.f; zg81 = 0.f; }
    }
    ws.l0 += p0 + p2; ws.l1 += p1 + p3;
    ws.z0 += zg0 + zg80; ws.z1 += zg1 + zg81;
    uint32_t B0, B1, C0, C1;
    pv_operands(P0, P1, P2, P3, cs.part0, cs.part1, cs.colsplit, B0, B1, C0, C1);
    if (u == NT - 1) {
      // last tile: load its V codes, then hand the stage(s) back before the math
      const uint32_t t = tile[u];
      uint32_t vw[D / 16];
      load_v_words<D, BITS>(t, lane, vw);
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < NT; ++k)
          if (k == 0 || eb[k] != eb[k - 1]) mbar_arrive(eb[k]);
      }
#pragma unroll
      for (int m = 0; m < D / 16; ++m) {
        uint32_t a0, a1, a2, a3;
        v_operands<BITS>(vw, m, a0, a1, a2, a3);
        mma_f16(ws.o[m], a0, a1, a2, a3, B0, B1);
        if (!cs.colsplit) mma_f16(ws.o[m], a0, a1, a2, a3, C0, C1);
      }
    } else {
      pv_int4<D, BITS>(tile[u], ws, lane, B0, B1, C0, C1, cs.colsplit);
    }
  }
}

// ---------------------------------------------------------------------------
// Paired columns: one query token and at most 4 query heads per KV head.
// Column 2c of the 16x8x32 score multiply holds the high byte of query head c,
// column 2c+1 its low byte, both signed (q = 256 hi + lo, |q| < 2^14), so one
// integer multiply per 32 dims gives both planes and lane (g, t) ends up with
// the two partial sums of head t for tokens g and g+8.  Each lane then owns
// head t alone through the softmax (m0, l0, z0 of WarpState), with no score
// handled twice.  The P.V weights pair the same way: column 2t carries
// fp16(P), column 2t+1 fp16(P - fp16(P)), and one 16x8x16 multiply per 16 dims
// accumulates both; o[m][0] + o[m][1] (dim 16m+g) and o[m][2] + o[m][3]
// (dim 16m+g+8) is head t's sum at the end of a segment.

// Online-softmax update of head t with the scores of n tokens (x[i], -inf for
// a token outside the range; every unit holds at least one visible token).
template <int D, int N>
__device__ __forceinline__ void softmax_pc(WarpState<D>& ws, const float (&x)[N], float (&pr)[N]) {
  float mx = x[0];
#pragma unroll
  for (int i = 1; i < N; ++i) mx = fmaxf(mx, x[i]);
  if (__any_sync(0xffffffffu, mx > ws.m0)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float n0 = fmaxf(ws.m0, mx);
    const float a0 = ex2(ws.m0 - n0);
    ws.l0 *= a0; ws.z0 *= a0;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) { ws.o[m][0] *= a0; ws.o[m][1] *= a0; ws.o[m][2] *= a0; ws.o[m][3] *= a0; }
    ws.m0 = n0;
  }
#pragma unroll
  for (int i = 0; i < N; ++i) pr[i] = ex2(x[i] - ws.m0);
}

// P.V weights of head t for tokens g and g+8 as the B fragments of one 16x8x16 multiply (fp16 P in
// column 2t, the fp16 remainder in column 2t+1).
__device__ __forceinline__ void pv_operands_pc(float P0, float P1, uint32_t& B0, uint32_t& B1) {
  const uint32_t h = pack_half2(P0, P1);
  const uint32_t l = pack_half2(P0 - half_lo(h), P1 - half_hi(h));
  B0 = movmatrix_trans(__byte_perm(h, l, 0x5410));   // token g: (hi, lo)
  B1 = movmatrix_trans(__byte_perm(h, l, 0x7632));   // token g+8
}

// Scores of head t from the paired integer sums, the zero point folded in.
__device__ __forceinline__ float score_pc(int hi, int lo, uint32_t szk, float kscale, float qs) {
  return fmaf(static_cast<float>(hi * 256 + lo), half_lo(szk) * kscale, half_hi(szk) * qs);
}

// unit_int4 with paired columns (one query token).  valid[u]: bit 0 token g,
// bit 2 token g+8 of tile u inside the range being read (MASKED).
template <int D, int NT, bool MASKED, int BITS = 4>
__device__ __forceinline__ void unit_int4_pc(const uint32_t* tile, const QFrag<D>& qf, WarpState<D>& ws, int lane,
                                             const int* valid, const uint32_t* eb) {
  static_assert(BITS == 4 || BITS == 2, "code width");
  constexpr int SZOFF = BITS == 4 ? 16 * D : 8 * D;
  constexpr float VCENTRE = BITS == 4 ? 8.f : 2.f;
  constexpr int NKK = D / 32;
  uint32_t kw[NT][2][NKK];
  uint4 sz[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    if constexpr (BITS == 4 && D == 128) {
      const uint4 a = lds128(tile[u] + lane * 16), bq = lds128(tile[u] + 512 + lane * 16);
      kw[u][0][0] = a.x; kw[u][0][1] = a.y; kw[u][0][2] = a.z; kw[u][0][3] = a.w;
      kw[u][1][0] = bq.x; kw[u][1][1] = bq.y; kw[u][1][2] = bq.z; kw[u][1][3] = bq.w;
    } else if constexpr (BITS == 4 || D == 128) {
      const uint2 a = lds64(tile[u] + lane * 8), bq = lds64(tile[u] + 256 + lane * 8);
      kw[u][0][0] = a.x; kw[u][0][1] = a.y; kw[u][1][0] = bq.x; kw[u][1][1] = bq.y;
    } else {
      kw[u][0][0] = lds32(tile[u] + lane * 4);
      kw[u][1][0] = lds32(tile[u] + 128 + lane * 4);
    }
    sz[u] = lds128(tile[u] + SZOFF + (lane >> 2) * 16);
  }
  int acc[NT][4];
#pragma unroll
  for (int u = 0; u < NT; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[u][i] = 0;
#pragma unroll
  for (int kk = 0; kk < NKK; ++kk) {
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      if constexpr (BITS == 4) {
        const uint32_t w0 = kw[u][0][kk], w1 = kw[u][1][kk];
        imma_u8s8(acc[u], w0 & 0x0F0F0F0Fu, w1 & 0x0F0F0F0Fu, (w0 >> 4) & 0x0F0F0F0Fu, (w1 >> 4) & 0x0F0F0F0Fu,
                  qf.b[kk][0], qf.b[kk][1]);
      } else {
        const int sh = 4 * (kk & 1);
        const uint32_t w0 = kw[u][0][kk >> 1] >> sh, w1 = kw[u][1][kk >> 1] >> sh;
        imma_u8s8(acc[u], w0 & 0x03030303u, w1 & 0x03030303u, (w0 >> 2) & 0x03030303u, (w1 >> 2) & 0x03030303u,
                  qf.b[kk][0], qf.b[kk][1]);
      }
    }
  }
  float x[2 * NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    x[2 * u] = score_pc(acc[u][0], acc[u][1], sz[u].x, qf.kscale, qf.qs0);
    x[2 * u + 1] = score_pc(acc[u][2], acc[u][3], sz[u].y, qf.kscale, qf.qs0);
    if constexpr (MASKED) {
      if (!(valid[u] & 1)) x[2 * u] = NEG_INF;
      if (!(valid[u] & 4)) x[2 * u + 1] = NEG_INF;
    }
  }
  float pr[2 * NT];
  softmax_pc<D, 2 * NT>(ws, x, pr);
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    const float p0 = pr[2 * u], p1 = pr[2 * u + 1];
    const float sVg = half_lo(sz[u].z), sVg8 = half_lo(sz[u].w);
    const float zVg = fmaf(VCENTRE, sVg, half_hi(sz[u].z)), zVg8 = fmaf(VCENTRE, sVg8, half_hi(sz[u].w));   // centred
    float P0 = p0 * sVg, P1 = p1 * sVg8;
    float zg = p0 * zVg, zg8 = p1 * zVg8;
    if constexpr (MASKED) {   // unwritten slots may hold non-finite scales
      if (!(valid[u] & 1)) { P0 = 0.f; zg = 0.f; }
      if (!(valid[u] & 4)) { P1 = 0.f; zg8 = 0.f; }
    }
    ws.l0 += p0 + p1;
    ws.z0 += zg + zg8;
    uint32_t B0, B1;
    pv_operands_pc(P0, P1, B0, B1);
    uint32_t vw[D / 16];
    load_v_words<D, BITS>(tile[u], lane, vw);
    if (u == NT - 1) {
      // the last V loads are done: hand the stage(s) back before the math
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < NT; ++k)
          if (k == 0 || eb[k] != eb[k - 1]) mbar_arrive(eb[k]);
      }
    }
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      uint32_t a0, a1, a2, a3;
      v_operands<BITS>(vw, m, a0, a1, a2, a3);
      mma_f16(ws.o[m], a0, a1, a2, a3, B0, B1);
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 pages ("KV Cache Quantization" topic page, item 3: NVFP4 storage of
// the paged KV cache).  A tile holds E2M1 codes and one E4M3 scale per token
// and 16 dims.  Both products run on 16x8x16 fp16 multiplies: the hardware
// conversion turns each code byte into an fp16 pair, and the block scale
// multiplies it exactly (e2m1 * e4m3 has at most 5 significant bits and stays
// in the normal fp16 range), so the operands are the dequantized values
// themselves.  The query is the fp16 fragment form (q * 2^e, exact for bf16
// values): block b of the K operand holds dims 16b + 4t, 4t+1 (k 2t, 2t+1) and
// 4t+2, 4t+3 (k 2t+8, 2t+9), and the query fragments use the same order.

// The four E2M1 pairs of a word (byte i: its low nibble -> low half) as fp16x2.
__device__ __forceinline__ void e2m1x8_to_half2(uint32_t w, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                uint32_t& r3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(w));
}
// Two E4M3 bytes (bits 0-7 -> low half, 8-15 -> high half) as fp16x2.
__device__ __forceinline__ uint32_t e4m3x2_to_half2(uint32_t w) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(static_cast<uint16_t>(w & 0xFFFFu)));
  return r;
}
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
// (lo, lo) and (hi, hi) of a half2.
__device__ __forceinline__ uint32_t half2_lolo(uint32_t x) { return __byte_perm(x, 0u, 0x1010); }
__device__ __forceinline__ uint32_t half2_hihi(uint32_t x) { return __byte_perm(x, 0u, 0x3232); }

// One unit of NT NVFP4 tiles at shared addresses tile[0 .. NT-1]: as unit_int4
// (valid[] the same visibility bits), without zero points.  nwr[u]: slots of
// tile u that hold written tokens (the rest may hold non-finite scales, which
// must not reach the P.V operands); used when MASKED.
template <int D, int NT, bool MASKED, bool CAUSAL = false>
__device__ __forceinline__ void unit_fp4(const uint32_t* tile, const QFrag<D>& qf, WarpState<D>& ws, int lane,
                                         const int* valid, const int* nwr, const uint32_t* eb, const ColSplit& cs) {
  constexpr int NB = D / 16;
  const int g8 = lane >> 2, t = lane & 3;
  float x[NT][4];
  uint32_t kw[NT][NB];
  uint32_t ks[NT][NB / 2];   // K scale pairs (token g, token g+8) of blocks 2i (bits 0-15) and 2i+1
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    if constexpr (D == 128) {
      const uint4 a = lds128(tile[u] + lane * 16), b = lds128(tile[u] + 512 + lane * 16);
      kw[u][0] = a.x; kw[u][1] = a.y; kw[u][2] = a.z; kw[u][3] = a.w;
      kw[u][4] = b.x; kw[u][5] = b.y; kw[u][6] = b.z; kw[u][7] = b.w;
      const uint4 sc = lds128(tile[u] + 16 * D + 16 * g8);
      ks[u][0] = sc.x; ks[u][1] = sc.y; ks[u][2] = sc.z; ks[u][3] = sc.w;
    } else {
      const uint4 a = lds128(tile[u] + lane * 16);
      kw[u][0] = a.x; kw[u][1] = a.y; kw[u][2] = a.z; kw[u][3] = a.w;
      const uint2 sc = lds64(tile[u] + 16 * D + 8 * g8);
      ks[u][0] = sc.x; ks[u][1] = sc.y;
    }
  }
  float acc[NT][4];
#pragma unroll
  for (int u = 0; u < NT; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[u][i] = 0.f;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      uint32_t a0, a1, a2, a3;   // (token g | g+8) x (dims 4t, 4t+1 | 4t+2, 4t+3) of block b
      e2m1x8_to_half2(kw[u][b], a0, a1, a2, a3);
      const uint32_t s2 = e4m3x2_to_half2(ks[u][b >> 1] >> (16 * (b & 1)));
      const uint32_t sg = half2_lolo(s2), sg8 = half2_hihi(s2);
      mma_f16(acc[u], hmul2_u(a0, sg), hmul2_u(a1, sg8), hmul2_u(a2, sg), hmul2_u(a3, sg8), qf.b[b][0],
              qf.b[b][1]);
    }
  }
#pragma unroll
  for (int u = 0; u < NT; ++u) {
#pragma unroll
    for (int i = 0; i < 4; ++i) x[u][i] = acc[u][i] * qf.kscale;
    if constexpr (MASKED && CAUSAL) {
      if (!(valid[u] & 1)) x[u][0] = NEG_INF;
      if (!(valid[u] & 2)) x[u][1] = NEG_INF;
      if (!(valid[u] & 4)) x[u][2] = NEG_INF;
      if (!(valid[u] & 8)) x[u][3] = NEG_INF;
    } else if constexpr (MASKED) {
      if (!(valid[u] & 1)) { x[u][0] = NEG_INF; x[u][1] = NEG_INF; }
      if (!(valid[u] & 4)) { x[u][2] = NEG_INF; x[u][3] = NEG_INF; }
    }
  }
  // online softmax over the unit (as unit_int4)
  float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
  for (int u = 1; u < NT; ++u) {
    mx0 = fmaxf(mx0, fmaxf(x[u][0], x[u][2]));
    mx1 = fmaxf(mx1, fmaxf(x[u][1], x[u][3]));
  }
  if (__any_sync(0xffffffffu, mx0 > ws.m0 || mx1 > ws.m1)) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float n0 = fmaxf(ws.m0, mx0), n1 = fmaxf(ws.m1, mx1);
    const float a0 = (CAUSAL && n0 == NEG_INF) ? 1.f : ex2(ws.m0 - n0);
    const float a1 = (CAUSAL && n1 == NEG_INF) ? 1.f : ex2(ws.m1 - n1);
    ws.l0 *= a0; ws.l1 *= a1;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      ws.o[m][0] *= a0; ws.o[m][1] *= a1; ws.o[m][2] *= a0; ws.o[m][3] *= a1;
    }
    ws.m0 = n0; ws.m1 = n1;
  }
  const float mu0 = (CAUSAL && ws.m0 == NEG_INF) ? 0.f : ws.m0;
  const float mu1 = (CAUSAL && ws.m1 == NEG_INF) ? 0.f : ws.m1;
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    float P0 = ex2(x[u][0] - mu0), P1 = ex2(x[u][1] - mu1);
    float P2 = ex2(x[u][2] - mu0), P3 = ex2(x[u][3] - mu1);
    if constexpr (MASKED && CAUSAL) {
      if (!(valid[u] & 1)) P0 = 0.f;
      if (!(valid[u] & 2)) P1 = 0.f;
      if (!(valid[u] & 4)) P2 = 0.f;
      if (!(valid[u] & 8)) P3 = 0.f;
    } else if constexpr (MASKED) {
      if (!(valid[u] & 1)) { P0 = 0.f; P1 = 0.f; }
      if (!(valid[u] & 4)) { P2 = 0.f; P3 = 0.f; }
    }
    ws.l0 += P0 + P2; ws.l1 += P1 + P3;
    uint32_t B0, B1, C0, C1;
    pv_operands(P0, P1, P2, P3, cs.part0, cs.part1, cs.colsplit, B0, B1, C0, C1);
    // V: the word of lane 4g + t and dim block m holds (dims g, g + 8) x (tokens 2t, 2t+1 | 2t+8, 2t+9);
    // the scales of those tokens in block m are the 4 bytes at 17D + (D/4) t + 4m
    const uint32_t tv = tile[u];
    uint32_t vw[NB], vs[NB];
    if constexpr (D == 128) {
      const uint4 v0 = lds128(tv + 8 * D + lane * 16), v1 = lds128(tv + 8 * D + 512 + lane * 16);
      vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
      vw[4] = v1.x; vw[5] = v1.y; vw[6] = v1.z; vw[7] = v1.w;
      const uint4 s0 = lds128(tv + 17 * D + (D / 4) * t), s1 = lds128(tv + 17 * D + (D / 4) * t + 16);
      vs[0] = s0.x; vs[1] = s0.y; vs[2] = s0.z; vs[3] = s0.w;
      vs[4] = s1.x; vs[5] = s1.y; vs[6] = s1.z; vs[7] = s1.w;
    } else {
      const uint4 v0 = lds128(tv + 8 * D + lane * 16);
      vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
      const uint4 s0 = lds128(tv + 17 * D + (D / 4) * t);
      vs[0] = s0.x; vs[1] = s0.y; vs[2] = s0.z; vs[3] = s0.w;
    }
    if (u == NT - 1) {   // the last loads of the unit are done: hand the stage(s) back
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < NT; ++k)
          if (k == 0 || eb[k] != eb[k - 1]) mbar_arrive(eb[k]);
      }
    }
    if constexpr (MASKED) {
      // unwritten slots (>= nwr[u]) may hold non-finite scales: zero them (their weights are zero)
      const int n = nwr[u];
      const uint32_t keep = (2 * t < n ? 0x000000FFu : 0u) | (2 * t + 1 < n ? 0x0000FF00u : 0u) |
                            (2 * t + 8 < n ? 0x00FF0000u : 0u) | (2 * t + 9 < n ? 0xFF000000u : 0u);
#pragma unroll
      for (int m = 0; m < NB; ++m) vs[m] &= keep;
    }
#pragma unroll
    for (int m = 0; m < NB; ++m) {
      uint32_t a0, a1, a2, a3;   // (dim g | g+8) x (tokens 2t, 2t+1 | 2t+8, 2t+9)
      e2m1x8_to_half2(vw[m], a0, a1, a2, a3);
      const uint32_t s01 = e4m3x2_to_half2(vs[m]), s89 = e4m3x2_to_half2(vs[m] >> 16);
      a0 = hmul2_u(a0, s01); a1 = hmul2_u(a1, s01); a2 = hmul2_u(a2, s89); a3 = hmul2_u(a3, s89);
      mma_f16(ws.o[m], a0, a1, a2, a3, B0, B1);
      if (!cs.colsplit) mma_f16(ws.o[m], a0, a1, a2, a3, C0, C1);
    }
  }
}

// One INT8 tile (protected store).
// HQ: the query operand holds fp16 B fragments (the cache's pages are NVFP4, see unit_fp4); the K
// codes then enter 16x8x16 fp16 multiplies as c - 128 (exact), the zero point as z + 128 s.
template <int D, bool MASKED, bool CAUSAL = false, bool HQ = false>
__device__ __forceinline__ void tile_int8(uint32_t st, const QFrag<D>& qf, WarpState<D>& ws, int lane, int vm,
                                          uint32_t empty_bar, const ColSplit& cs) {
  constexpr int NK = D / 16;
  uint32_t kw[2][NK], vw[2 * NK];
  // K: per row (g, g+8) D/4 bytes at (D/4)*lane; word 2kk + hf holds dims 32kk + 16hf + 4t .. +3
#pragma unroll
  for (int rowhi = 0; rowhi < 2; ++rowhi)
#pragma unroll
    for (int kq = 0; kq < D / 64; ++kq) {
      const uint4 a = lds128(st + rowhi * 8 * D + (D / 4) * lane + 16 * kq);
      kw[rowhi][4 * kq] = a.x; kw[rowhi][4 * kq + 1] = a.y; kw[rowhi][4 * kq + 2] = a.z; kw[rowhi][4 * kq + 3] = a.w;
    }
#pragma unroll
  for (int q4 = 0; q4 < NK / 2; ++q4) {
    const uint4 a = lds128(st + 16 * D + 16 * (32 * q4 + lane));
    vw[4 * q4] = a.x; vw[4 * q4 + 1] = a.y; vw[4 * q4 + 2] = a.z; vw[4 * q4 + 3] = a.w;
  }
  const uint4 sz = lds128(st + 32 * D + (lane >> 2) * 16);
  __syncwarp();
  if (lane == 0) mbar_arrive(empty_bar);
  float acc[4];
  if constexpr (HQ) {
    // word k of a row holds dims 16k + 4t .. 16k + 4t + 3: the fp16 fragments' dim order
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = 0.f;
#pragma unroll
    for (int k = 0; k < NK; ++k)
      mma_f16(acc, bytes01_c(kw[0][k]), bytes01_c(kw[1][k]), bytes23_c(kw[0][k]), bytes23_c(kw[1][k]), qf.b[k][0],
              qf.b[k][1]);
  } else {
    int ahi[4] = {0, 0, 0, 0}, alo[4] = {0, 0, 0, 0};
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk)
      qk_block<D>(ahi, alo, kw[0][2 * kk], kw[1][2 * kk], kw[0][2 * kk + 1], kw[1][2 * kk + 1], qf, kk);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = static_cast<float>(ahi[i] * 256 + alo[i]);
  }
  const float sKg = half_lo(sz.x) * qf.kscale, sKg8 = half_lo(sz.y) * qf.kscale;
  const float zKg = HQ ? fmaf(128.f, half_lo(sz.x), half_hi(sz.x)) : half_hi(sz.x);
  const float zKg8 = HQ ? fmaf(128.f, half_lo(sz.y), half_hi(sz.y)) : half_hi(sz.y);
  float x0 = fmaf(acc[0], sKg, zKg * qf.qs0);
  float x1 = fmaf(acc[1], sKg, zKg * qf.qs1);
  float x2 = fmaf(acc[2], sKg8, zKg8 * qf.qs0);
  float x3 = fmaf(acc[3], sKg8, zKg8 * qf.qs1);
  if constexpr (MASKED && CAUSAL) {   // vm: the visibility bits of unit_int4's valid[]
    if (!(vm & 1)) x0 = NEG_INF;
    if (!(vm & 2)) x1 = NEG_INF;
    if (!(vm & 4)) x2 = NEG_INF;
    if (!(vm & 8)) x3 = NEG_INF;
  } else if constexpr (MASKED) {
    if (!(vm & 1)) { x0 = NEG_INF; x1 = NEG_INF; }
    if (!(vm & 4)) { x2 = NEG_INF; x3 = NEG_INF; }
  }
  float p0, p1, p2, p3;
  online_softmax_pv<D, CAUSAL>(ws, x0, x1, x2, x3, p0, p1, p2, p3);
  const float sVg = half_lo(sz.z), sVg8 = half_lo(sz.w);
  const float zVg = fmaf(128.f, sVg, half_hi(sz.z)), zVg8 = fmaf(128.f, sVg8, half_hi(sz.w));   // centred codes
  float P0 = p0 * sVg, P1 = p1 * sVg, P2 = p2 * sVg8, P3 = p3 * sVg8;
  float zg0 = p0 * zVg, zg1 = p1 * zVg, zg80 = p2 * zVg8, zg81 = p3 * zVg8;
  if constexpr (MASKED && CAUSAL) {
    if (!(vm & 1)) { P0 = 0.f; zg0 = 0.f; }
    if (!(vm & 2)) { P1 = 0.f; zg1 = 0.f; }
    if (!(vm & 4)) { P2 = 0.f; zg80 = 0.f; }
    if (!(vm & 8)) { P3 = 0.f; zg81 = 0.f; }
  } else if constexpr (MASKED) {
    if (!(vm & 1)) { P0 = 0.f; P1 = 0.f; zg0 = 0.f; zg1 = 0.f; }
    if (!(vm & 4)) { P2 = 0.f; P3 = 0.f; zg80 = 0.f; zg81 = 0.f; }
  }
  ws.l0 += p0 + p2; ws.l1 += p1 + p3;
  ws.z0 += zg0 + zg80; ws.z1 += zg1 + zg81;
  uint32_t B0, B1, C0, C1;
  pv_operands(P0, P1, P2, P3, cs.part0, cs.part1, cs.colsplit, B0, B1, C0, C1);
#pragma unroll
  for (int m = 0; m < NK; ++m) {
    const uint32_t w0 = vw[2 * m], w1 = vw[2 * m + 1];
    const uint32_t a0 = byte_lo_c(w0), a1 = byte_lo_c(w0 >> 8), a2 = byte_lo_c(w1), a3 = byte_lo_c(w1 >> 8);
    mma_f16(ws.o[m], a0, a1, a2, a3, B0, B1);
    if (!cs.colsplit) mma_f16(ws.o[m], a0, a1, a2, a3, C0, C1);
  }
}

// tile_int8 with paired columns (one query token, integer query planes).  vm:
// bit 0 token g, bit 2 token g+8 inside the protected range (MASKED).
template <int D, bool MASKED>
__device__ __forceinline__ void tile_int8_pc(uint32_t st, const QFrag<D>& qf, WarpState<D>& ws, int lane, int vm,
                                             uint32_t empty_bar) {
  constexpr int NK = D / 16;
  uint32_t kw[2][NK], vw[2 * NK];
#pragma unroll
  for (int rowhi = 0; rowhi < 2; ++rowhi)
#pragma unroll
    for (int kq = 0; kq < D / 64; ++kq) {
      const uint4 a = lds128(st + rowhi * 8 * D + (D / 4) * lane + 16 * kq);
      kw[rowhi][4 * kq] = a.x; kw[rowhi][4 * kq + 1] = a.y; kw[rowhi][4 * kq + 2] = a.z; kw[rowhi][4 * kq + 3] = a.w;
    }
#pragma unroll
  for (int q4 = 0; q4 < NK / 2; ++q4) {
    const uint4 a = lds128(st + 16 * D + 16 * (32 * q4 + lane));
    vw[4 * q4] = a.x; vw[4 * q4 + 1] = a.y; vw[4 * q4 + 2] = a.z; vw[4 * q4 + 3] = a.w;
  }
  const uint4 sz = lds128(st + 32 * D + (lane >> 2) * 16);
  __syncwarp();
  if (lane == 0) mbar_arrive(empty_bar);
  int acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int kk = 0; kk < D / 32; ++kk)
    imma_u8s8(acc, kw[0][2 * kk], kw[1][2 * kk], kw[0][2 * kk + 1], kw[1][2 * kk + 1], qf.b[kk][0], qf.b[kk][1]);
  float x[2] = {score_pc(acc[0], acc[1], sz.x, qf.kscale, qf.qs0), score_pc(acc[2], acc[3], sz.y, qf.kscale, qf.qs0)};
  if constexpr (MASKED) {
    if (!(vm & 1)) x[0] = NEG_INF;
    if (!(vm & 4)) x[1] = NEG_INF;
  }
  float pr[2];
  softmax_pc<D, 2>(ws, x, pr);
  const float sVg = half_lo(sz.z), sVg8 = half_lo(sz.w);
  const float zVg = fmaf(128.f, sVg, half_hi(sz.z)), zVg8 = fmaf(128.f, sVg8, half_hi(sz.w));   // centred codes
  float P0 = pr[0] * sVg, P1 = pr[1] * sVg8;
  float zg = pr[0] * zVg, zg8 = pr[1] * zVg8;
  if constexpr (MASKED) {
    if (!(vm & 1)) { P0 = 0.f; zg = 0.f; }
    if (!(vm & 4)) { P1 = 0.f; zg8 = 0.f; }
  }
  ws.l0 += pr[0] + pr[1];
  ws.z0 += zg + zg8;
  uint32_t B0, B1;
  pv_operands_pc(P0, P1, B0, B1);
#pragma unroll
  for (int m = 0; m < NK; ++m) {
    const uint32_t w0 = vw[2 * m], w1 = vw[2 * m + 1];
    mma_f16(ws.o[m], byte_lo_c(w0), byte_lo_c(w0 >> 8), byte_lo_c(w1), byte_lo_c(w1 >> 8), B0, B1);
  }
}

// One BF16 tile (baseline cache).  Holds the stage until the V loads are done.
// vmask01 / vmask89: per-thread masks of the V operand halves of tokens 2t, 2t+1
// and 2t+8, 2t+9 (unwritten slots of a page may hold NaN bit patterns, and
// 0 * NaN would poison the accumulator).
template <int D, bool MASKED>
__device__ __forceinline__ void tile_bf16(uint32_t st, const QFrag<D>& qf, WarpState<D>& ws, int lane, bool vg,
                                          bool vg8, uint32_t empty_bar, uint32_t vmask01, uint32_t vmask89) {
  constexpr int NK = D / 16;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < NK; ++k) {
    const uint4 a = lds128(st + 16 * (32 * k + lane));
    mma_bf16(acc, a.x, a.y, a.z, a.w, qf.b[k][0], qf.b[k][1]);
  }
  uint4 v[NK];
#pragma unroll
  for (int m = 0; m < NK; ++m) {
    v[m] = lds128(st + 32 * D + 16 * (32 * m + lane));
    if constexpr (MASKED) {
      v[m].x &= vmask01; v[m].y &= vmask01; v[m].z &= vmask89; v[m].w &= vmask89;
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(empty_bar);
  float x0 = acc[0] * qf.kscale, x1 = acc[1] * qf.kscale, x2 = acc[2] * qf.kscale, x3 = acc[3] * qf.kscale;
  if constexpr (MASKED) {
    if (!vg) { x0 = NEG_INF; x1 = NEG_INF; }
    if (!vg8) { x2 = NEG_INF; x3 = NEG_INF; }
  }
  float p0, p1, p2, p3;
  online_softmax_pv<D>(ws, x0, x1, x2, x3, p0, p1, p2, p3);
  ws.l0 += p0 + p2; ws.l1 += p1 + p3;
  const uint32_t B0 = movmatrix_trans(pack_bf162(p0, p1));
  const uint32_t B1 = movmatrix_trans(pack_bf162(p2, p3));
#pragma unroll
  for (int m = 0; m < NK; ++m) mma_bf16(ws.o[m], v[m].x, v[m].y, v[m].z, v[m].w, B0, B1);
}


// Rotated queries of one (sequence, KV head) as 16x8x16 B operands, written to
// qblob[b * Hkv + h]: fp32 FWHT (same order as the append), bf16 rounding, then
// fp16 with a power-of-two scale (INT4 cache) or plain bf16 (BF16 cache); the
// tail holds sigma*log2(e)*sum(q) per column and the key scale factor.
// sq: shared scratch of G*D floats for this warp.
template <int D>
__device__ __forceinline__ void load_qfrag(const AttnParams& p, int b, int h, int lane, QFrag<D>& qf,
                                           int L_known = -1);
template <int D>
__device__ __forceinline__ void store_qblob(uint8_t* blob, const QFrag<D>& qf, int lane, bool paired);

template <int D, bool BF16>
__device__ __forceinline__ void build_qblob(const AttnParams& p, int b, int h, int lane, float* sq) {
  constexpr int VPL = D / 32;
  const int G = p.G;
  const int gw = b * p.Hkv + h;
  if constexpr (!BF16) {   // INT4/INT8 caches: the integer query planes
    QFrag<D> qf;
    load_qfrag<D>(p, b, h, lane, qf);
    store_qblob<D>(p.qblob + static_cast<size_t>(gw) * qblob_bytes(D), qf, lane, p.qfmt == 3);
    return;
  }
  float qsum[MAX_G];
  float amax = 0.f;
  const float rot_c = p.rot_c;
  for (int g = 0; g < G; ++g) {
    const uint16_t* src = p.q + q_row(p, b, h, g) * D;
    float x[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) x[i] = __bfloat162float(__ushort_as_bfloat16(src[VPL * lane + i]));
    if constexpr (!BF16) {
      fwht_row<VPL>(x, p.Bh, lane);
#pragma unroll
      for (int i = 0; i < VPL; ++i) x[i] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(x[i], rot_c)));
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      sq[g * D + VPL * lane + i] = x[i];
      s += x[i];
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    qsum[g] = s;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __syncwarp();
  // fp16 operands: q * 2^e with max|q| * 2^e in [2^14, 2^15) (exact for normal values)
  int e = 0;
  if (!BF16 && amax > 0.f && amax <= 3.0e38f) {
    int ex;
    frexpf(amax, &ex);
    e = 15 - ex;
  }
  uint32_t* blob = reinterpret_cast<uint32_t*>(p.qblob + static_cast<size_t>(gw) * qblob_bytes(D));
  const int g = lane >> 2, t = lane & 3;
  // B-operand column n holds query head n % G when the column split applies
  // (G = 1, 2, 4: the spare columns carry the low part of the P.V weights),
  // otherwise head n for n < G and zeros.
  const bool colsplit = (G == 1 || G == 2 || G == 4);
  const int gsrc = colsplit ? g % G : g;
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[4];
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int k = 2 * c + kk;
#pragma unroll
      for (int reg = 0; reg < 2; ++reg) {
        const int d = 16 * k + 2 * t + 8 * reg;
        float a = 0.f, bb = 0.f;
        if (gsrc < G) { a = sq[gsrc * D + d]; bb = sq[gsrc * D + d + 1]; }
        if constexpr (BF16) {
          r[2 * kk + reg] = pack_bf162(a, bb);
        } else {
          r[2 * kk + reg] = pack_half2(ldexpf(a, e), ldexpf(bb, e));
        }
      }
    }
    reinterpret_cast<uint4*>(blob)[c * 32 + lane] = make_uint4(r[0], r[1], r[2], r[3]);
  }
  float* tail = reinterpret_cast<float*>(p.qblob + static_cast<size_t>(gw) * qblob_bytes(D) + 16 * D);
  if (lane < MAX_G) {
    const int src = colsplit ? lane % G : lane;
    float v = 0.f;
#pragma unroll
    for (int gg = 0; gg < MAX_G; ++gg)
      if (gg == src && gg < G) v = qsum[gg];
    tail[lane] = BF16 ? 0.f : v * p.scale_log2;
  }
  if (lane == MAX_G) tail[MAX_G] = ldexpf(p.scale_log2, -e);
}


// The query operand of KV head h of batch entry b, built straight into the
// registers of the 16x8x32 B fragments.  Lane (g8 = lane/4, t = lane%4) holds
// column g8 (query head g8 % G with the column split, else g8, zero when that
// head does not exist) at dimensions d = 32kk + 16hf + 4t + j, j < 4: dimension
// bits 0-1 (j), 4 (hf) and 5.. (kk) are in-lane, bits 2-3 are the lane bits 0-1.
// The block-diagonal Hadamard runs in ascending butterfly stages with the same
// fp32 operations as the rotation of the keys, so q_rot is the same bf16
// vector whichever lane holds it.  Then q_rot * 2^e (max |q_rot| * 2^e in
// [2^14, 2^15)) is rounded to a 16-bit integer and split into the planes
// hi = floor(q / 256) (signed byte) and lo = q mod 256 (unsigned byte).
// RoPE of a query held in the fragment layout (x[kk][hf][j] = dim 32kk + 16hf
// + 4t + j), at table row `pos`, with the arithmetic of the keys' RoPE: neox
// pairs (d, d + R/2) are 16-dim blocks SH = R/32 apart, gptj pairs (d, d + 1)
// are neighbours in j; both always sit in the same lane.
__device__ __forceinline__ void rope_turn(float& a, float& b, float c, float s) {
  const float a0 = a, b0 = b;
  a = __fsub_rn(__fmul_rn(a0, c), __fmul_rn(b0, s));
  b = __fadd_rn(__fmul_rn(b0, c), __fmul_rn(a0, s));
}

template <int NKK, int SH>
__device__ __forceinline__ void rope_qfrag_neox(float (&x)[NKK][2][4], const float* cs, int t) {
  constexpr int HALF = 16 * SH;
#pragma unroll
  for (int b1 = 0; b1 < SH; ++b1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = 16 * b1 + 4 * t + j;
      rope_turn(x[b1 >> 1][b1 & 1][j], x[(b1 + SH) >> 1][(b1 + SH) & 1][j], __ldg(cs + i), __ldg(cs + HALF + i));
    }
}

template <int NKK>
__device__ __forceinline__ void rope_qfrag(float (&x)[NKK][2][4], const RopeParams& r, int pos, int t) {
  const float* cs = r.cs + static_cast<long long>(pos) * r.R;
  if (r.style == KV4_ROPE_GPTJ) {
    const int half = r.R >> 1;
#pragma unroll
    for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int d = 32 * kk + 16 * hf + 4 * t;
        if (d < r.R) {
          const int i = d >> 1;
          rope_turn(x[kk][hf][0], x[kk][hf][1], __ldg(cs + i), __ldg(cs + half + i));
          rope_turn(x[kk][hf][2], x[kk][hf][3], __ldg(cs + i + 1), __ldg(cs + half + i + 1));
        }
      }
  } else if (r.R == 32) {
    rope_qfrag_neox<NKK, 1>(x, cs, t);
  } else if (r.R == 64) {
    rope_qfrag_neox<NKK, 2>(x, cs, t);
  } else if constexpr (NKK >= 4) {
    rope_qfrag_neox<NKK, 4>(x, cs, t);   // R = 128
  }
}

// L_known >= 0: the sequence's length, when the caller already has it (the
// RoPE position of query token i is L - qtot + i); else it is read.
template <int D>
__device__ __forceinline__ void load_qfrag(const AttnParams& p, int b, int h, int lane, QFrag<D>& qf, int L_known) {
  constexpr int NKK = D / 32;
  const int G = p.G, g8 = lane >> 2, t = lane & 3;
  const bool colsplit = (G == 1 || G == 2 || G == 4);
  const bool pc = p.qfmt == 3;   // paired columns: column g8 is plane g8 % 2 of head g8 / 2
  const int gsrc = pc ? (g8 >> 1) : (colsplit ? g8 % G : g8);
  const bool active = gsrc < G;
  const uint16_t* src = p.q + q_row(p, b, h, active ? gsrc : 0) * D + 4 * t;
  float x[NKK][2][4];
#pragma unroll
  for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint2 w = make_uint2(0u, 0u);
      if (active) w = __ldg(reinterpret_cast<const uint2*>(src + 32 * kk + 16 * hf));
      x[kk][hf][0] = __uint_as_float(w.x << 16);
      x[kk][hf][1] = __uint_as_float(w.x & 0xFFFF0000u);
      x[kk][hf][2] = __uint_as_float(w.y << 16);
      x[kk][hf][3] = __uint_as_float(w.y & 0xFFFF0000u);
    }
  if (p.rope.cs != nullptr && active) {
    // the column's query token sits at position L - qlen + i of its sequence
    int L = L_known;
    if (L < 0) {
      const int seq = p.seq_ids[b];
      L = (seq >= 0 && seq < p.max_seqs) ? p.seq_lens[seq] : 0;
    }
    int pos = max(L - p.qtot + p.q0 + gsrc / p.Gh, 0);
    if (pos >= p.rope.max_pos) {
      atomicOr(&p.state->status, KV4_DEV_ROPE_POS);
      pos = p.rope.max_pos - 1;
    }
    rope_qfrag<NKK>(x, p.rope, pos, t);
  }
  const int Bh = p.Bh_q;
  // stages 1 and 2: dimension bits 0-1 (j)
#pragma unroll
  for (int jb = 1; jb <= 2; jb <<= 1) {
    if (jb < Bh) {
#pragma unroll
      for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if ((j & jb) == 0) {
              const float a = x[kk][hf][j], c = x[kk][hf][j + jb];
              x[kk][hf][j] = __fadd_rn(a, c);
              x[kk][hf][j + jb] = __fsub_rn(a, c);
            }
    }
  }
  // stages 4 and 8: dimension bits 2-3 are the lane bits 0-1
#pragma unroll
  for (int lm = 1; lm <= 2; lm <<= 1) {
    if (4 * lm < Bh) {
      const bool upper = (t & lm) != 0;
#pragma unroll
      for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, x[kk][hf][j], lm);
            x[kk][hf][j] = upper ? __fsub_rn(o, x[kk][hf][j]) : __fadd_rn(x[kk][hf][j], o);
          }
    }
  }
  // stage 16: dimension bit 4 (hf)
  if (16 < Bh) {
#pragma unroll
    for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = x[kk][0][j], c = x[kk][1][j];
        x[kk][0][j] = __fadd_rn(a, c);
        x[kk][1][j] = __fsub_rn(a, c);
      }
  }
  // stages 32, 64, ...: dimension bits 5.. (kk)
#pragma unroll
  for (int kb = 1; kb < NKK; kb <<= 1) {
    if (32 * kb < Bh) {
#pragma unroll
      for (int kk = 0; kk < NKK; ++kk)
        if ((kk & kb) == 0)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float a = x[kk][hf][j], c = x[kk + kb][hf][j];
              x[kk][hf][j] = __fadd_rn(a, c);
              x[kk + kb][hf][j] = __fsub_rn(a, c);
            }
    }
  }
  const float rot_c = p.rc_q;
  float amax = 0.f, qs = 0.f;
#pragma unroll
  for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float v = __bfloat162float(__float2bfloat16_rn(__fmul_rn(x[kk][hf][j], rot_c)));
        x[kk][hf][j] = v;
        qs += v;
        amax = fmaxf(amax, fabsf(v));
      }
  qs += __shfl_xor_sync(0xffffffffu, qs, 1);
  qs += __shfl_xor_sync(0xffffffffu, qs, 2);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e = 0;
  if (amax > 0.f && amax <= 3.0e38f) {
    int ex;
    frexpf(amax, &ex);
    e = 15 - ex;
    // paired columns: 256 hi + lo with both signed bytes reaches 32639; the one scaled bf16 value above
    // it (32640, an all-ones mantissa at the top of the range) takes one bit less for the whole operand
    if (pc && ldexpf(amax, e) > 32639.f) e = 14 - ex;
  }
  if (p.qfmt == 2) {
    // fp16 B fragments of 16x8x16 multiplies (NVFP4 pages): block 2kk + hf holds dims 4t, 4t+1
    // (register 0) and 4t+2, 4t+3 (register 1) of column g, times 2^e (exact for bf16 values)
#pragma unroll
    for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        qf.b[2 * kk + hf][0] = pack_half2(ldexpf(x[kk][hf][0], e), ldexpf(x[kk][hf][1], e));
        qf.b[2 * kk + hf][1] = pack_half2(ldexpf(x[kk][hf][2], e), ldexpf(x[kk][hf][3], e));
      }
  } else if (pc) {
    // |q| <= 32639: hi = round(q / 256) and lo = q - 256 hi are both signed bytes
#pragma unroll
    for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t w = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qi = __float2int_rn(ldexpf(x[kk][hf][j], e));
          const int hi = (qi + 128) >> 8;
          w |= (static_cast<uint32_t>((g8 & 1) ? qi - 256 * hi : hi) & 0xFFu) << (8 * j);
        }
        qf.b[kk][hf] = w;
        qf.b[NKK + kk][hf] = 0u;
      }
  } else {
#pragma unroll
    for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t whi = 0u, wlo = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int qi = __float2int_rn(ldexpf(x[kk][hf][j], e));   // |qi| < 2^15
          whi |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * j);
          wlo |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * j);
        }
        qf.b[kk][hf] = whi;
        qf.b[NKK + kk][hf] = wlo;
      }
  }
  // sum(q) of the heads of this lane's columns 2t and 2t+1 (held by lanes 8t and 8t+4); with paired
  // columns lane 8t holds head t, the one this lane owns
  qf.qs0 = __shfl_sync(0xffffffffu, qs, 8 * t) * p.scale_log2;
  qf.qs1 = __shfl_sync(0xffffffffu, qs, 8 * t + 4) * p.scale_log2;
  qf.kscale = ldexpf(p.scale_log2, -e);
}

// Store a query operand as the 16*D + 64 byte blob the attention kernels read:
// the 16-byte B-fragment words of every lane, then the sums of the 8 columns
// and kscale.
template <int D>
__device__ __forceinline__ void store_qblob(uint8_t* blob, const QFrag<D>& qf, int lane, bool paired) {
  // paired columns: both planes share b[0 .. D/32), half the words
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc)
    if (cc < D / 64 || !paired)
      reinterpret_cast<uint4*>(blob)[cc * 32 + lane] =
          make_uint4(qf.b[2 * cc][0], qf.b[2 * cc][1], qf.b[2 * cc + 1][0], qf.b[2 * cc + 1][1]);
  float* tail = reinterpret_cast<float*>(blob + 16 * D);
  if (lane < 4) { tail[2 * lane] = qf.qs0; tail[2 * lane + 1] = qf.qs1; }   // lanes 0-3: columns 2t, 2t+1
  if (lane == 0) tail[MAX_G] = qf.kscale;
}

// The same query operand in the layout of the tensor-memory kernel: the two
// 8-bit planes as B matrices of its score multiplies (K-major, no swizzle;
// N = 8 columns, K = the 128 code bytes of a TMEM row), hi plane in the first
// 1 KB, lo plane in the second; the tail as in store_qblob.  Code byte p of a
// row (p = (D/4) t + 8 kk + 4 hf + j) holds dim 32 kk + 16 hf + 4 t + j; byte
// (column n, p) of a plane sits at 128 (p / 16) + 16 n + p % 16.
template <int D>
__device__ __forceinline__ void store_qblob_tc(uint8_t* blob, const QFrag<D>& qf, int lane) {
  static_assert(D == 128, "the tensor-memory kernel covers D = 128");
  constexpr int NKK = D / 32;
  const int n = lane >> 2, t = lane & 3;
  uint32_t* w = reinterpret_cast<uint32_t*>(blob);
#pragma unroll
  for (int kk = 0; kk < NKK; ++kk)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int pos = (D / 4) * t + 8 * kk + 4 * hf;
      const int a = (128 * (pos >> 4) + 16 * n + (pos & 15)) >> 2;
      w[a] = qf.b[kk][hf];
      w[256 + a] = qf.b[NKK + kk][hf];
    }
  float* tail = reinterpret_cast<float*>(blob + 16 * D);
  if (lane < 4) { tail[2 * lane] = qf.qs0; tail[2 * lane + 1] = qf.qs1; }
  if (lane == 0) tail[MAX_G] = qf.kscale;
}

}  // namespace tiles
}  // namespace kv4

// Device pieces of the fused rotate + quantize + append, shared by the append
// kernel and the fused decode step.  See kv4_append.cu for the arithmetic.
#pragma once
#include "kv4_common.cuh"

namespace kv4 {

namespace {

struct AppendParams {
  uint8_t* pool;             // INT4 or BF16 pool of the layer
  uint8_t* prot;             // INT8 store of the layer (INT4 cache only)
  const int32_t* block_table;
  int32_t* seq_lens;         // this layer's row
  const int32_t* seq_ids;
  const int32_t* cu_new;
  const uint16_t* k_new;
  const uint16_t* v_new;
  State* state;
  int n_seqs, total_new, Hkv, D, P, S, W, Bh;
  int max_seqs, num_pages, max_pages_per_seq;
  int fmt;                   // page format: KV4_FORMAT_INT4 or KV4_FORMAT_NVFP4
  float rot_c;               // fp32(1/sqrt(Bh))
  RopeParams rope;           // RoPE of the keys at their positions (cs == nullptr: none)
};

// RoPE of one row held VPL consecutive dims per lane (dims VPL*lane ..), at
// table row `pos`: pair (a, b) -> (a*c - b*s, b*c + a*s), every product and
// sum rounded to fp32.  Neox pairs (d, d + R/2) sit R/(2*VPL) lanes apart (R
// a power of two), gptj pairs (d, d + 1) in one lane.  All lanes call it.
template <int VPL>
__device__ __forceinline__ void rope_row(float (&x)[VPL], const RopeParams& r, int pos, int lane) {
  const float* cs = r.cs + static_cast<long long>(pos) * r.R;
  const int half = r.R >> 1, d0 = VPL * lane;
  if (r.style == KV4_ROPE_GPTJ) {
    if (d0 < r.R) {
#pragma unroll
      for (int k = 0; k < VPL; k += 2) {
        const int i = (d0 + k) >> 1;
        const float c = __ldg(cs + i), s = __ldg(cs + half + i);
        const float a = x[k], b = x[k + 1];
        x[k] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
        x[k + 1] = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
      }
    }
  } else {
    float y[VPL];
#pragma unroll
    for (int k = 0; k < VPL; ++k) y[k] = __shfl_xor_sync(0xffffffffu, x[k], half / VPL);
    if (d0 < r.R) {
      const bool first = d0 < half;   // holds a; the partner lane holds b
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int i = first ? d0 + k : d0 + k - half;
        const float c = __ldg(cs + i), s = __ldg(cs + half + i);
        x[k] = first ? __fsub_rn(__fmul_rn(x[k], c), __fmul_rn(y[k], s))
                     : __fadd_rn(__fmul_rn(x[k], c), __fmul_rn(y[k], s));
      }
    }
  }
}

template <int VPL>
__device__ __forceinline__ void fwht_warp(float (&x)[VPL], int Bh, float c, int lane) {
  fwht_row<VPL>(x, Bh, lane);
#pragma unroll
  for (int i = 0; i < VPL; ++i) x[i] = __fmul_rn(x[i], c);
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Quantize the warp's group with Q = 2^bits - 1; codes go to smem, (s, z) are returned packed as half2 bits.
template <int VPL>
__device__ __forceinline__ uint32_t quantize_group(const float (&x)[VPL], float mn, float mx, float Q,
                                                   uint8_t* codes, int lane) {
  const __half z16 = __float2half_rd(mn);
  const float z = __half2float(z16);
  const float r = __fsub_rn(mx, z);
  const __half s16 = (r == 0.f) ? __float2half(1.f) : __float2half_ru(__fdiv_rn(r, Q));
  const float s = __half2float(s16);
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    float c = rintf(__fdiv_rn(__fsub_rn(x[i], z), s));
    c = fminf(fmaxf(c, 0.f), Q);
    codes[VPL * lane + i] = static_cast<uint8_t>(c);
  }
  return static_cast<uint32_t>(__half_as_ushort(s16)) | (static_cast<uint32_t>(__half_as_ushort(z16)) << 16);
}

// Write one token's INT4 codes (K: tensor 0, V: tensor 1) and scales into its tile.
__device__ __forceinline__ void store_int4(uint8_t* tile, int r, int tensor, const uint8_t* codes, uint32_t sz,
                                           int D, int lane) {
  if (tensor == 0) {
    // word (t, kk): byte j holds dim 32kk + 4t + j (low nibble) and 32kk + 16 + 4t + j (high nibble)
    const int nkk = D / 32;
    if (lane < D / 8) {
      const int t = lane / nkk, kk = lane % nkk;
      uint32_t w = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w |= static_cast<uint32_t>(codes[32 * kk + 4 * t + j]) << (8 * j);
        w |= static_cast<uint32_t>(codes[32 * kk + 16 + 4 * t + j]) << (8 * j + 4);
      }
      *reinterpret_cast<uint32_t*>(tile + r * (D / 2) + t * (D / 8) + 4 * kk) = w;
    }
  } else {
    const int t = (r & 7) >> 1, e = r & 1, th = r >> 3;
    for (int q = lane; q < D / 2; q += 32) {
      const int m = q >> 3, g = q & 7;
      const uint8_t b = static_cast<uint8_t>(codes[16 * m + g] | (codes[16 * m + g + 8] << 4));
      tile[8 * D + 512 * (m >> 2) + 16 * (4 * g + t) + 4 * (m & 3) + th + 2 * e] = b;
    }
  }
  if (lane == 0) *reinterpret_cast<uint32_t*>(tile + 16 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3))) = sz;
}

// ---------------------------------------------------------------------------
// NVFP4 pages ("KV Cache Quantization" topic page, item 3: NVFP4 storage of the
// paged KV cache; blocks of 16 dims, E2M1 codes, one E4M3 scale, per-tensor
// scale 1).  Per block: amax = max |x| (exact), s = fp32(amax / 6), s8 = s
// rounded to the nearest E4M3 value (ties to even, saturating at 448); code =
// the nearest E2M1 magnitude of fp32(x / s8) (ties to the even mantissa,
// saturating at 6), sign bit only for a nonzero magnitude; s8 = 0 gives codes 0.

// E4M3 code of s >= 0 (round to nearest even, saturated at 448).
__device__ __forceinline__ uint32_t e4m3_rn(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(s));
  return r & 0xFFu;
}
// Value of an E4M3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(code & 0xFFu)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}
// E2M1 code of q: seven comparisons on |q| (ties at 0.25, 1.25, 2.5, 5 stay down, at 0.75, 1.75, 3.5
// go up: the even mantissa), saturating at 6; the sign bit only for a nonzero magnitude.
__device__ __forceinline__ uint32_t e2m1_code(float q) {
  const float a = fabsf(q);
  const uint32_t mag = static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
                       static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
                       static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) +
                       static_cast<uint32_t>(a > 5.f);
  return mag | ((q < 0.f && mag != 0u) ? 8u : 0u);
}

// Quantize the warp's row (VPL dims per lane) in blocks of 16 dims: codes (one byte per dim) to smem,
// the E4M3 scale code of the lane's block returned.
template <int VPL>
__device__ __forceinline__ uint32_t quantize_fp4(const float (&x)[VPL], uint8_t* codes, int lane) {
  constexpr int LPB = 16 / VPL;   // lanes per block
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
  for (int o = 1; o < LPB; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  const uint32_t s8 = e4m3_rn(__fdiv_rn(a, 6.f));
  const float s = e4m3_value(s8);
#pragma unroll
  for (int i = 0; i < VPL; ++i) codes[VPL * lane + i] = static_cast<uint8_t>(s > 0.f ? e2m1_code(__fdiv_rn(x[i], s)) : 0u);
  return s8;
}

// Write one token's NVFP4 codes and scales into its page tile (layout: see the tile description of the
// attention kernel).  K bytes belong to the token; a V byte holds one dim of tokens 2i and 2i+1, so the
// token's V nibbles go in with atomic and/or on their 32-bit words (the other token may be written by
// another warp of the same launch).  s8: the E4M3 code of the lane's block (VPL dims per lane).
template <int VPL>
__device__ __forceinline__ void store_fp4(uint8_t* tile, int r, int tensor, const uint8_t* codes, uint32_t s8,
                                          int D, int lane) {
  constexpr int LPB = 16 / VPL;
  const int nb = D / 16;
  const uint32_t sb = __shfl_sync(0xffffffffu, s8, (lane % nb) * LPB);   // lane b < nb: the scale of block b
  if (tensor == 0) {
    const int g = r & 7, rh = r >> 3;
    for (int q = lane; q < D / 2; q += 32) {   // q = 8 b + 2 t + j: dims 16 b + 4 t + 2 j, +1
      const int j = q & 1, t = (q >> 1) & 3, b = q >> 3;
      const int d = 16 * b + 4 * t + 2 * j;
      tile[16 * (4 * g + t) + 4 * (b & 3) + 512 * (b >> 2) + rh + 2 * j] =
          static_cast<uint8_t>(codes[d] | (codes[d + 1] << 4));
    }
    if (lane < nb) tile[16 * D + (D / 8) * g + 2 * lane + rh] = static_cast<uint8_t>(sb);
  } else {
    const int th = r >> 3, t = (r & 7) >> 1, e = r & 1;
    for (int q = lane; q < D / 2; q += 32) {   // q = 8 m + gg: dims 16 m + gg (byte 2 th) and + 8 (byte 2 th + 1)
      const int m = q >> 3, gg = q & 7;
      uint32_t* w = reinterpret_cast<uint32_t*>(tile + 8 * D + 16 * (4 * gg + t) + 4 * (m & 3) + 512 * (m >> 2));
      const int sh = 16 * th + 4 * e;
      const uint32_t mask = (0xFu << sh) | (0xFu << (sh + 8));
      const uint32_t val = (static_cast<uint32_t>(codes[16 * m + gg]) << sh) |
                           (static_cast<uint32_t>(codes[16 * m + gg + 8]) << (sh + 8));
      atomicAnd(w, ~mask);
      atomicOr(w, val);
    }
    if (lane < nb) tile[17 * D + (D / 4) * t + 4 * lane + 2 * th + e] = static_cast<uint8_t>(sb);
  }
}

// Write one token's INT2 codes (four a byte; every byte belongs to the token) and scales into its page
// tile: K byte r D/4 + t D/16 + 4 kq + j holds dims 64 kq + 16 c + 4 t + j in bits 2c, 2c+1; V byte
// 4D + (D/8)(4 g + t) + 4 mp + th + 2 e (token 8 th + 2 t + e) holds dims 16 (2 mp + mb) + 8 dh + g in
// bits 2 (dh + 2 mb); the half2 (s, z) block at 8D as in the INT4 tile.
__device__ __forceinline__ void store_int2(uint8_t* tile, int r, int tensor, const uint8_t* codes, uint32_t sz,
                                           int D, int lane) {
  for (int q = lane; q < D / 4; q += 32) {
    uint32_t b = 0u;
    int off;
    if (tensor == 0) {
      const int t = q / (D / 16), rem = q % (D / 16), kq = rem >> 2, j = rem & 3;
#pragma unroll
      for (int c = 0; c < 4; ++c) b |= static_cast<uint32_t>(codes[64 * kq + 16 * c + 4 * t + j]) << (2 * c);
      off = r * (D / 4) + q;
    } else {
      const int th = r >> 3, t = (r & 7) >> 1, e = r & 1, g = q & 7, mp = q >> 3;
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int dh = 0; dh < 2; ++dh)
          b |= static_cast<uint32_t>(codes[16 * (2 * mp + mb) + 8 * dh + g]) << (2 * (dh + 2 * mb));
      off = 4 * D + (D / 8) * (4 * g + t) + 4 * mp + th + 2 * e;
    }
    tile[off] = static_cast<uint8_t>(b);
  }
  if (lane == 0) *reinterpret_cast<uint32_t*>(tile + 8 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3))) = sz;
}

// Write one token's INT8 codes and scales into its protected tile.
__device__ __forceinline__ void store_int8(uint8_t* tile, int r, int tensor, const uint8_t* codes, uint32_t sz,
                                           int D, int lane) {
  if (tensor == 0) {
    // word L = (D/16) t + 2 kk + hf of the token: dims 32kk + 16hf + 4t + 0..3, one per byte
    if (lane < D / 4) {
      const int t = lane / (D / 16), wi = lane % (D / 16), kk = wi >> 1, hf = wi & 1;
      const int d = 32 * kk + 16 * hf + 4 * t;
      const uint32_t w = static_cast<uint32_t>(codes[d]) | (static_cast<uint32_t>(codes[d + 1]) << 8) |
                         (static_cast<uint32_t>(codes[d + 2]) << 16) | (static_cast<uint32_t>(codes[d + 3]) << 24);
      *reinterpret_cast<uint32_t*>(tile + r * D + 4 * lane) = w;
    }
  } else {
    const int t = (r & 7) >> 1, e = r & 1, th = r >> 3;
    for (int q = lane; q < D / 2; q += 32) {
      const int m = q >> 3, gg = q & 7;
      const int w = 2 * m + th;
      const uint16_t v = static_cast<uint16_t>(codes[16 * m + gg] | (codes[16 * m + gg + 8] << 8));
      *reinterpret_cast<uint16_t*>(tile + 16 * D + 16 * (32 * (w >> 2) + 4 * gg + t) + 4 * (w & 3) + 2 * e) = v;
    }
  }
  if (lane == 0) *reinterpret_cast<uint32_t*>(tile + 32 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3))) = sz;
}

// Launch parameters of an append into `layer` of cache c.
inline AppendParams append_params(const kv4_cache* c, int layer, const int32_t* seq_ids, const int32_t* cu_new,
                                  int n_seqs, int total_new, const void* k_new, const void* v_new, bool rope) {
  const kv4_config& cfg = c->cfg;
  AppendParams p{};
  if (rope) p.rope = c->rope;
  uint8_t* lbase = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  p.pool = lbase;
  p.prot = c->bf16 ? nullptr : lbase + c->pool_bytes;
  p.block_table = c->block_table;
  p.seq_lens = c->seq_lens + static_cast<size_t>(layer) * cfg.max_seqs;
  p.seq_ids = seq_ids;
  p.cu_new = cu_new;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.state = c->state;
  p.n_seqs = n_seqs;
  p.total_new = total_new;
  p.Hkv = cfg.num_kv_heads;
  p.D = cfg.head_dim;
  p.P = cfg.page_size;
  p.S = cfg.sink_tokens;
  p.W = cfg.recent_window;
  p.Bh = c->bf16 ? 1 : cfg.hadamard_block;
  p.max_seqs = cfg.max_seqs;
  p.num_pages = cfg.num_pages;
  p.max_pages_per_seq = cfg.max_pages_per_seq;
  p.rot_c = static_cast<float>(1.0 / sqrt(static_cast<double>(p.Bh)));
  p.fmt = c->bf16 ? KV4_FORMAT_INT4 : cfg.page_format;
  return p;
}

// Encode one (token, KV head, K or V) row held as bf16 bits raw[] (dims
// VPL*lane ..): RoPE of a key when a table is set, rotation, clamp, INT4 codes
// into its page tile and, for a protected position, INT8 codes into the
// sequence's protected store.  tile_idx: the row's INT4 tile; r: its slot
// there.  c4 / c8: the warp's code staging in shared memory.  All lanes call it.
template <int D>
__device__ __forceinline__ void encode_row(const AppendParams& p, const uint16_t (&raw)[D / 32], int tensor, int h,
                                           int seq, int pos, int L_new, long long tile_idx, int r, uint8_t* c4,
                                           uint8_t* c8, int lane) {
  constexpr int VPL = D / 32;
  float x[VPL];
  bool bad = false;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const float v = __bfloat162float(__ushort_as_bfloat16(raw[k]));
    bad |= !(fabsf(v) <= 3.0e38f);
    x[k] = v;
  }
  if (tensor == 0 && p.rope.cs != nullptr) rope_row<VPL>(x, p.rope, pos, lane);   // the key at its position
  fwht_warp<VPL>(x, p.Bh, p.rot_c, lane);
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const float c = fminf(fmaxf(x[k], -65504.f), 65504.f);
    bad |= (c != x[k]);
    x[k] = c;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&p.state->status, KV4_DEV_RANGE);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int k = 1; k < VPL; ++k) { mn = fminf(mn, x[k]); mx = fmaxf(mx, x[k]); }
  mn = warp_min(mn);
  mx = warp_max(mx);
  const bool fp4 = p.fmt == KV4_FORMAT_NVFP4, int2 = p.fmt == KV4_FORMAT_INT2;
  const uint32_t sz4 = fp4 ? quantize_fp4<VPL>(x, c4, lane)
                           : quantize_group<VPL>(x, mn, mx, int2 ? 3.f : 15.f, c4, lane);
  const bool protect = pos < p.S || pos >= L_new - p.W;
  uint32_t sz8 = 0;
  if (protect) sz8 = quantize_group<VPL>(x, mn, mx, 255.f, c8, lane);
  __syncwarp();
  if (fp4) store_fp4<VPL>(p.pool + tile_idx * tilef_bytes(D), r, tensor, c4, sz4, D, lane);
  else if (int2) store_int2(p.pool + tile_idx * tile2_bytes(D), r, tensor, c4, sz4, D, lane);
  else store_int4(p.pool + tile_idx * tile4_bytes(D), r, tensor, c4, sz4, D, lane);
  if (protect) {
    const int slot = pos < p.S ? pos : p.S + (pos - p.S) % p.W;
    const int npt = n_prot_tiles(p.S, p.W);
    uint8_t* t8 = p.prot + ((static_cast<long long>(seq) * npt + slot / TILE) * p.Hkv + h) * tile8_bytes(D);
    store_int8(t8, slot & (TILE - 1), tensor, c8, sz8, D, lane);
  }
}

}  // namespace

}  // namespace kv4

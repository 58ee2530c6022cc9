// Internal definitions shared by the kv4 CUDA sources (sm_100a only).
//
// Tile format (one KV head, 16 consecutive token slots):
//   INT4 tile  [K codes 8*D][V codes 8*D][scales 128]      16*D + 128 bytes
//   INT8 tile  [K codes 16*D][V codes 16*D][scales 128]    32*D + 128 bytes
//   BF16 tile  [K 16*D bf16][V 16*D bf16]                  64*D bytes
// Inside a code block the nibbles/bytes are ordered so that one 16-byte
// shared-memory load per lane yields the A operands of the 16x8x16 tensor-core
// multiply directly (lane = 4*g + t holds rows g, g+8 and columns 2t, 2t+1,
// 2t+8, 2t+9 of each 16x16 operand):
//   INT4 K, token r = 8*rowhi + g, dim d = 32*kk + 8*j + 2*t + e:
//       nibble (j + 4*e) of the word at byte r*D/2 + t*D/8 + 4*kk
//   INT4 V, dim d = 16*m + 8*dh + g, token r = 8*th + 2*t + e:
//       nibble (dh + 2*th + 4*e) of the word at byte 512*(m/4) + 16*(4*g+t) + 4*(m%4)
//   INT8 K: byte (h8 + 2*e) of the word at 16*(32*(rowhi*D/64 + k/4) + 4*g + t) + 4*(k%4)
//           for d = 16*k + 8*h8 + 2*t + e
//   INT8 V: byte (dh + 2*e) of the word at 16*(32*(w/4) + 4*g + t) + 4*(w%4), w = 2*m + th
//   BF16 K: element 8*(32*k + 4*g + t) + 2*(rowhi + 2*h8) + e
//   BF16 V: element 8*(32*m + 4*g + t) + 2*(dh + 2*th) + e
//   scales: half2 (s, z) of token r, tensor T (K=0, V=1) at byte 16*(r%8) + 4*(2*T + r/8)
// Pools are head-innermost: INT4/BF16 pool [page][P/16][Hkv][tile], INT8 store
// [seq][ceil((S+W)/16)][Hkv][tile8], so one page position of all KV heads is
// one contiguous run.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kv4.h"

namespace kv4 {

constexpr int TILE = 16;
constexpr int MAX_G = 8;                 // query heads per KV head handled by one n8 tile
constexpr int STATE_BYTES = 256;

__host__ __device__ constexpr int tile4_bytes(int D) { return 16 * D + 128; }
__host__ __device__ constexpr int tile8_bytes(int D) { return 32 * D + 128; }
__host__ __device__ constexpr int tile16_bytes(int D) { return 64 * D; }
// NVFP4 page tile: K codes 8*D, V codes 8*D, K scales D, V scales D (one E4M3 byte per token and 16 dims)
__host__ __device__ constexpr int tilef_bytes(int D) { return 18 * D; }
// INT2 page tile: K codes 4*D, V codes 4*D, the half2 (s, z) block of 128 bytes
__host__ __device__ constexpr int tile2_bytes(int D) { return 8 * D + 128; }
__host__ __device__ constexpr int page_tile_bytes(int D, int fmt) {
  return fmt == 1 ? tilef_bytes(D) : (fmt == 2 ? tile2_bytes(D) : tile4_bytes(D));
}
__host__ __device__ constexpr int qblob_bytes(int D) { return 16 * D + 64; }
__host__ __device__ inline int n_prot_tiles(int S, int W) { return (S + W + TILE - 1) / TILE; }

// Device state block at the start of every cache buffer (zeroed at creation).
struct State {
  int status;          // KV4_DEV_* bits
  int append_done;     // blocks of the current append launch that finished
  int n_items[3];      // work items of the current attention call: full chunks, tails, protected
  int n_parts;         // partial slots allocated by the current attention call
  int work;            // next work item to claim (persistent attention kernel)
  int pad[57];
};
static_assert(sizeof(State) == STATE_BYTES, "state block size");

// One unit of split-K work: a token range of one (sequence, KV head).
struct Item {
  int b;        // index into the call's seq_ids
  int seq;      // sequence id
  int h;        // KV head
  int kind;     // 0 = INT4 page tiles, 1 = INT8 protected tiles, 2 = BF16 tiles
  int t_begin;  // first tile (INT4/BF16: absolute tile index pos/16; INT8: store tile)
  int t_end;    // one past the last tile
  int lo, hi;   // valid positions (INT8: store slots) [lo, hi)
  int part;     // partial slot written by this item
  int pad[3];
};
static_assert(sizeof(Item) == 48, "item size");

// Per (sequence, KV head) record written by the planning kernel: the partials
// of this head are part_base + j * stride, j < n_parts.
struct SeqHead {
  int part_base;
  int n_parts;
  int len;
  int pad;    // stride between consecutive partials of the head
};

// Parameters shared by the attention kernels.
// A caller's RoPE table: fp32 [max_pos][R], cos of the R/2 angles then their
// sin; style KV4_ROPE_NEOX or KV4_ROPE_GPTJ.
struct RopeParams {
  const float* cs;
  int max_pos, R, style;
};

struct AttnParams {
  const uint8_t* pool;        // INT4 (or BF16) page pool of the layer
  const uint8_t* prot;        // INT8 store of the layer (INT4 mode)
  const int32_t* block_table;
  const int32_t* seq_lens;    // this layer's row [max_seqs]
  const int32_t* seq_ids;
  const uint16_t* q;          // bf16 [n_seqs][qlen][Hq][D]
  void* out;
  State* state;
  Item* items[3];             // item regions
  int cap[3];
  SeqHead* seqhead;           // [n_seqs * Hkv]
  uint8_t* qblob;             // [n_seqs * Hkv][qblob_bytes]
  float* partials;            // [cap_parts][G][D + 4]: o[D], m, l, pad
  int cap_parts;
  int n_seqs, Hq, Hkv, G, D, P, S, W, Bh;   // G: operand columns per KV head (qlen * Gh)
  int qlen, Gh;               // query tokens of this launch, query heads per KV head
  int q0, qtot;               // first query token of this launch, query tokens per sequence (the last qtot
                              // positions; a call with more tokens than one operand holds runs in chunks)
  int max_seqs, num_pages, max_pages_per_seq;
  int chunk_tiles;
  int mode;
  float scale_log2;           // softmax_scale * log2(e)
  float rot_c;                // fp32(1/sqrt(Bh))
  RopeParams rope;            // RoPE of q at its position (cs == nullptr: none)
  int Bh_q, Bh_o;             // block of the rotation applied to q / to the output (1: none, the
  float rc_q, rc_o;           // caller folded it into the projections), and its fp32(1/sqrt(block))
  size_t pool_bytes, prot_bytes, qblob_total;   // extents, for the self-checks of debug builds
  int ns;                     // shared-memory ring depth of the attention kernel
  int grid;                   // CTAs of the page-major attention kernel
  int stall_stage;            // test hook: stage the first CTA leaves unfilled (-1: none)
  int qfmt;                   // query operand layout the query kernels write: 0 integer fragments, 1 tensor-memory
                              // kernel, 2 fp16 fragments (NVFP4 pages), 3 paired integer columns (one query
                              // token, at most 4 query heads per KV head)
  int wait_first;             // the attention kernel is the programmatic dependent of the fused step kernel: it
                              // waits for that grid before its first instruction (the plan reads the new lengths)
};

// Row of q (and of the output) that operand column c of KV head h of batch
// entry b stands for: query token q0 + c / Gh of the entry (the tokens are the
// last qtot positions, oldest first), query head h * Gh + c % Gh.
__device__ __forceinline__ long long q_row(const AttnParams& p, int b, int h, int c) {
  const int i = c / p.Gh, g = c - i * p.Gh;
  return (static_cast<long long>(b) * p.qtot + p.q0 + i) * p.Hq + h * p.Gh + g;
}

// ---------------------------------------------------------------------------
// Self-checks (debug builds, -DKV4_DEBUG_CHECKS): every shared-memory access,
// bulk copy and mbarrier address is checked against its buffer; a bad access is
// recorded in kv4_debug_slot (first failure wins) and skipped.

#ifdef KV4_DEBUG_CHECKS
static __device__ unsigned long long kv4_debug_slot[4];   // code, value a, value b, count (per translation unit)
extern __shared__ __align__(128) uint8_t kv4_dyn_smem[];
__device__ __forceinline__ uint32_t dyn_smem_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}
__device__ __forceinline__ bool dbg_fail(int code, unsigned long long a, unsigned long long b) {
  if (atomicCAS(&kv4_debug_slot[0], 0ull, static_cast<unsigned long long>(code)) == 0ull) {
    kv4_debug_slot[1] = a;
    kv4_debug_slot[2] = b;
  }
  atomicAdd(&kv4_debug_slot[3], 1ull);
  return true;
}
// true when [addr, addr+bytes) is inside the dynamic shared window and aligned
__device__ __forceinline__ bool smem_ok(uint32_t addr, uint32_t bytes, uint32_t align, int code) {
  const uint32_t lo = static_cast<uint32_t>(__cvta_generic_to_shared(kv4_dyn_smem));
  if (addr < lo || addr + bytes > lo + dyn_smem_size() || (addr & (align - 1))) {
    dbg_fail(code, addr - lo, bytes);
    return false;
  }
  return true;
}
#define KV4_SMEM_OK(addr, bytes, align, code) ::kv4::smem_ok((addr), (bytes), (align), (code))
#else
#define KV4_SMEM_OK(addr, bytes, align, code) true
#endif

// ---------------------------------------------------------------------------
// PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  if (!KV4_SMEM_OK(bar, 8, 8, 1)) return;
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  if (!KV4_SMEM_OK(bar, 8, 8, 2)) return;
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  if (!KV4_SMEM_OK(bar, 8, 8, 3)) return;
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  if (!KV4_SMEM_OK(bar, 8, 8, 4)) return true;
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase.  Gives up after ~1 s (or at once when
// *abort is set by another warp), sets KV4_DEV_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > 1000000000ull) {
        atomicOr(status, KV4_DEV_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

// 1-D bulk copy global -> shared (no multicast), completion on an mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  if (!KV4_SMEM_OK(dst, bytes, 16, 5) || !KV4_SMEM_OK(bar, 8, 8, 6)) return;
#ifdef KV4_DEBUG_CHECKS
  if ((reinterpret_cast<uintptr_t>(src) & 15) || (bytes & 15)) {
    dbg_fail(7, reinterpret_cast<uintptr_t>(src), bytes);
    return;
  }
#endif
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  if (!KV4_SMEM_OK(addr, 16, 16, 8)) return make_uint4(0, 0, 0, 0);
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  if (!KV4_SMEM_OK(addr, 8, 8, 9)) return make_uint2(0, 0);
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  if (!KV4_SMEM_OK(addr, 4, 4, 14)) return 0u;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}

// D = A * B + D, 16x8x16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B + D, 16x8x32, A unsigned 8-bit, B signed 8-bit, int32 accumulate.
__device__ __forceinline__ void imma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B + D, 16x8x32, A and B unsigned 8-bit, int32 accumulate.
__device__ __forceinline__ void imma_u8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B + D, 16x8x16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit elements held in the 16x8x16 fragment order.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Codes -> fp16 operands.  The magic exponent 0x6400 makes (0x6400 | c) the
// half value 1024 + c for c < 1024; subtracting 1024 (or, for a nibble left at
// bits 4-7, scaling by 1/16 and subtracting 64) gives c exactly.
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) {  // nibbles at bits 0-3 and 16-19
  uint32_t x = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1024.f), __half(1024.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t nib_hi(uint32_t w) {  // nibbles at bits 4-7 and 20-23
  uint32_t x = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  __half2 h = __hfma2(*reinterpret_cast<__half2*>(&x), __half2(__half(0.0625f), __half(0.0625f)),
                      __half2(__half(-64.f), __half(-64.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t byte_lo(uint32_t w) {  // bytes 0 and 2
  uint32_t x = lop3_and_or(w, 0x00FF00FFu, 0x64006400u);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1024.f), __half(1024.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Centred operands for P.V: a code c becomes c - 8 (INT4) or c - 128 (INT8),
// still exact in fp16, and the zero point z becomes z + 8 s (or z + 128 s).
// The code term then has both signs and no longer nearly cancels a large
// zero-point sum after thousands of tensor-core accumulations.
__device__ __forceinline__ uint32_t nib_lo_c(uint32_t w) {  // nibbles at bits 0-3 and 16-19, minus 8
  uint32_t x = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1032.f), __half(1032.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t nib_hi_c(uint32_t w) {  // nibbles at bits 4-7 and 20-23, minus 8
  uint32_t x = lop3_and_or(w, 0x00F000F0u, 0x64006400u);
  __half2 h = __hfma2(*reinterpret_cast<__half2*>(&x), __half2(__half(0.0625f), __half(0.0625f)),
                      __half2(__half(-72.f), __half(-72.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t byte_lo_c(uint32_t w) {  // bytes 0 and 2, minus 128
  uint32_t x = lop3_and_or(w, 0x00FF00FFu, 0x64006400u);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1152.f), __half(1152.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Bytes 0, 1 (or 2, 3) of w as an fp16 pair, minus 128 (exact).
__device__ __forceinline__ uint32_t bytes01_c(uint32_t w) {
  uint32_t x = __byte_perm(w, 0x64646464u, 0x4140);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1152.f), __half(1152.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t bytes23_c(uint32_t w) {
  uint32_t x = __byte_perm(w, 0x64646464u, 0x4342);
  __half2 h = __hsub2(*reinterpret_cast<__half2*>(&x), __half2(__half(1152.f), __half(1152.f)));
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float half_lo(uint32_t x) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(x & 0xFFFFu)));
}
__device__ __forceinline__ float half_hi(uint32_t x) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(x >> 16)));
}

// Butterfly stages hh = 1, 2, 4, ... (ascending, those with hh < Bh) of the
// block-diagonal Hadamard over a row of 32*VPL values held VPL per lane
// (element d = VPL*lane + i): the lower element of each pair becomes a + b,
// the upper a - b.  The stages are unrolled at compile time (static register
// indices) and skipped at run time.
template <int VPL>
__device__ __forceinline__ void fwht_row(float (&x)[VPL], int Bh, int lane) {
#pragma unroll
  for (int hh = 1; hh < 32 * VPL; hh <<= 1) {
    if (hh < Bh) {
      if (hh < VPL) {
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if ((i & hh) == 0) {
            const float a = x[i], c = x[i + hh];
            x[i] = __fadd_rn(a, c);
            x[i + hh] = __fsub_rn(a, c);
          }
      } else {
        const int lm = hh / VPL;
        const bool upper = (lane & lm) != 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const float o = __shfl_xor_sync(0xffffffffu, x[i], lm);
          x[i] = upper ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host-side handle (one struct for both cache kinds).

}  // namespace kv4

struct kv4_cache {
  kv4_config cfg;
  bool bf16;                 // true for a kv4bf16_cache
  int device;
  int num_sms;
  uint8_t* base;
  kv4::State* state;
  int32_t* seq_lens;         // [num_layers][max_seqs]
  int32_t* block_table;
  size_t layer_stride;       // bytes between consecutive layers' pools
  size_t pool_offset;        // from base to layer 0's pool
  size_t pool_bytes;         // per layer
  size_t prot_bytes;         // per layer (INT4 cache only)
  int attn_blocks_per_sm;
  int attn_ring;             // ring depth chosen for the per-head attention kernel
  int gattn_ring;            // ring depth of the page-major kernel (0: not used by this cache)
  int gattn_pair;            // INT4 tiles per consumer iteration of the page-major kernel (1 or 2)
  kv4::RopeParams rope;      // registered RoPE table (cs == nullptr: none)
  cudaEvent_t ev_before;     // optional timing events around the split-K kernel
  cudaEvent_t ev_after;
  int test_stall;            // kv4_test_stall_next_attention: stage to leave unfilled in the next call (-1: none)
  bool use_tc;               // one-token attention with 4-head groups at D = 128 runs the tensor-memory kernel
  int tattn_ring;            // its ring depth
};

namespace kv4 {

// Makes the cache's device current for the lifetime of the object and gives
// the calling thread its previous current device back afterwards, so a call
// into the library leaves the caller's device selection as it found it.
class DeviceScope {
 public:
  explicit DeviceScope(int device) {
    if (cudaGetDevice(&prev_) != cudaSuccess) {
      cudaGetLastError();
      prev_ = -1;
    }
    ok_ = prev_ == device || cudaSetDevice(device) == cudaSuccess;
  }
  ~DeviceScope() {
    int cur = -1;
    if (prev_ >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev_) cudaSetDevice(prev_);
  }
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  bool ok() const { return ok_; }

 private:
  int prev_ = -1;
  bool ok_ = false;
};

// Launchers (defined in the .cu files).
int launch_append(kv4_cache* c, int layer, const int32_t* seq_ids, const int32_t* cu_new, int n_seqs, int total_new,
                  const void* k_new, const void* v_new, bool rope, cudaStream_t stream);
int launch_seq_reset(kv4_cache* c, int seq_id, cudaStream_t stream);
int launch_dequantize_debug(kv4_cache* c, int layer, int seq_id, int start, int count, int view, float* k_out,
                            float* v_out, cudaStream_t stream);
int launch_attention(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* q, void* out,
                     float softmax_scale, int mode, void* ws, size_t ws_bytes, cudaStream_t stream);
size_t attention_workspace_bytes(const kv4_cache* c, int n_seqs, int max_ctx);
int launch_extend_attention(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, int qlen, const void* q,
                            void* out, float softmax_scale, int mode, void* ws, size_t ws_bytes, cudaStream_t stream);
int attention_blocks_per_sm(kv4_cache* c);
void fill_common(const kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* q, void* out,
                 float softmax_scale, int mode, AttnParams& p);
int launch_decode_step(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* k_new,
                       const void* v_new, const void* q, void* out, float softmax_scale, int mode, void* ws,
                       size_t ws_bytes, cudaStream_t stream);
// page-major path (INT4 cache, KV heads a multiple of 4)
bool grouped_path(const kv4_cache* c);
int grouped_ring(kv4_cache* c);
size_t grouped_workspace_bytes(const kv4_cache* c, int n_seqs, int qlen);
int extend_chunk(const kv4_cache* c, int qlen);
int launch_grouped(kv4_cache* c, const AttnParams& p, void* ws, size_t ws_bytes, cudaStream_t stream);

}  // namespace kv4

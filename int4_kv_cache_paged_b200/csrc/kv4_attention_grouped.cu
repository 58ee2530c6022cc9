// Page-major, stream-K decode attention over the paged INT4/INT8 cache (every
// KV-head count: groups of 4 KV heads, or of 2 or 1 when the count is not a
// multiple of 4).
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Abstract (fused attention over the paged, rotated token-wise INT4
// cache) and "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4
// KV Cache Quantization", Abstract (sinks and recent positions read from INT8).
//
// One launch does the attention proper (a small query kernel runs alongside).
//
// Work decomposition.  A head group is GWR consecutive KV heads of one
// sequence (4 when the KV-head count is a multiple of 4, else 2 or 1).  Its
// work is a list of stages: one stage per 16-token INT4 tile position (the
// tiles of the group's heads are contiguous in the head-innermost pool: one
// 8.7 KB bulk copy for 4 heads at D = 128), then one or two stages per INT8
// protected tile (two halves of the heads when the group has 2 or 4).  Three
// CTAs share an SM: with 4-head groups, four consumer warps per scheduler hide
// the latency of each warp's dependent tile math.
// The stage lists of all head groups are concatenated, each group charged a
// few extra units for the cost of starting it (T units in all), and CTA c of
// the persistent grid takes units [c*T/N, (c+1)*T/N): every CTA gets the same
// share of bytes plus group starts (stream-K).  Every CTA derives this plan
// itself from the sequence lengths (a block scan over the head groups), so no
// planning kernel runs first.  Where a CTA's range crosses head groups it
// works on segments.
//
// Inside a CTA: a producer warp issues the bulk copies into a ring of
// shared-memory stages (each lane one stage of a batch, mbarrier completion);
// consumer warp w handles KV head w of every stage, so every warp consumes
// every stage in order (which keeps the mbarrier parity waits exact) and no
// warp waits for another.  The rotated query operands come from a small
// kernel launched just before (this kernel is its programmatic dependent and
// waits for it only before its first operand read).  A group that one CTA
// covers whole is normalised, rotated back and stored straight from registers;
// a group split over several CTAs leaves one partial (m, l, o) per segment in
// the workspace, and a merge kernel launched as this kernel's programmatic
// dependent (its blocks become resident while this grid still runs) combines
// them, one warp per query head.  Every CTA records where the groups that
// start in its range sit in the split, for that merge.
#include "kv4_attn_tiles.cuh"
#include "kv4_append_ops.cuh"
#include "kv4_tc.cuh"

#include <stdlib.h>
#include <string.h>

namespace kv4 {

namespace {

using namespace tiles;

// CTAs per SM: three (with 4-head groups, 4 warps per scheduler, which caps
// registers at 128 per thread)
constexpr int CTAS_PER_SM = 3;
constexpr int GQD = 2;                  // segment queue depth

// Shape of a kernel instantiation with groups of GWR KV heads (one consumer
// warp per head, plus the producer warp).  A protected tile position of the
// group's heads is H8 heads per stage, S8 stages.
template <int GWR>
struct GShape {
  static_assert(GWR == 1 || GWR == 2 || GWR == 4, "group width");
  static constexpr int THREADS = 32 * (GWR + 1);
  static constexpr int H8 = GWR >= 2 ? GWR / 2 : 1;
  static constexpr int S8 = GWR / H8;
};

// F: page format (0 INT4, 1 NVFP4, 2 INT2)
template <int D, int GWR, int F = 0>
struct GCfg {
  static constexpr int STAGE4 = GWR * page_tile_bytes(D, F);          // one tile position of the group's heads
  static constexpr int STAGE8 = GShape<GWR>::H8 * tile8_bytes(D);      // part of a protected tile position
  static constexpr int STAGE = STAGE4 > STAGE8 ? STAGE4 : STAGE8;
};

// KV heads per group for a cache: 4, else 2, else 1.
inline int group_width(int Hkv) { return Hkv % 4 == 0 ? 4 : (Hkv % 2 == 0 ? 2 : 1); }

// One head group of the call: batch entry b, KV heads GWR*hg .. GWR*hg+GWR-1.
struct Group {
  int b, seq, hg, L;  // index into seq_ids, sequence id, head group, sequence length
  int n4;             // INT4 stages (tiles t0 .. t0+n4-1)
  int t0, lo4, hi4;   // first INT4 tile, valid INT4 positions [lo4, hi4)
  int n8;             // INT8 tiles (S8 stages each), valid slots [0, nprot)
  int nprot;
  int start;          // first global stage index
  int pad;
};
static_assert(sizeof(Group) == 48, "group size");

// Where a head group sits in the split, written once per group by the CTA
// whose range holds its start (and the totals by CTA 0), read by the merge kernel.
struct GPlanRec {
  int start;          // first cost unit of the group
  int stages;         // its stages (0: an empty sequence)
};
struct GPlanHdr {
  int T, N;           // total cost units, active CTAs
  int pad[2];
};

struct SegQ {         // one queued segment
  Group g;
  int u0, n;          // local stages [u0, u0+n)
  int k, nseg;        // segment index within the group, segments of the group
};

// Per-CTA bookkeeping in shared memory.
struct GMisc {
  int abort;          // a wait gave up
  int pad1;
  int pad0;
  Group first;        // the group holding the CTA's first stage (start filled in)
  int n_empty;        // empty groups this CTA writes zeros for
  int pad[3];
  int red[32];        // block-scan scratch
  int empty[32];
  int last_fill[16];  // last ring fill per stage (drained before an aborting producer exits)
};

constexpr int MAX_NS = 16;
// A CTA takes at least this many stages: a short batch is spread over fewer
// CTAs, so that merging the partials costs less than the streaming it saves.
constexpr int MIN_STAGES = 16;
// Extra stages charged to every head group in the split: starting a group
// costs a CTA about as much as streaming this many stages (query operands,
// the segment's result, its partial), so a CTA that starts more groups gets
// fewer stages.
constexpr int GROUP_COST = 4;

template <int GWR>
__host__ __device__ inline int group_stages(const Group& g) { return g.n4 + GShape<GWR>::S8 * g.n8; }
// Length of a group in the units of the split: its stages plus the start cost (0 when empty).
template <int GWR>
__host__ __device__ inline int group_cost(const Group& g) {
  const int n = group_stages<GWR>(g);
  return n > 0 ? n + GROUP_COST : 0;
}

// CTA owning global stage j: the largest c with floor(c*T/N) <= j.
__device__ __forceinline__ int cta_of(long long j, long long T, long long N) {
  return static_cast<int>(((j + 1) * N - 1) / T);
}

template <int D, int GWR, int F = 0>
__host__ __device__ inline size_t gattn_smem_bytes(int ns) {
  using C = GCfg<D, GWR, F>;
  return static_cast<size_t>(ns) * C::STAGE + GQD * sizeof(SegQ) + (2 * ns + 2 * GQD) * sizeof(uint64_t) +
         sizeof(GMisc);
}

// Block-wide exclusive scan of one value per thread; returns the thread's prefix, *total the sum.
__device__ int block_exclusive_scan(int v, int* s_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? s_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_tmp[lane] = w;   // inclusive prefix of warp sums
  }
  __syncthreads();
  const int before = (warp > 0 ? s_tmp[warp - 1] : 0) + x - v;
  *total = s_tmp[nwarps - 1];
  __syncthreads();
  return before;
}

// Head group i of the call: which positions are read from INT4 pages and which
// from the INT8 store.
__device__ Group describe(const AttnParams& p, int i, int HGN, bool flag_bad) {
  Group g;
  g.b = i / HGN;
  g.hg = i - g.b * HGN;
  g.seq = p.seq_ids[g.b];
  int L = 0;
  if (g.seq >= 0 && g.seq < p.max_seqs) L = p.seq_lens[g.seq];
  else if (flag_bad && g.hg == 0) atomicOr(&p.state->status, KV4_DEV_BAD_SEQ);
  g.L = L;
  int lo4, hi4, nprot;
  if (p.mode & KV4_MODE_INT4_ONLY) { lo4 = 0; hi4 = L; nprot = 0; }
  else { nprot = min(L, p.S + p.W); lo4 = p.S; hi4 = L - p.W; }
  g.lo4 = lo4; g.hi4 = hi4; g.nprot = nprot;
  g.t0 = 0; g.n4 = 0;
  if (hi4 > lo4) { g.t0 = lo4 / TILE; g.n4 = (hi4 + TILE - 1) / TILE - g.t0; }
  g.n8 = (nprot + TILE - 1) / TILE;
  g.start = 0;
  g.pad = 0;
  return g;
}

// Zeros for the output rows of head group i (a sequence of length 0), elements e0, e0+step, ...
template <int GWR>
__device__ void zero_group(const AttnParams& p, int i, int e0, int step) {
  const int HGN = p.Hkv / GWR;
  const int b = i / HGN, hg = i - b * HGN;
  const int n = GWR * p.G * p.D;
  for (int e = e0; e < n; e += step) {
    const int r = e / p.D, d = e - r * p.D;   // r = KV head within the group * G + operand column
    const long long off = q_row(p, b, hg * GWR + r / p.G, r % p.G) * p.D + d;
    if (p.mode & KV4_MODE_OUT_F32) static_cast<float*>(p.out)[off] = 0.f;
    else static_cast<uint16_t*>(p.out)[off] = 0;
  }
}

// Normalise, rotate back and store the output of one KV head: lane (g8, t)
// holds o for heads 2t, 2t+1 (valid when < G) at dimensions 16m+g8 (o[m][0],
// o[m][1]) and 16m+g8+8 (o[m][2], o[m][3]); with paired columns (PC) it holds
// head t alone, in o[m][0] and o[m][2], and l1 is unused.  out = c_B * H_blk
// (o / l): the normalised block Hadamard is its own inverse.
template <int D, bool MULTI, bool PC = false>
__device__ __forceinline__ void store_head(const AttnParams& p, int b, int hkv, int lane, float (&o)[D / 16][4],
                                           float l0, float l1) {
  constexpr int NM = D / 16;
  constexpr int IS = PC ? 2 : 1;   // step over the lane's o[m][i] that hold values
  const int g8 = lane >> 2, t = lane & 3;
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int m = 0; m < NM; ++m) {
    o[m][0] *= inv0; o[m][2] *= inv0;
    if constexpr (!PC) { o[m][1] *= inv1; o[m][3] *= inv1; }
  }
  const int Bh = p.Bh_o;
  // stages 1, 2, 4: dimension bits 0-2 are the lane bits 2-4
#pragma unroll
  for (int hh = 1; hh <= 4; hh <<= 1) {
    if (hh < Bh) {
      const bool upper = (g8 & hh) != 0;
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int i = 0; i < 4; i += IS) {
          const float other = __shfl_xor_sync(0xffffffffu, o[m][i], 4 * hh);
          o[m][i] = upper ? other - o[m][i] : o[m][i] + other;
        }
    }
  }
  // stage 8: dimension bit 3 (o[m][0..1] vs o[m][2..3])
  if (8 < Bh) {
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int i = 0; i < 2; i += IS) {
        const float a = o[m][i], c = o[m][i + 2];
        o[m][i] = a + c;
        o[m][i + 2] = a - c;
      }
  }
  // stages 16, 32, ...: dimension bits 4.. (m)
#pragma unroll
  for (int mb = 1; mb < NM; mb <<= 1) {
    if (16 * mb < Bh) {
#pragma unroll
      for (int m = 0; m < NM; ++m)
        if ((m & mb) == 0)
#pragma unroll
          for (int i = 0; i < 4; i += IS) {
            const float a = o[m][i], c = o[m + mb][i];
            o[m][i] = a + c;
            o[m + mb][i] = a - c;
          }
    }
  }
  const float rc = p.rc_o;
  const int G = p.G;
#pragma unroll
  for (int hp = 0; hp < (PC ? 1 : 2); ++hp) {
    const int head = PC ? t : 2 * t + hp;
    if (head >= G) continue;
    const long long row = (MULTI ? q_row(p, b, hkv, head) : static_cast<long long>(b) * p.Hq + hkv * G + head) * D;
    if (p.mode & KV4_MODE_OUT_F32) {
      float* out = static_cast<float*>(p.out) + row;
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        out[16 * m + g8] = o[m][hp] * rc;
        out[16 * m + g8 + 8] = o[m][hp + 2] * rc;
      }
    } else {
      uint16_t* out = static_cast<uint16_t*>(p.out) + row;
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        out[16 * m + g8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[m][hp] * rc));
        out[16 * m + g8 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(o[m][hp + 2] * rc));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// query operands: one warp per (batch entry, KV head) rotates its G query
// heads and stores the integer tensor-core B fragments of both query planes,
// sum(q) per fragment column and the exponent scale.  The attention kernel is
// launched as its programmatic dependent, so it plans and starts streaming
// pages while this runs, and waits for it only before the first operand read.

constexpr int QWARPS = 4;

template <int D>
__global__ void __launch_bounds__(32 * QWARPS) gq_kernel(AttnParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * QWARPS + (threadIdx.x >> 5);
  if (gw >= p.n_seqs * p.Hkv) return;
  QFrag<D> qf;
  load_qfrag<D>(p, gw / p.Hkv, gw % p.Hkv, lane, qf);
  uint8_t* blob = p.qblob + static_cast<size_t>(gw) * qblob_bytes(D);
  if constexpr (D == 128) {
    if (p.qfmt == 1) store_qblob_tc<D>(blob, qf, lane);
    else store_qblob<D>(blob, qf, lane, p.qfmt == 3);
  } else {
    store_qblob<D>(blob, qf, lane, p.qfmt == 3);
  }
}

// ---------------------------------------------------------------------------
// fused decode step, first kernel: one block per batch entry, two warps per
// KV head.  Warp (tensor, h) appends the entry's new token of head h, K for
// tensor 0 and V for tensor 1 (rotate, quantize, INT4 page and INT8 ring);
// the V warp also builds the query operands of head h as gq_kernel does (RoPE
// of q, when asked, at the new length).  Each warp loads its new row before
// the sequence's state arrives.  The block advances the sequence length at
// the end; the attention kernel follows in stream order, so it sees the new
// token and the new length.

// MAXW: the most warps a block of this instantiation has (2 * Hkv <= MAXW);
// 16 for up to 8 KV heads (128 registers a thread), 32 for up to 16.
template <int D, int MAXW>
__global__ void __launch_bounds__(32 * MAXW, 32 / MAXW) gstep_kernel(AttnParams p, AppendParams ap) {
  constexpr int VPL = D / 32;
  __shared__ __align__(16) uint8_t s_codes[MAXW][2][D];
  __shared__ int s_seq, s_L, s_ok, s_page;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tensor = warp >= p.Hkv ? 1 : 0, h = warp - tensor * p.Hkv;
  const int b = blockIdx.x;
  // the attention kernel may be scheduled as blocks of this grid retire (it waits for the whole grid)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this warp's new row: k_new / v_new [n_seqs][Hkv][D], entry b
  uint16_t raw[VPL];
  {
    const uint16_t* src = (tensor ? ap.v_new : ap.k_new) + (static_cast<long long>(b) * p.Hkv + h) * D + VPL * lane;
#pragma unroll
    for (int k = 0; k < VPL; ++k) raw[k] = src[k];
  }
  if (threadIdx.x == 0) {
    const int seq = p.seq_ids[b];
    int ok = seq >= 0 && seq < p.max_seqs;
    if (!ok) atomicOr(&p.state->status, KV4_DEV_BAD_SEQ);
    const int L = ok ? p.seq_lens[seq] : 0;
    if (ok && L + 1 > p.max_pages_per_seq * p.P) {
      atomicOr(&p.state->status, KV4_DEV_OVERFLOW);
      ok = 0;
    }
    int page = -1;
    if (ok) {
      page = p.block_table[static_cast<long long>(seq) * p.max_pages_per_seq + L / p.P];
      if (page < 0 || page >= p.num_pages) {
        atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
        page = -1;
      }
    }
    s_seq = seq;
    s_L = L;
    s_ok = ok;
    s_page = page;
  }
  __syncthreads();
  const int seq = s_seq, L = s_L, page = s_page;
  if (tensor == 1) {   // the query operands of head h (independent of the append)
    QFrag<D> qf;
    load_qfrag<D>(p, b, h, lane, qf, s_ok ? L + 1 : L);
    uint8_t* blob = p.qblob + (static_cast<size_t>(b) * p.Hkv + h) * qblob_bytes(D);
    if constexpr (D == 128) {
      if (p.qfmt == 1) store_qblob_tc<D>(blob, qf, lane);
      else store_qblob<D>(blob, qf, lane, p.qfmt == 3);
    } else {
      store_qblob<D>(blob, qf, lane, p.qfmt == 3);
    }
  }
  if (s_ok && page >= 0) {
    const long long tile_idx = (static_cast<long long>(page) * (p.P / TILE) + (L % p.P) / TILE) * p.Hkv + h;
    const bool rope_past = tensor == 0 && ap.rope.cs != nullptr && L >= ap.rope.max_pos;
    if (rope_past && lane == 0) atomicOr(&p.state->status, KV4_DEV_ROPE_POS);
    if (!rope_past)
      encode_row<D>(ap, raw, tensor, h, seq, L, L + 1, tile_idx, L & (TILE - 1), s_codes[warp][0], s_codes[warp][1],
                    lane);
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_ok) ap.seq_lens[seq] = L + 1;
}

// ---------------------------------------------------------------------------
// the attention kernel

template <int D, int GWR, int F>
__device__ __forceinline__ const uint8_t* stage_source(const AttnParams& p, const Group& g, int u, uint32_t& bytes) {
  using C = GCfg<D, GWR, F>;
  using SH = GShape<GWR>;
  if (u < g.n4) {
    const int pos = (g.t0 + u) * TILE;
    int page = p.block_table[static_cast<long long>(g.seq) * p.max_pages_per_seq + pos / p.P];
    if (page < 0 || page >= p.num_pages) {
      atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
      page = 0;
    }
    bytes = C::STAGE4;
    return p.pool + ((static_cast<long long>(page) * (p.P / TILE) + (pos % p.P) / TILE) * p.Hkv + g.hg * GWR) *
                        page_tile_bytes(D, F);
  }
  // part (v % S8) of protected tile v / S8: heads H8 * (v % S8) .. of the group
  const int v = u - g.n4;
  bytes = C::STAGE8;
  return p.prot + ((static_cast<long long>(g.seq) * n_prot_tiles(p.S, p.W) + v / SH::S8) * p.Hkv + g.hg * GWR +
                   (v % SH::S8) * SH::H8) *
                      tile8_bytes(D);
}

// The CTA's share of the stream-K split.  Every CTA derives the same plan
// from the sequence lengths: the costs of all head groups (a block scan) give
// T, and CTA c takes units [c*T/N, (c+1)*T/N).  Group i spans
// [S_i, S_i + GROUP_COST + n_i) in cost units; its stage u sits at
// S_i + GROUP_COST + u.  The CTA whose range holds a group's start records the
// group in `plan` (for the merge kernel), CTA 0 the totals; empty sequences get
// zero rows.  misc->first = the group holding the CTA's first unit.  Called by
// every thread of the block; returns whether the CTA has stages to stream.
template <int GWR>
__device__ bool plan_share(const AttnParams& p, GPlanRec* plan, GMisc* misc, int c, int tid, int nthreads,
                           long long& T_out, long long& N_out, int& j0_out, int& j1_out) {
  const int HGN = p.Hkv / GWR, n_groups = p.n_seqs * HGN;
  // ---- plan (every CTA the same): costs of all head groups -> T, then the
  // stream-K range [j0, j1) of this CTA and the group holding j0.  Group i
  // spans [S_i, S_i + GROUP_COST + n_i) in cost units; its stage u sits at
  // S_i + GROUP_COST + u.
  Group my_g{};
  int my_start = 0, T = 0;
  for (int c0 = 0; c0 < n_groups; c0 += nthreads) {
    const int i = c0 + tid;
    Group gd{};
    if (i < n_groups) gd = describe(p, i, HGN, c == 0);
    int tot;
    const int ex = block_exclusive_scan(group_cost<GWR>(gd), misc->red, &tot);
    if (c0 == 0) { my_g = gd; my_start = ex; }
    T += tot;
  }
  long long N = (T + MIN_STAGES - 1) / MIN_STAGES;   // active CTAs: each owns at least one stage
  if (N > p.grid) N = p.grid;
  const bool zero_all = T == 0;
  const int j0 = zero_all ? 0 : static_cast<int>(c * static_cast<long long>(T) / N);
  const int j1 = zero_all ? 0 : static_cast<int>((c + 1) * static_cast<long long>(T) / N);
  auto visit = [&](int i, const Group& gd, int st) {
    if (i >= n_groups) return;
    const int n = group_cost<GWR>(gd);
    if (n > 0) {
      if (st <= j0 && j0 < st + n) {
        misc->first = gd;
        misc->first.start = st;
      }
      if (st >= j0 && st < j1) plan[i] = GPlanRec{st, group_stages<GWR>(gd)};
    } else {
      const int owner = zero_all ? 0 : cta_of(min(st, T - 1), T, N);
      if (owner == c) {
        plan[i] = GPlanRec{st, 0};
        const int k = atomicAdd(&misc->n_empty, 1);
        if (k < 32) misc->empty[k] = i;
        else zero_group<GWR>(p, i, 0, 1);
      }
    }
  };
  if (n_groups <= nthreads) {
    visit(tid, my_g, my_start);
  } else {
    int base = 0;
    for (int c0 = 0; c0 < n_groups; c0 += nthreads) {
      const int i = c0 + tid;
      Group gd{};
      if (i < n_groups) gd = describe(p, i, HGN, false);
      int tot;
      const int ex = block_exclusive_scan(group_cost<GWR>(gd), misc->red, &tot);
      visit(i, gd, base + ex);
      base += tot;
    }
  }
  if (c == 0 && tid == 0) {
    GPlanHdr* hdr = reinterpret_cast<GPlanHdr*>(plan + n_groups);
    hdr->T = T;
    hdr->N = static_cast<int>(N);
  }
  __syncthreads();
  {
    const int ne = min(misc->n_empty, 32);
    for (int e = 0; e < ne; ++e) zero_group<GWR>(p, misc->empty[e], tid, nthreads);
  }
  T_out = T;
  N_out = N;
  j0_out = j0;
  j1_out = j1;
  return !(zero_all || c >= N || j0 >= j1);
}

// The producer warp of a CTA: walks the CTA's range [j0, j1) of the split,
// queues one segment descriptor per head group it touches, and issues the
// group's stages as 1-D bulk copies into the shared-memory ring (each lane one
// stage of a batch, mbarrier completion).  Consumers release a stage once per
// group of consumers (the empty barriers count GWR arrivals).  Every wait is
// bounded; before the warp exits, every copy it issued has landed.
template <int D, int GWR, int F = 0>
__device__ void produce(const AttnParams& p, GMisc* misc, SegQ* segq, uint8_t* ring, int NS, uint32_t full0,
                        uint32_t empty0, uint32_t iqf0, uint32_t iqe0, int c, int j0, int j1, long long T, long long N,
                        int lane, volatile int* abort_flag, int* status) {
  using C = GCfg<D, GWR, F>;
  const int HGN = p.Hkv / GWR;
  // ------------------------------------------------------------ producer
  const int nbatch = NS < 32 ? NS : 32;
  Group g = misc->first;
  int gi = g.b * HGN + g.hg;
  int j = j0;        // position in cost units
  uint32_t jj = 0;   // CTA-local stage counter
  int q = 0;
  bool ok = true;
  while (j < j1 && ok) {
    const int gst = group_stages<GWR>(g);
    const int a = g.start + GROUP_COST, e = a + gst;   // the group's stages in cost units
    if (a >= j1) break;                                // only its start cost falls in this range
    const int u = max(j, a) - a;
    const int n = min(e, j1) - max(j, a);
    const int slot = q % GQD;
    if (lane == 0) ok = mbar_wait(iqe0 + 8 * slot, ((q / GQD) & 1) ^ 1, abort_flag, status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    if (lane == 0) {
      SegQ sq;
      sq.g = g;
      sq.u0 = u;
      sq.n = n;
      const int cf = cta_of(a, T, N);
      sq.k = c - cf;
      sq.nseg = cta_of(e - 1, T, N) - cf + 1;
      segq[slot] = sq;
      mbar_arrive(iqf0 + 8 * slot);
    }
    // the next group's descriptor (its loads overlap the copies below)
    int gn = gi + 1;
    Group nxt{};
    if (e < j1) nxt = describe(p, gn, HGN, false);
    // stages u .. u+n-1: one lane per stage, batches of at most NS stages
    for (int base = 0; base < n; base += nbatch) {
      bool lane_ok = true;
      if (lane < nbatch && base + lane < n) {
        uint32_t bytes;
        const uint8_t* src = stage_source<D, GWR, F>(p, g, u + base + lane, bytes);
        const uint32_t jl = jj + base + lane;
        const int s = jl % NS;
        lane_ok = mbar_wait(empty0 + 8 * s, ((jl / NS) & 1) ^ 1, abort_flag, status);
        if (lane_ok) {
          // test hook (kv4_test_stall_next_attention): the first CTA leaves one stage unfilled, so its
          // consumers' bounded wait runs out
          if (c != 0 || static_cast<int>(jl) != p.stall_stage) {
            mbar_arrive_expect_tx(full0 + 8 * s, bytes);
            bulk_g2s(smem_u32(ring + static_cast<size_t>(s) * C::STAGE), src, bytes, full0 + 8 * s);
            misc->last_fill[s] = static_cast<int>(jl);
          }
        } else {
          *abort_flag = 1;
        }
      }
      ok = __all_sync(0xffffffffu, lane_ok);
      if (!ok) break;
    }
    jj += n;
    j = e;
    ++q;
    if (j < j1 && ok) {
      while (group_stages<GWR>(nxt) == 0) nxt = describe(p, ++gn, HGN, false);   // empty sequences own no stage
      nxt.start = e;
      gi = gn;
      g = nxt;
    }
  }
  if (ok) {
    const int slot = q % GQD;
    if (lane == 0) ok = mbar_wait(iqe0 + 8 * slot, ((q / GQD) & 1) ^ 1, abort_flag, status);
    if (lane == 0 && ok) { segq[slot].n = -1; mbar_arrive(iqf0 + 8 * slot); }
    ok = __shfl_sync(0xffffffffu, ok, 0);
  }
  if (lane == 0) {
    // let every copy this warp issued land before it exits: consumers that gave up a wait may have left
    // the CTA already, and its shared memory must not go away under a copy in flight
    for (int st = 0; st < NS; ++st)
      if (misc->last_fill[st] >= 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(full0 + 8 * st, (misc->last_fill[st] / NS) & 1) &&
               globaltimer_ns() - t0 < 1000000000ull) {}
      }
  }
}

// PAIR = INT4 tiles per iteration of a consumer warp (1, 2 or 4).  MULTI:
// several query tokens per sequence (causal visibility per operand column);
// the one-token variant carries none of that code.  GWR: KV heads per group.
// F: page format (0 INT4, 1 NVFP4, 2 INT2; the INT8 store is the same).
// PCOL: paired columns (one query token, at most 4 query heads per KV head,
// integer query planes; see unit_int4_pc).
template <int D, int PAIR, bool MULTI, int GWR, int F = 0, bool PCOL = false>
__global__ void __maxnreg__(128) gattn_kernel(AttnParams p, GPlanRec* plan) {
  static_assert(!PCOL || (!MULTI && F != 1), "paired columns: one query token, integer query planes");
  using C = GCfg<D, GWR, F>;
  using SH = GShape<GWR>;
  constexpr int GTHREADS = SH::THREADS;
  extern __shared__ __align__(128) uint8_t smem[];
  const int NS = p.ns;
  uint8_t* ring = smem;
  SegQ* segq = reinterpret_cast<SegQ*>(ring + static_cast<size_t>(NS) * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(segq + GQD);
  GMisc* misc = reinterpret_cast<GMisc*>(bars + 2 * NS + 2 * GQD);
  volatile int* abort_flag = &misc->abort;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * NS;
  const uint32_t iqf0 = full0 + 16 * NS, iqe0 = iqf0 + 8 * GQD;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* status = &p.state->status;
  const int c = blockIdx.x;

  // the merge kernel may be scheduled now: it waits for this grid before reading its results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // after the fused step kernel: its lengths, pages and query operands are written once that grid is done
  if (p.wait_first) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, GWR); }
    for (int s = 0; s < GQD; ++s) { mbar_init(iqf0 + 8 * s, 1); mbar_init(iqe0 + 8 * s, GWR); }
    misc->abort = 0;
    misc->n_empty = 0;
    for (int s = 0; s < MAX_NS; ++s) misc->last_fill[s] = -1;
    fence_barrier_init();
  }

  long long T = 0, N = 0;
  int j0 = 0, j1 = 0;
  if (!plan_share<GWR>(p, plan, misc, c, tid, GTHREADS, T, N, j0, j1)) return;

  if (warp == GWR) {
    produce<D, GWR, F>(p, misc, segq, ring, NS, full0, empty0, iqf0, iqe0, c, j0, j1, T, N, lane, abort_flag,
                       status);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int w = warp;   // KV head within the group
  const int g8 = lane >> 2, t = lane & 3;
  const int G = p.G;
  constexpr int HS = head_stride(D);
  const int pstride = partial_stride(G, D);
  ColSplit cs;
  cs.colsplit = (G == 1 || G == 2 || G == 4);
  cs.part0 = cs.colsplit ? (2 * t) / G : 0;
  cs.part1 = cs.colsplit ? (2 * t + 1) / G : 0;
  const int h0 = 2 * t, h1 = 2 * t + 1;
  // query token of the thread's columns (the last qlen positions are the
  // query tokens; token i sees the positions up to L - qlen + i)
  const int qt0 = MULTI ? (cs.colsplit ? h0 % G : h0) / p.Gh : 0;
  const int qt1 = MULTI ? (cs.colsplit ? h1 % G : h1) / p.Gh : 0;
  int s = 0;          // stage of the next CTA-local stage index
  uint32_t par = 0;   // its fill parity

  auto advance = [&]() {
    if (++s == NS) { s = 0; par ^= 1u; }
  };
  for (int q = 0;; ++q) {
    const int slot = q % GQD;
    if (!mbar_wait(iqf0 + 8 * slot, (q / GQD) & 1, abort_flag, status)) break;
    const SegQ sq = segq[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(iqe0 + 8 * slot);
    if (sq.n < 0) break;
    const Group& g = sq.g;
    if (q == 0) asm volatile("griddepcontrol.wait;" ::: "memory");   // the query operands are written
    QFrag<D> qf;
    {
      const uint8_t* blob = p.qblob + static_cast<size_t>(g.b * p.Hkv + g.hg * GWR + w) * qblob_bytes(D);
#pragma unroll
      for (int cc = 0; cc < (PCOL ? D / 64 : D / 32); ++cc) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(blob) + 32 * cc + lane);
        qf.b[2 * cc][0] = v.x; qf.b[2 * cc][1] = v.y; qf.b[2 * cc + 1][0] = v.z; qf.b[2 * cc + 1][1] = v.w;
      }
      const float* tail = reinterpret_cast<const float*>(blob + 16 * D);
      qf.qs0 = __ldcg(tail + 2 * t);
      qf.qs1 = __ldcg(tail + 2 * t + 1);
      qf.kscale = __ldcg(tail + MAX_G);
    }

    WarpState<D> ws;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) ws.o[m][0] = ws.o[m][1] = ws.o[m][2] = ws.o[m][3] = 0.f;
    ws.m0 = ws.m1 = NEG_INF;
    ws.l0 = ws.l1 = ws.z0 = ws.z1 = 0.f;

    const int u_end = sq.u0 + sq.n;
    bool ok = true;
    for (int u = sq.u0; u < u_end && ok;) {
      if (u < g.n4) {
        // PAIR INT4 stages at once when the segment has that many left, else one:
        // the tiles of this warp's head
        const int avail = min(u_end, g.n4) - u;
        const int nt = avail >= PAIR ? PAIR : 1;
        uint32_t tl[PAIR], eb[PAIR];
        int valid[PAIR];
#pragma unroll
        for (int k = 0; k < PAIR; ++k) {
          if (k < nt) {
            tl[k] = smem_u32(ring + static_cast<size_t>(s) * C::STAGE + w * page_tile_bytes(D, F));
            eb[k] = empty0 + 8 * s;
            if (ok) ok = mbar_wait(full0 + 8 * s, par, abort_flag, status);
            advance();
          } else {
            tl[k] = tl[0];
            eb[k] = eb[0];
          }
        }
        if (!ok) break;
        const int pos0 = (g.t0 + u) * TILE;
        const int vis = MULTI ? g.L - p.qtot + p.q0 : g.L - 1;   // the last position every column sees
        const bool inside = pos0 >= g.lo4 && pos0 + nt * TILE <= (MULTI ? min(g.hi4, vis + 1) : g.hi4);
        if (inside) {
#pragma unroll
          for (int k = 0; k < PAIR; ++k) valid[k] = 15;
          if constexpr (F == 1) {
            if (nt == PAIR) unit_fp4<D, PAIR, false>(tl, qf, ws, lane, valid, valid, eb, cs);
            else unit_fp4<D, 1, false>(tl, qf, ws, lane, valid, valid, eb, cs);
          } else if constexpr (PCOL) {
            constexpr int BITS = F == 2 ? 2 : 4;
            if (nt == PAIR) unit_int4_pc<D, PAIR, false, BITS>(tl, qf, ws, lane, valid, eb);
            else unit_int4_pc<D, 1, false, BITS>(tl, qf, ws, lane, valid, eb);
          } else {
            constexpr int BITS = F == 2 ? 2 : 4;
            if (nt == PAIR) unit_int4<D, PAIR, false, false, BITS>(tl, qf, ws, lane, valid, eb, cs);
            else unit_int4<D, 1, false, false, BITS>(tl, qf, ws, lane, valid, eb, cs);
          }
        } else {
#pragma unroll
          for (int k = 0; k < PAIR; ++k) {
            const int pg = pos0 + k * TILE + g8;
            const bool r0 = pg >= g.lo4 && pg < g.hi4, r8 = pg + 8 >= g.lo4 && pg + 8 < g.hi4;
            if constexpr (MULTI)
              valid[k] = (r0 && pg <= vis + qt0 ? 1 : 0) | (r0 && pg <= vis + qt1 ? 2 : 0) |
                         (r8 && pg + 8 <= vis + qt0 ? 4 : 0) | (r8 && pg + 8 <= vis + qt1 ? 8 : 0);
            else
              valid[k] = (r0 ? 3 : 0) | (r8 ? 12 : 0);
          }
          if constexpr (F == 1) {
            int nwr[PAIR];   // written slots of each tile (the sequence's positions below L)
#pragma unroll
            for (int k = 0; k < PAIR; ++k) nwr[k] = min(max(g.L - (pos0 + k * TILE), 0), TILE);
            if (nt == PAIR) unit_fp4<D, PAIR, true, MULTI>(tl, qf, ws, lane, valid, nwr, eb, cs);
            else unit_fp4<D, 1, true, MULTI>(tl, qf, ws, lane, valid, nwr, eb, cs);
          } else if constexpr (PCOL) {
            constexpr int BITS = F == 2 ? 2 : 4;
            if (nt == PAIR) unit_int4_pc<D, PAIR, true, BITS>(tl, qf, ws, lane, valid, eb);
            else unit_int4_pc<D, 1, true, BITS>(tl, qf, ws, lane, valid, eb);
          } else {
            constexpr int BITS = F == 2 ? 2 : 4;
            if (nt == PAIR) unit_int4<D, PAIR, true, MULTI, BITS>(tl, qf, ws, lane, valid, eb, cs);
            else unit_int4<D, 1, true, MULTI, BITS>(tl, qf, ws, lane, valid, eb, cs);
          }
        }
        u += nt;
      } else {
        // one INT8 stage: part (v % S8) of protected tile v / S8 holds heads H8*(v % S8) .. +H8-1
        const int v = u - g.n4;
        const int s0 = s;
        const uint32_t p0 = par;
        advance();
        ok = mbar_wait(full0 + 8 * s0, p0, abort_flag, status);
        if (!ok) break;
        const uint32_t eb = empty0 + 8 * s0;
        if (v % SH::S8 == w / SH::H8) {
          const uint32_t st = smem_u32(ring + static_cast<size_t>(s0) * C::STAGE + (w % SH::H8) * tile8_bytes(D));
          const int slot0 = (v / SH::S8) * TILE;
          if constexpr (PCOL) {
            if (slot0 + TILE <= g.nprot) tile_int8_pc<D, false>(st, qf, ws, lane, 15, eb);
            else tile_int8_pc<D, true>(st, qf, ws, lane, (slot0 + g8 < g.nprot ? 3 : 0) | (slot0 + g8 + 8 < g.nprot ? 12 : 0), eb);
          } else if (slot0 + TILE <= g.nprot && !MULTI) {
            tile_int8<D, false, false, F == 1>(st, qf, ws, lane, 15, eb, cs);
          } else if (!MULTI) {
            tile_int8<D, true, false, F == 1>(st, qf, ws, lane,
                                              (slot0 + g8 < g.nprot ? 3 : 0) | (slot0 + g8 + 8 < g.nprot ? 12 : 0),
                                              eb, cs);
          } else {
            // position of protected slot sl: a sink below S, else the ring position
            // in [max(S, L - W), L) congruent to sl - S modulo W
            const int rlo = max(p.S, g.L - p.W), vis = g.L - p.qtot + p.q0;
            auto pos_of = [&](int sl) {
              return sl < p.S ? sl : rlo + (((sl - p.S) - (rlo - p.S)) % p.W + p.W) % p.W;
            };
            const int sa = slot0 + g8, sb = sa + 8;
            const bool ra = sa < g.nprot, rb = sb < g.nprot;
            const int pa = pos_of(sa), pb = pos_of(sb);
            const int vm = (ra && pa <= vis + qt0 ? 1 : 0) | (ra && pa <= vis + qt1 ? 2 : 0) |
                           (rb && pb <= vis + qt0 ? 4 : 0) | (rb && pb <= vis + qt1 ? 8 : 0);
            tile_int8<D, true, true, F == 1>(st, qf, ws, lane, vm, eb, cs);
          }
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(eb);
        }
        u += 1;
      }
    }
    if (!ok) break;

    // ---- the segment's result for this warp's head
    if constexpr (PCOL) {
      // head t: its two column sums, then l and the zero-point sum over the lane's row groups
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { ws.o[m][0] += ws.o[m][1]; ws.o[m][2] += ws.o[m][3]; }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        ws.l0 += __shfl_xor_sync(0xffffffffu, ws.l0, o);
        ws.z0 += __shfl_xor_sync(0xffffffffu, ws.z0, o);
      }
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { ws.o[m][0] += ws.z0; ws.o[m][2] += ws.z0; }
      const int hkv = g.hg * GWR + w;
      if (sq.nseg == 1) {
        store_head<D, false, true>(p, g.b, hkv, lane, ws.o, ws.l0, 0.f);
        continue;
      }
      const int slotp = (c * 2 + (q == 0 ? 0 : 1)) * GWR + w;
      if (t < G) {
        float* r = p.partials + static_cast<size_t>(slotp) * pstride + t * HS;
#pragma unroll
        for (int m = 0; m < D / 16; ++m) { r[16 * m + g8] = ws.o[m][0]; r[16 * m + g8 + 8] = ws.o[m][2]; }
        if (g8 == 0) { r[D] = ws.m0; r[D + 1] = ws.l0; }
      }
      continue;
    }
    if (cs.colsplit) {
      if (G == 1) {
#pragma unroll
        for (int m = 0; m < D / 16; ++m) { ws.o[m][0] += ws.o[m][1]; ws.o[m][2] += ws.o[m][3]; }
      } else {
        const int x = G == 4 ? 2 : 1;
#pragma unroll
        for (int m = 0; m < D / 16; ++m)
#pragma unroll
          for (int i = 0; i < 4; ++i) ws.o[m][i] += __shfl_xor_sync(0xffffffffu, ws.o[m][i], x);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      ws.l0 += __shfl_xor_sync(0xffffffffu, ws.l0, o);
      ws.l1 += __shfl_xor_sync(0xffffffffu, ws.l1, o);
      ws.z0 += __shfl_xor_sync(0xffffffffu, ws.z0, o);
      ws.z1 += __shfl_xor_sync(0xffffffffu, ws.z1, o);
    }
#pragma unroll
    for (int m = 0; m < D / 16; ++m) { ws.o[m][0] += ws.z0; ws.o[m][2] += ws.z0; ws.o[m][1] += ws.z1; ws.o[m][3] += ws.z1; }
    const int hkv = g.hg * GWR + w;
    if (sq.nseg == 1) {
      store_head<D, MULTI>(p, g.b, hkv, lane, ws.o, ws.l0, ws.l1);
      continue;
    }
    // several CTAs share the group: its partial to the workspace (slot 0 = this
    // CTA's first segment, slot 1 = its last), merged by the merge kernel
    const int slotp = (c * 2 + (q == 0 ? 0 : 1)) * GWR + w;
    float* part = p.partials + static_cast<size_t>(slotp) * pstride;
    if (h0 < G) {
      float* r = part + h0 * HS;
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { r[16 * m + g8] = ws.o[m][0]; r[16 * m + g8 + 8] = ws.o[m][2]; }
      if (g8 == 0) { r[D] = ws.m0; r[D + 1] = ws.l0; }
    }
    if (h1 < G) {
      float* r = part + h1 * HS;
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { r[16 * m + g8] = ws.o[m][1]; r[16 * m + g8 + 8] = ws.o[m][3]; }
      if (g8 == 0) { r[D] = ws.m1; r[D + 1] = ws.l1; }
    }
  }
}

// ---------------------------------------------------------------------------
// merge of the split groups: one warp per (batch entry, query head).  Launched
// as the programmatic dependent of the attention kernel, so its blocks are
// resident before the attention grid ends; it waits for that grid first.

constexpr int MWARPS = 8;

template <int D, int GWR>
__global__ void __launch_bounds__(32 * MWARPS) gmerge_kernel(AttnParams p, const GPlanRec* plan) {
  constexpr int VPL = D / 32;
  constexpr int HS = head_stride(D);
  constexpr int U = 8;   // segments in flight
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * MWARPS + (threadIdx.x >> 5);
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the partials and the plan are written
  const int G = p.G, HGN = p.Hkv / GWR, per_b = p.Hkv * G;   // G: operand columns (query tokens x heads)
  if (gw >= p.n_seqs * per_b) return;
  const int b = gw / per_b, r = gw - b * per_b, hkv = r / G, gq = r - hkv * G;
  const int hg = hkv / GWR, w = hkv - hg * GWR;
  const GPlanHdr* hdr = reinterpret_cast<const GPlanHdr*>(plan + p.n_seqs * HGN);
  const long long T = __ldcg(&hdr->T), N = __ldcg(&hdr->N);
  const GPlanRec rec = {__ldcg(&plan[b * HGN + hg].start), __ldcg(&plan[b * HGN + hg].stages)};
  if (rec.stages == 0 || N <= 0) return;   // empty sequence: zero rows written by the attention kernel
  const int a = rec.start + GROUP_COST, e = a + rec.stages;
  const int cf = cta_of(a, T, N);
  const int nseg = cta_of(e - 1, T, N) - cf + 1;
  if (nseg == 1) return;                   // stored by the attention kernel
  // segment k sits on CTA cf + k, in its slot 0 (its first segment) or slot 1 (its last)
  const bool first_is_last = cf * T / N < rec.start;
  const int pstride = partial_stride(G, D);
  auto row = [&](int k) -> const float* {
    const int sl = (k == 0 && first_is_last) ? 1 : 0;
    return p.partials + static_cast<size_t>(((cf + k) * 2 + sl) * GWR + w) * pstride + gq * HS;
  };
  float M = NEG_INF;
  for (int k = lane; k < nseg; k += 32) M = fmaxf(M, __ldcg(row(k) + D));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[VPL], L = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  for (int k0 = 0; k0 < nseg; k0 += U) {
    float v[U][VPL], mv[U], lv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float* r = row(min(k0 + u, nseg - 1));
      mv[u] = __ldcg(r + D);
      lv[u] = __ldcg(r + D + 1);
      if constexpr (VPL == 4) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(r) + lane);
        v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
      } else {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(r) + lane);
        v[u][0] = x.x; v[u][1] = x.y;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      // a segment (or a column) with no visible position has m = -inf
      const float f = (k0 + u < nseg && mv[u] != NEG_INF) ? ex2(mv[u] - M) : 0.f;
      L = fmaf(f, lv[u], L);
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc[i] = fmaf(f, v[u][i], acc[i]);
    }
  }
  float o[VPL];
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) o[i] = acc[i] * inv;
  fwht_row<VPL>(o, p.Bh_o, lane);   // o = H_blk o_rot (the normalised block Hadamard is its own inverse)
  const float rc = p.rc_o;
  const long long off = q_row(p, b, hkv, gq) * D + VPL * lane;
  if (p.mode & KV4_MODE_OUT_F32) {
    float* out = static_cast<float*>(p.out) + off;
    if constexpr (VPL == 4) *reinterpret_cast<float4*>(out) = make_float4(o[0] * rc, o[1] * rc, o[2] * rc, o[3] * rc);
    else *reinterpret_cast<float2*>(out) = make_float2(o[0] * rc, o[1] * rc);
  } else {
    uint16_t* out = static_cast<uint16_t*>(p.out) + off;
    if constexpr (VPL == 4)
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf162(o[0] * rc, o[1] * rc), pack_bf162(o[2] * rc, o[3] * rc));
    else
      *reinterpret_cast<uint32_t*>(out) = pack_bf162(o[0] * rc, o[1] * rc);
  }
}

// ---------------------------------------------------------------------------
// The attention kernel on the fifth-generation tensor cores (tcgen05, operands
// and accumulators in tensor memory), for 4-KV-head groups at D = 128 and one
// query token.  Same split, producer warp, stage ring and merge kernel as
// gattn_kernel; one CTA per SM with four consumer warpgroups, warpgroup h
// handling KV head h of every stage, 128 tokens (8 tiles) per block:
//   K phase   thread i = token i of the block: its 128 K codes as bytes
//             (INT4 nibbles unpacked; INT8 rows as stored) to TMEM lane i;
//   scores    16 multiplies M=128 tokens x N=8 x K=32 (kind::i8, A = codes in
//             TMEM, B = the two 8-bit planes of the rotated query in shared
//             memory) -> int32 scores in TMEM, one token per thread;
//   softmax   per token and query head, no column duplicates; the running max
//             is kept per warpgroup and moved only when a score passes it by
//             more than TAU (a vote), so most blocks need no reduction;
//   weights   w = p * s_V as 32-bit fixed point (F = 2^(32-TAU) / s_ref, s_ref
//             an upper bound of the V scales seen), stored as 4 bytes per
//             head: the four byte planes of 4 heads are the N = 16 columns;
//   V phase   thread i = dim i: its 16 codes of every tile as bytes to TMEM;
//   P.V       4 multiplies M=128 dims x N=16 x K=32 tokens (kind::i8) into an
//             exact int32 accumulator in TMEM, folded into fp32 per-dim sums
//             only when the max or s_ref moves and at the end of a segment.
// The zero points enter through sum_p p z (exact fp32 per token) and the scale
// of K through the per-token factor of the integer score, as in the folded
// form of the other kernels.

constexpr int TC_WG = 4;                           // consumer warpgroups = KV heads of a group
constexpr int TC_THREADS = 32 * (4 * TC_WG + 1);   // + producer warp
constexpr int TC_BLOCK = 8;                        // 16-token tiles per block (128 tokens = TMEM lanes)
constexpr uint32_t TC_COLS = 512;                  // TMEM columns of the CTA, 128 per warpgroup
constexpr uint32_t TC_AK = 0;                      // QK A operand: 128 tokens x 128 code bytes (32 columns)
constexpr uint32_t TC_S = 32;                      // scores: hi query plane 32..39, lo plane 40..47
constexpr uint32_t TC_AV = 48;                     // P.V A operands, two buffers of 32 columns
constexpr uint32_t TC_O = 112;                     // P.V accumulator: 4 heads x 4 byte planes
constexpr int TC_QB = 2048;                        // query planes: hi 1 KB, lo 1 KB (K-major, N = 8)
constexpr int TC_PB = 2048;                        // one weight buffer: 128 tokens x 16 bytes (MN-major)
constexpr int TC_SCR = 2048;                       // reduction / rotation scratch
constexpr int TC_WGSMEM = TC_QB + 2 * TC_PB + TC_SCR;
constexpr float TC_TAU = 2.f;                      // allowed excess of a score over the running max (log2)
constexpr int TC_FLUSH_BLOCKS = 512;               // fold the int32 accumulator at least every 65536 tokens
constexpr uint32_t TC_IDESC_QK_HI = tc::idesc_i8(8, true, false);
constexpr uint32_t TC_IDESC_QK_LO = tc::idesc_i8(8, false, false);
constexpr uint32_t TC_IDESC_PV = tc::idesc_i8(16, false, true);

template <int D>
__host__ __device__ inline size_t tattn_smem_bytes(int ns) {
  using C = GCfg<D, 4>;
  size_t off = static_cast<size_t>(ns) * C::STAGE + GQD * sizeof(SegQ) + (2 * ns + 2 * GQD) * sizeof(uint64_t) +
               sizeof(GMisc);
  off = (off + 127) & ~static_cast<size_t>(127);
  return off + TC_WG * TC_WGSMEM + 3 * TC_WG * sizeof(uint64_t) + 64;
}

__device__ __forceinline__ void wg_sync(int h) { asm volatile("bar.sync %0, 128;" ::"r"(1 + h) : "memory"); }
// Warpgroup barrier that also ANDs a predicate over its 128 threads: every exit decision after a bounded
// wait is taken here, the same for the whole warpgroup, so no thread leaves while others wait at a barrier.
__device__ __forceinline__ bool wg_and(int h, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbarrier.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(1 + h)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 6, 512;" ::: "memory"); }
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t f2u_sat(float x) {
  uint32_t r;
  asm("cvt.rni.sat.u32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float fold_planes(const uint32_t* o) {   // 4 byte planes (lowest first) of one head
  return fmaf(static_cast<float>(static_cast<int>(o[3])), 16777216.f,
              fmaf(static_cast<float>(static_cast<int>(o[2])), 65536.f,
                   fmaf(static_cast<float>(static_cast<int>(o[1])), 256.f, static_cast<float>(static_cast<int>(o[0])))));
}
// Row of the weight buffer (= A column order) of token r of a tile: the V codes of a tile come out of
// the stored words in the token order 0, 8, 1, 9, 2, 10, ... (word t gives tokens 2t, 8+2t, 2t+1, 9+2t).
__device__ __forceinline__ int tc_row_of(int r) { return 4 * ((r & 7) >> 1) + 2 * (r & 1) + (r >> 3); }

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1) tattn_kernel(AttnParams p, GPlanRec* plan) {
  static_assert(D == 128, "the tensor-memory kernel covers D = 128");
  using C = GCfg<D, 4>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int NS = p.ns;
  uint8_t* ring = smem;
  SegQ* segq = reinterpret_cast<SegQ*>(ring + static_cast<size_t>(NS) * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(segq + GQD);
  GMisc* misc = reinterpret_cast<GMisc*>(bars + 2 * NS + 2 * GQD);
  size_t off = static_cast<size_t>(reinterpret_cast<uint8_t*>(misc + 1) - smem);
  off = (off + 127) & ~static_cast<size_t>(127);
  uint8_t* wgbase = smem + off;
  uint64_t* tbars = reinterpret_cast<uint64_t*>(wgbase + TC_WG * TC_WGSMEM);   // per warpgroup: scores, P.V x2
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tbars + 3 * TC_WG);
  int* flags = reinterpret_cast<int*>(tmem_slot + 2);                          // per warpgroup: 2 words
  volatile int* abort_flag = &misc->abort;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * NS;
  const uint32_t iqf0 = full0 + 16 * NS, iqe0 = iqf0 + 8 * GQD;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* status = &p.state->status;
  const int c = blockIdx.x;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (p.wait_first) asm volatile("griddepcontrol.wait;" ::: "memory");   // after the fused step kernel
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, TC_WG); }
    for (int s = 0; s < GQD; ++s) { mbar_init(iqf0 + 8 * s, 1); mbar_init(iqe0 + 8 * s, TC_WG); }
    for (int i = 0; i < 3 * TC_WG; ++i) mbar_init(smem_u32(tbars + i), 1);
    for (int i = 0; i < 2 * TC_WG; ++i) flags[i] = 0;
    misc->abort = 0;
    misc->n_empty = 0;
    for (int s = 0; s < MAX_NS; ++s) misc->last_fill[s] = -1;
    fence_barrier_init();
  }

  long long T = 0, N = 0;
  int j0 = 0, j1 = 0;
  if (!plan_share<4>(p, plan, misc, c, tid, TC_THREADS, T, N, j0, j1)) return;

  if (warp == 4 * TC_WG) {
    produce<D, 4>(p, misc, segq, ring, NS, full0, empty0, iqf0, iqe0, c, j0, j1, T, N, lane, abort_flag, status);
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int h = warp >> 2, wt = tid & 127;
  if (warp == 0) {
    tc::alloc(smem_u32(tmem_slot), TC_COLS);
    tc::relinquish();
  }
  tc::fence_before();
  consumers_sync();
  tc::fence_after();
  const uint32_t tcol = *tmem_slot + 128u * static_cast<uint32_t>(h);                 // lane 0 (multiplies)
  const uint32_t tlane = tcol + (static_cast<uint32_t>(32 * (warp & 3)) << 16);     // this warp's lanes
  uint8_t* wgs = wgbase + h * TC_WGSMEM;
  const uint32_t qB = smem_u32(wgs), PB = qB + TC_QB;
  float* scratch = reinterpret_cast<float*>(wgs + TC_QB + 2 * TC_PB);
  const uint32_t sbar = smem_u32(tbars + 3 * h), pvbar0 = sbar + 8;
  int* myflags = flags + 2 * h;
  constexpr int HS = head_stride(D);
  const int pstride = partial_stride(p.G, D);
  const float NEGINF = -INFINITY;

  uint32_t s = 0, par = 0;   // ring position of the next stage and its fill parity
  uint32_t nb = 0;           // blocks issued by this warpgroup (phases of its tensor-core barriers)
  uint32_t n_qk = 0, n_pv = 0;   // tensor-core commits issued on the score and P.V barriers
  bool ok = true;
  for (int q = 0; ok; ++q) {
    const int slot = q % GQD;
    ok = mbar_wait(iqf0 + 8 * slot, (q / GQD) & 1, abort_flag, status);
    const SegQ sq = segq[slot];
    ok = wg_and(h, ok);
    if (!ok) break;
    if (wt == 0) mbar_arrive(iqe0 + 8 * slot);
    if (sq.n < 0) break;
    const Group g = sq.g;
    if (q == 0) asm volatile("griddepcontrol.wait;" ::: "memory");   // the query operands are written
    const int hkv = g.hg * 4 + h;
    const uint8_t* blob = p.qblob + static_cast<size_t>(g.b * p.Hkv + hkv) * qblob_bytes(D);
    {
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(blob) + wt);   // 128 threads x 16 B = both planes
      sts128(qB + 16 * wt, v.x, v.y, v.z, v.w);
    }
    const float* tail = reinterpret_cast<const float*>(blob + 16 * D);
    float qs[4];
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) qs[hh] = __ldcg(tail + hh);
    const float kscale = __ldcg(tail + MAX_G);
    fence_proxy_async_smem();   // the planes are read by the tensor cores

    float m[4], l[4], zs[4], oacc[4];
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) { m[hh] = NEGINF; l[hh] = 0.f; zs[hh] = 0.f; oacc[hh] = 0.f; }
    float sref = 0.f, F = 0.f;
    bool ostarted = false;
    int since_fold = 0;

    int u = sq.u0;
    const int u_end = sq.u0 + sq.n;
    while (u < u_end) {
      // ---- the next block: up to 8 tiles of this head, and the stages they span
      uint32_t ts[TC_BLOCK];
      int tp[TC_BLOCK];
      uint32_t tk = 0;   // bit i: tile i is INT8
      int nt = 0, nst = 0;
      const uint32_t s_first = s;
      while (u < u_end && nt < TC_BLOCK) {
        const bool int8 = u >= g.n4;
        const int v = u - g.n4;
        if (!int8 || (v & 1) == (h >> 1)) {
          ts[nt] = s;
          tp[nt] = int8 ? (v >> 1) * TILE : (g.t0 + u) * TILE;
          if (int8) tk |= 1u << nt;
          ++nt;
        }
        if (ok && !mbar_wait(full0 + 8 * s, par, abort_flag, status)) ok = false;
        if (++s == static_cast<uint32_t>(NS)) { s = 0; par ^= 1u; }
        ++nst;
        ++u;
      }
      if (nt == 0) {   // only the other half of a protected tile: hand the stages back
        ok = wg_and(h, ok);
        if (!ok) break;
        if (wt == 0)
          for (int k = 0, ss = static_cast<int>(s_first); k < nst; ++k, ss = (ss + 1 == NS) ? 0 : ss + 1)
            mbar_arrive(empty0 + 8 * ss);
        continue;
      }
      const uint32_t buf = nb & 1u;

      // ---- K phase: thread wt = token wt of the block
      const int it = wt >> 4, r = wt & 15;
      float sK = 0.f, zK = 0.f, sV = 0.f, zV = 0.f;
      bool valid = false;
      {
        uint32_t kw[32];
        if (it < nt) {
          const bool i8 = (tk >> it) & 1u;
          const uint32_t ta = smem_u32(ring + static_cast<size_t>(ts[it]) * C::STAGE) +
                              (i8 ? (h & 1) * tile8_bytes(D) : h * tile4_bytes(D));
          if (!i8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 w = lds128(ta + r * (D / 2) + 16 * i);
              kw[8 * i + 0] = w.x & 0x0F0F0F0Fu; kw[8 * i + 1] = (w.x >> 4) & 0x0F0F0F0Fu;
              kw[8 * i + 2] = w.y & 0x0F0F0F0Fu; kw[8 * i + 3] = (w.y >> 4) & 0x0F0F0F0Fu;
              kw[8 * i + 4] = w.z & 0x0F0F0F0Fu; kw[8 * i + 5] = (w.z >> 4) & 0x0F0F0F0Fu;
              kw[8 * i + 6] = w.w & 0x0F0F0F0Fu; kw[8 * i + 7] = (w.w >> 4) & 0x0F0F0F0Fu;
            }
            const uint32_t so = ta + 16 * D + 16 * (r & 7) + 4 * (r >> 3);
            const uint32_t szk = lds32(so), szv = lds32(so + 8);
            sK = half_lo(szk); zK = half_hi(szk); sV = half_lo(szv); zV = half_hi(szv);
            const int pos = tp[it] + r;
            valid = pos >= g.lo4 && pos < g.hi4;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint4 w = lds128(ta + r * D + 16 * i);
              kw[4 * i + 0] = w.x; kw[4 * i + 1] = w.y; kw[4 * i + 2] = w.z; kw[4 * i + 3] = w.w;
            }
            const uint32_t so = ta + 32 * D + 16 * (r & 7) + 4 * (r >> 3);
            const uint32_t szk = lds32(so), szv = lds32(so + 8);
            sK = half_lo(szk); zK = half_hi(szk); sV = half_lo(szv); zV = half_hi(szv);
            valid = tp[it] + r < g.nprot;
          }
          if (!valid) { sK = 0.f; zK = 0.f; sV = 0.f; zV = 0.f; }   // unwritten slots may hold non-finite scales
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) kw[i] = 0u;
        }
        tc::st32x32(tlane + TC_AK, kw);
      }
      tc::wait_st();
      tc::fence_before();
      ok = wg_and(h, ok);                           // the K codes of the block are in TMEM
      tc::fence_after();
      if (!ok) break;
      if (wt == 0) {
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          tc::mma_i8(tcol + TC_S, tcol + TC_AK + 8 * j, tc::sdesc(qB + 256 * j, 128, 256), TC_IDESC_QK_HI, j > 0);
          tc::mma_i8(tcol + TC_S + 8, tcol + TC_AK + 8 * j, tc::sdesc(qB + 1024 + 256 * j, 128, 256), TC_IDESC_QK_LO,
                     j > 0);
        }
        tc::commit(sbar);
      }
      // ---- V phase: thread wt = dim wt; the buffer's previous multiplies (block nb - 2) must be done
      if (ok && nb >= 2 && !mbar_wait(pvbar0 + 8 * buf, ((nb - 2) >> 1) & 1u, abort_flag, status)) ok = false;
      tc::fence_after();   // the tensor-memory stores below follow those multiplies
      {
        uint32_t vw[32];
        const int d = wt, mb = d >> 4, dh = (d >> 3) & 1, gg = d & 7;
#pragma unroll
        for (int i = 0; i < TC_BLOCK; ++i) {
          if (i < nt) {
            const bool i8 = (tk >> i) & 1u;
            const uint32_t ta = smem_u32(ring + static_cast<size_t>(ts[i]) * C::STAGE) +
                                (i8 ? (h & 1) * tile8_bytes(D) : h * tile4_bytes(D));
            if (!i8) {
              const uint32_t va = ta + 8 * D + 512 * (mb >> 2) + 64 * gg + 4 * (mb & 3);
#pragma unroll
              for (int t = 0; t < 4; ++t) vw[4 * i + t] = (lds32(va + 16 * t) >> (4 * dh)) & 0x0F0F0F0Fu;
            } else {
              // words of th = 0 and th = 1 of the pair (w = 2 mb, 2 mb + 1) sit 4 bytes apart
              const uint32_t va = ta + 16 * D + 16 * (32 * (mb >> 1) + 4 * gg) + 4 * (2 * (mb & 1));
              const uint32_t sel = dh ? 0x7351u : 0x6240u;
#pragma unroll
              for (int t = 0; t < 4; ++t) vw[4 * i + t] = __byte_perm(lds32(va + 16 * t), lds32(va + 16 * t + 4), sel);
            }
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) vw[4 * i + t] = 0u;
          }
        }
        tc::st32x32(tlane + TC_AV + 32 * buf, vw);
      }
      tc::wait_st();   // the V codes are in TMEM (read by the P.V multiplies after the next barrier)
      ++n_qk;
      ok = ok && mbar_wait(sbar, nb & 1u, abort_flag, status);
      tc::fence_after();
      uint32_t sr[16];
      if (ok) {
        tc::ld32x16(tlane + TC_S, sr);
        tc::wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) sr[i] = 0u;
      }

      // ---- softmax of token wt (4 query heads), weights with the current max and scale
      const float sKs = sK * kscale;
      float x[4], pr[4];
      bool need = since_fold >= TC_FLUSH_BLOCKS;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        x[hh] = valid ? fmaf(static_cast<float>(static_cast<int>(sr[hh]) * 256 + static_cast<int>(sr[8 + hh])), sKs,
                             zK * qs[hh])
                      : NEGINF;
        need |= x[hh] > m[hh] + TC_TAU;
      }
      need |= valid && sV > sref;
      if (__any_sync(0xffffffffu, need) && lane == 0) atomicOr(myflags + (nb & 1u), 1);
      if (wt == 0) myflags[(nb + 1) & 1u] = 0;   // the next block's flag (last read before this block began)
      const int row = 16 * it + tc_row_of(r);
      const uint32_t prow = PB + TC_PB * buf + 16 * row;
      {
        const float sVF = sV * F;
        uint32_t W[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          pr[hh] = valid ? ex2(x[hh] - m[hh]) : 0.f;
          W[hh] = valid ? f2u_sat(pr[hh] * sVF) : 0u;
        }
        sts128(prow, W[0], W[1], W[2], W[3]);
      }
      fence_proxy_async_smem();
      tc::fence_before();
      ok = wg_and(h, ok);                           // weights stored, V codes in TMEM, the stages read
      tc::fence_after();
      if (!ok) break;
      if (wt == 0)
        for (int k = 0, ss = static_cast<int>(s_first); k < nst; ++k, ss = (ss + 1 == NS) ? 0 : ss + 1)
          mbar_arrive(empty0 + 8 * ss);
      if (*reinterpret_cast<volatile int*>(myflags + (nb & 1u))) {
        // ---- rare path (the whole warpgroup): block maxima, new max and fixed-point scale, fold the
        // accumulator into the fp32 sums in the old scale, then redo this block's weights
        float bm[5] = {x[0], x[1], x[2], x[3], valid ? sV : 0.f};
#pragma unroll
        for (int i = 0; i < 5; ++i)
#pragma unroll
          for (int o = 16; o; o >>= 1) bm[i] = fmaxf(bm[i], __shfl_xor_sync(0xffffffffu, bm[i], o));
        if (lane == 0)
#pragma unroll
          for (int i = 0; i < 5; ++i) scratch[8 * (warp & 3) + i] = bm[i];
        wg_sync(h);
#pragma unroll
        for (int i = 0; i < 5; ++i)
          bm[i] = fmaxf(fmaxf(scratch[i], scratch[8 + i]), fmaxf(scratch[16 + i], scratch[24 + i]));
        wg_sync(h);
        float alpha[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float mn = fmaxf(m[hh], bm[hh]);
          alpha[hh] = (m[hh] == NEGINF) ? 0.f : ex2(m[hh] - mn);
          m[hh] = mn;
        }
        if (ostarted) {
          const uint32_t pb = (nb - 1) & 1u;
          ok = wg_and(h, mbar_wait(pvbar0 + 8 * pb, ((nb - 1) >> 1) & 1u, abort_flag, status));
          if (!ok) break;
          tc::fence_after();
          uint32_t o16[16];
          tc::ld32x16(tlane + TC_O, o16);
          tc::wait_ld();
          const float invF = F > 0.f ? 1.f / F : 0.f;
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) oacc[hh] = fmaf(fold_planes(o16 + 4 * hh), invF, oacc[hh]);
          ostarted = false;
        }
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) { oacc[hh] *= alpha[hh]; l[hh] *= alpha[hh]; zs[hh] *= alpha[hh]; }
        if (2.f * bm[4] > sref) {
          sref = 2.f * bm[4];
          F = 1073741824.f / sref;   // 2^(32 - TAU) / s_ref
        }
        since_fold = 0;
        const float sVF = sV * F;
        uint32_t W[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          pr[hh] = (valid && m[hh] != NEGINF) ? ex2(x[hh] - m[hh]) : 0.f;
          W[hh] = valid ? f2u_sat(pr[hh] * sVF) : 0u;
        }
        sts128(prow, W[0], W[1], W[2], W[3]);
        fence_proxy_async_smem();
        tc::fence_before();
        wg_sync(h);
        tc::fence_after();
      }
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) { l[hh] += pr[hh]; zs[hh] = fmaf(pr[hh], zV, zs[hh]); }
      // ---- P.V: 4 multiplies of 32 tokens into the int32 accumulator
      if (wt == 0) {
#pragma unroll
        for (int j = 0; j < TC_BLOCK / 2; ++j)
          tc::mma_i8(tcol + TC_O, tcol + TC_AV + 32 * buf + 8 * j, tc::sdesc(PB + TC_PB * buf + 512 * j, 128, 512),
                     TC_IDESC_PV, (ostarted || j > 0) ? 1u : 0u);
        tc::commit(pvbar0 + 8 * buf);
      }
      ++n_pv;
      ostarted = true;
      ++since_fold;
      ++nb;
    }
    if (!ok) break;

    // ---- the segment's result: fold the accumulator, sum l and z over the warpgroup's tokens
    if (ostarted) {
      const uint32_t pb = (nb - 1) & 1u;
      ok = wg_and(h, mbar_wait(pvbar0 + 8 * pb, ((nb - 1) >> 1) & 1u, abort_flag, status));
      if (!ok) break;
      tc::fence_after();
      uint32_t o16[16];
      tc::ld32x16(tlane + TC_O, o16);
      tc::wait_ld();
      const float invF = F > 0.f ? 1.f / F : 0.f;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) oacc[hh] = fmaf(fold_planes(o16 + 4 * hh), invF, oacc[hh]);
    }
    float red[8] = {l[0], l[1], l[2], l[3], zs[0], zs[1], zs[2], zs[3]};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int o = 16; o; o >>= 1) red[i] += __shfl_xor_sync(0xffffffffu, red[i], o);
    if (lane == 0)
#pragma unroll
      for (int i = 0; i < 8; ++i) scratch[8 * (warp & 3) + i] = red[i];
    wg_sync(h);
#pragma unroll
    for (int i = 0; i < 8; ++i) red[i] = (scratch[i] + scratch[8 + i]) + (scratch[16 + i] + scratch[24 + i]);
    wg_sync(h);
    float o[4];
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) o[hh] = oacc[hh] + red[4 + hh];   // unnormalised o_rot of dim wt
    if (sq.nseg == 1) {
      const int d = wt;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) o[hh] *= red[hh] > 0.f ? 1.f / red[hh] : 0.f;
      // o = H_blk o_rot: ascending butterfly stages over the dims (one dim per thread)
      const int Bh = p.Bh_o;
#pragma unroll
      for (int st = 1; st < 32; st <<= 1)
        if (st < Bh)
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            const float other = __shfl_xor_sync(0xffffffffu, o[hh], st);
            o[hh] = (d & st) ? other - o[hh] : o[hh] + other;
          }
      for (int st = 32; st < D && st < Bh; st <<= 1) {
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) scratch[4 * d + hh] = o[hh];
        wg_sync(h);
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float other = scratch[4 * (d ^ st) + hh];
          o[hh] = (d & st) ? other - o[hh] : o[hh] + other;
        }
        wg_sync(h);
      }
      const float rc = p.rc_o;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const long long off = (static_cast<long long>(g.b) * p.Hq + hkv * 4 + hh) * D + d;
        if (p.mode & KV4_MODE_OUT_F32) static_cast<float*>(p.out)[off] = o[hh] * rc;
        else static_cast<uint16_t*>(p.out)[off] = __bfloat16_as_ushort(__float2bfloat16_rn(o[hh] * rc));
      }
    } else {
      // a group split over several CTAs: this segment's partial (m, l, unnormalised o) for the merge kernel
      float* part = p.partials + static_cast<size_t>((c * 2 + (q == 0 ? 0 : 1)) * 4 + h) * pstride;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) part[hh * HS + wt] = o[hh];
      if (wt == 0)
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) { part[hh * HS + D] = m[hh]; part[hh * HS + D + 1] = red[hh]; }
    }
  }
  // no multiply may be in flight when the tensor memory is freed: after an abort, wait (bounded) for the
  // last commits this warpgroup issued (the P.V ones of block n_pv - 1, the score ones of block n_qk - 1)
  if (!ok) {
    if (n_pv > 0) {
      const uint32_t b = n_pv - 1;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(pvbar0 + 8 * (b & 1u), (b >> 1) & 1u) && globaltimer_ns() - t0 < 1000000000ull) {}
    }
    if (n_qk > 0) {
      const uint64_t t1 = globaltimer_ns();
      while (!mbar_try_wait(sbar, (n_qk - 1) & 1u) && globaltimer_ns() - t1 < 1000000000ull) {}
    }
  }
  tc::fence_before();
  consumers_sync();
  tc::fence_after();
  if (warp == 0) tc::dealloc(*tmem_slot, TC_COLS);
}

// ---------------------------------------------------------------------------
// host side

#ifndef KV4_GROUPED_PAIR
#define KV4_GROUPED_PAIR 2
#endif
constexpr int kPair = KV4_GROUPED_PAIR;   // INT4 tiles per consumer iteration of the compiled variant
static_assert(kPair == 1 || kPair == 2 || kPair == 4, "tiles per iteration");
#ifndef KV4_PC_PAIR
#define KV4_PC_PAIR 4
#endif
// INT4 tiles per iteration of the paired-column variant: it has the registers for four (117 at D = 128),
// which measured 2-3 % faster than two on batches of 256 and 512 sequences
constexpr int kPairPC = KV4_PC_PAIR;
static_assert(kPairPC == 1 || kPairPC == 2 || kPairPC == 4, "tiles per iteration");

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Grid of the kernel variant in use (CTAs per SM x SMs).
inline int g_grid(const kv4_cache* c) { return c->num_sms * CTAS_PER_SM; }

// Workspace: the query operands of every (batch entry, KV head), then two
// partial slots per CTA and KV head of a group (the CTA's first and last
// segment; segments in between cover whole groups and need none).
struct GLayout {
  size_t qblob, partials, plan, total;
};

GLayout g_layout(const kv4_cache* c, int n_seqs, int qlen) {
  const kv4_config& cfg = c->cfg;
  const int G = qlen * (cfg.num_q_heads / cfg.num_kv_heads);   // operand columns per KV head
  const int gw = group_width(cfg.num_kv_heads);
  GLayout l{};
  l.qblob = 0;
  l.partials = al256(static_cast<size_t>(n_seqs) * cfg.num_kv_heads * qblob_bytes(cfg.head_dim));
  l.plan = l.partials + al256(static_cast<size_t>(g_grid(c)) * 2 * gw * partial_stride(G, cfg.head_dim) * sizeof(float));
  const size_t n_groups = static_cast<size_t>(n_seqs) * (cfg.num_kv_heads / gw);
  l.total = l.plan + al256(n_groups * sizeof(GPlanRec) + sizeof(GPlanHdr));
  return l;
}

// Deepest ring (at most MAX_NS stages) that keeps CTAS_PER_SM CTAs of both
// variants (one and several query tokens) of page format F resident per SM.
template <int D, int PAIR, int PAIRPC, int GWR, int F>
int g_choose_ring(int device) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess) return -1;
  // the paired-column variant exists for the integer page formats (the NVFP4 one instantiates the plain one twice)
  constexpr bool PCV = F != 1;
  if (cudaFuncSetAttribute(gattn_kernel<D, PAIR, false, GWR, F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess ||
      cudaFuncSetAttribute(gattn_kernel<D, PAIR, true, GWR, F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess ||
      cudaFuncSetAttribute(gattn_kernel<D, PAIRPC, false, GWR, F, PCV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin) != cudaSuccess)
    return -1;
  const int want = CTAS_PER_SM;
  // a consumer warp holds up to PAIR stages of a unit at once: keep as many more in flight
  constexpr int NS_MIN = 2 * (PAIR > PAIRPC ? PAIR : PAIRPC);
  for (int ns = MAX_NS; ns >= NS_MIN; --ns) {
    const size_t smem = gattn_smem_bytes<D, GWR, F>(ns);
    if (smem > static_cast<size_t>(optin)) continue;
    int blocks = 0;
    int blocks_multi = 0;
    int blocks_pc = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, gattn_kernel<D, PAIR, false, GWR, F>,
                                                      GShape<GWR>::THREADS, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_multi, gattn_kernel<D, PAIR, true, GWR, F>,
                                                      GShape<GWR>::THREADS, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_pc, gattn_kernel<D, PAIRPC, false, GWR, F, PCV>,
                                                      GShape<GWR>::THREADS, smem) != cudaSuccess)
      return -1;
    if (blocks >= want && blocks_multi >= want && blocks_pc >= want) return ns;
  }
  return -1;
}

template <int D, int GWR>
int g_launch(kv4_cache* c, AttnParams p, void* ws, cudaStream_t stream, const AppendParams* step) {
  const GLayout l = g_layout(c, p.n_seqs, p.qlen);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.qblob = wsb + l.qblob;
  p.partials = reinterpret_cast<float*>(wsb + l.partials);
  GPlanRec* plan = reinterpret_cast<GPlanRec*>(wsb + l.plan);
  // one query token, 4-head groups, D = 128, INT4 pages: the tensor-memory kernel when selected, one CTA per SM
  const bool fp4 = c->cfg.page_format == KV4_FORMAT_NVFP4, int2 = c->cfg.page_format == KV4_FORMAT_INT2;
  const bool tcpath = D == 128 && GWR == 4 && c->use_tc && p.qtot == 1 && c->cfg.page_format == KV4_FORMAT_INT4;
  // one query token and at most 4 query heads per KV head on integer pages: paired columns
  const bool pcol = !tcpath && !fp4 && p.qtot == 1 && p.G <= 4;
  p.qfmt = tcpath ? 1 : (fp4 ? 2 : (pcol ? 3 : 0));
  p.grid = tcpath ? c->num_sms : g_grid(c);
  p.cap_parts = p.grid * 2 * GWR;
  p.ns = tcpath ? c->tattn_ring : c->gattn_ring;
  p.stall_stage = c->test_stall;   // test hook, for this launch only
  c->test_stall = -1;
  if (step) {
    // fused decode step: the append and the query operands first; the attention
    // kernel then starts in plain stream order (it plans from the new lengths)
    if (p.Hkv <= 8) gstep_kernel<D, 16><<<p.n_seqs, 64 * p.Hkv, 0, stream>>>(p, *step);
    else gstep_kernel<D, 32><<<p.n_seqs, 64 * p.Hkv, 0, stream>>>(p, *step);
    if (c->ev_before) cudaEventRecord(c->ev_before, stream);
  } else {
    if (c->ev_before) cudaEventRecord(c->ev_before, stream);
    const int pairs = p.n_seqs * p.Hkv;
    gq_kernel<D><<<(pairs + QWARPS - 1) / QWARPS, 32 * QWARPS, 0, stream>>>(p);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(tcpath ? TC_THREADS : GShape<GWR>::THREADS);
  cfg.dynamicSmemBytes = tcpath ? tattn_smem_bytes<D>(p.ns)
                                : (fp4 ? gattn_smem_bytes<D, GWR, 1>(p.ns)
                                       : (int2 ? gattn_smem_bytes<D, GWR, 2>(p.ns) : gattn_smem_bytes<D, GWR>(p.ns)));
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // programmatic dependent of the query kernel (it waits only before its first query read) or of the
  // fused step kernel (it waits before its first instruction); an event marker between the two launches
  // leaves them in plain stream order
  cfg.numAttrs = (step && c->ev_before) ? 0 : 1;
  p.wait_first = step ? 1 : 0;
  // several query tokens per sequence (even a pass of one of them): the causal variant
  cudaError_t e;
  if (fp4) {
    e = p.qtot > 1 ? cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, true, GWR, 1>, p, plan)
                   : cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, false, GWR, 1>, p, plan);
  } else if (int2) {
    e = p.qtot > 1 ? cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, true, GWR, 2>, p, plan)
        : pcol     ? cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPairPC, false, GWR, 2, true>, p, plan)
                   : cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, false, GWR, 2>, p, plan);
  } else if (tcpath) {
    if constexpr (D == 128 && GWR == 4) e = cudaLaunchKernelEx(&cfg, tattn_kernel<D>, p, plan);
    else e = cudaErrorInvalidValue;
  } else {
    e = p.qtot > 1 ? cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, true, GWR>, p, plan)
        : pcol     ? cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPairPC, false, GWR, 0, true>, p, plan)
                   : cudaLaunchKernelEx(&cfg, gattn_kernel<D, kPair, false, GWR>, p, plan);
  }
  if (e == cudaSuccess) {
    cudaLaunchConfig_t mcfg = cfg;
    mcfg.gridDim = dim3((p.n_seqs * p.Hkv * p.G + MWARPS - 1) / MWARPS);
    mcfg.blockDim = dim3(32 * MWARPS);
    mcfg.dynamicSmemBytes = 0;
    mcfg.numAttrs = 1;   // programmatic dependent of the attention kernel
    e = cudaLaunchKernelEx(&mcfg, gmerge_kernel<D, GWR>, p, static_cast<const GPlanRec*>(plan));
  }
  if (c->ev_after) cudaEventRecord(c->ev_after, stream);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

template <int D>
int g_launch_gw(kv4_cache* c, const AttnParams& p, void* ws, cudaStream_t stream, const AppendParams* step = nullptr) {
  switch (group_width(p.Hkv)) {
    case 4: return g_launch<D, 4>(c, p, ws, stream, step);
    case 2: return g_launch<D, 2>(c, p, ws, stream, step);
    default: return g_launch<D, 1>(c, p, ws, stream, step);
  }
}

template <int D, int F>
int g_choose_ring_gw(int device, int Hkv) {
  switch (group_width(Hkv)) {
    case 4: return g_choose_ring<D, kPair, kPairPC, 4, F>(device);
    case 2: return g_choose_ring<D, kPair, kPairPC, 2, F>(device);
    default: return g_choose_ring<D, kPair, kPairPC, 1, F>(device);
  }
}

// Ring depth of the tensor-memory kernel (one CTA per SM), or -1 when it cannot run.
int tattn_choose_ring(int device) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess) return -1;
  if (cudaFuncSetAttribute(tattn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess)
    return -1;
  for (int ns = MAX_NS; ns >= 2 * TC_BLOCK; --ns) {
    const size_t smem = tattn_smem_bytes<128>(ns);
    if (smem > static_cast<size_t>(optin)) continue;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, tattn_kernel<128>, TC_THREADS, smem) != cudaSuccess)
      return -1;
    if (blocks >= 1) return ns;
  }
  return -1;
}

}  // namespace

bool grouped_path(const kv4_cache* c) { return !c->bf16; }

int grouped_ring(kv4_cache* c) {
  c->gattn_pair = kPair;
  c->use_tc = false;
  c->tattn_ring = 0;
  if (c->cfg.head_dim == 128 && group_width(c->cfg.num_kv_heads) == 4 && c->cfg.page_format == KV4_FORMAT_INT4) {
    // "tc": the tensor-memory kernel, an opt-in alternative (slower than the mma.sync kernel on B200)
    const char* env = getenv("KV4_ATTENTION_KERNEL");
    if (env && strcmp(env, "tc") == 0) {
      const int ns = tattn_choose_ring(c->device);
      if (ns > 0) {
        c->use_tc = true;
        c->tattn_ring = ns;
      } else {
        cudaGetLastError();
      }
    }
  }
  const int Hkv = c->cfg.num_kv_heads;
  if (c->cfg.page_format == KV4_FORMAT_NVFP4)
    return c->cfg.head_dim == 128 ? g_choose_ring_gw<128, 1>(c->device, Hkv) : g_choose_ring_gw<64, 1>(c->device, Hkv);
  if (c->cfg.page_format == KV4_FORMAT_INT2)
    return c->cfg.head_dim == 128 ? g_choose_ring_gw<128, 2>(c->device, Hkv) : g_choose_ring_gw<64, 2>(c->device, Hkv);
  return c->cfg.head_dim == 128 ? g_choose_ring_gw<128, 0>(c->device, Hkv) : g_choose_ring_gw<64, 0>(c->device, Hkv);
}

size_t grouped_workspace_bytes(const kv4_cache* c, int n_seqs, int qlen) { return g_layout(c, n_seqs, qlen).total; }

int launch_decode_step(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* k_new,
                       const void* v_new, const void* q, void* out, float softmax_scale, int mode, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  if (!grouped_path(c) || c->cfg.num_kv_heads > 16) return KV4_ERR_UNSUPPORTED;   // two warps per KV head
  if (c->gattn_ring <= 0 || c->gattn_ring > MAX_NS) return KV4_ERR_UNSUPPORTED;
  if (n_seqs > c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  if (ws_bytes < g_layout(c, n_seqs, 1).total) return KV4_ERR_WORKSPACE;
  AttnParams p{};
  fill_common(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, p);
  const AppendParams ap = append_params(c, layer, seq_ids, nullptr, n_seqs, n_seqs, k_new, v_new,
                                        (mode & KV4_MODE_ROPE_Q) != 0);
  return p.D == 128 ? g_launch_gw<128>(c, p, ws, stream, &ap) : g_launch_gw<64>(c, p, ws, stream, &ap);
}

int launch_grouped(kv4_cache* c, const AttnParams& p, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (p.qlen < 1 || p.G != p.qlen * p.Gh || p.G > MAX_G || p.q0 < 0 || p.q0 + p.qlen > p.qtot)
    return KV4_ERR_UNSUPPORTED;
  if (ws_bytes < g_layout(c, p.n_seqs, p.qlen).total) return KV4_ERR_WORKSPACE;
  if (c->gattn_ring <= 0 || c->gattn_ring > MAX_NS) return KV4_ERR_UNSUPPORTED;
  if (p.n_seqs > c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  return p.D == 128 ? g_launch_gw<128>(c, p, ws, stream) : g_launch_gw<64>(c, p, ws, stream);
}

}  // namespace kv4

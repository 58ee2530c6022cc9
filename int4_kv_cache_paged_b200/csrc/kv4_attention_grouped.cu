// Page-major, stream-K decode attention over the paged INT4/INT8 cache, used
// when the number of KV heads is a multiple of 8.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Abstract (fused attention over the paged, rotated token-wise INT4
// cache) and "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4
// KV Cache Quantization", Abstract (sinks and recent positions read from INT8).
//
// Work decomposition.  A head group is 8 consecutive KV heads of one sequence.
// Its work is a list of stages: one stage per 16-token INT4 tile position (the
// tiles of the 8 heads are contiguous in the head-innermost pool, one 17 KB
// bulk copy), then two stages per INT8 protected tile (heads 0-3, heads 4-7).
// The planner concatenates the stage lists of all head groups (T stages) and
// CTA c of the persistent grid (one per SM) takes stages [c*T/N, (c+1)*T/N):
// every CTA streams the same number of bytes (stream-K), no scheduling atomics.
// Where a CTA's range crosses head groups it works on segments; each segment
// ends in one partial (m, l, o) per KV head and query head, merged later.
//
// Inside a CTA: a producer warp issues the bulk copies into a ring of
// shared-memory stages (each lane one stage of a batch, mbarrier completion);
// consumer warp w handles KV head w of every stage, so every warp consumes
// every stage in order (which keeps the mbarrier parity waits exact) and no
// warp waits for another: each writes its own partial.
#include "kv4_attn_tiles.cuh"

namespace kv4 {

namespace {

using namespace tiles;

constexpr int GW = 8;                   // consumer warps = KV heads per group
constexpr int GTHREADS = 32 * (GW + 1);  // + producer warp
constexpr int GQD = 2;                  // segment queue depth

template <int D>
struct GCfg {
  static constexpr int STAGE4 = GW * tile4_bytes(D);        // one tile position, 8 heads
  static constexpr int STAGE8 = (GW / 2) * tile8_bytes(D);  // one protected tile, 4 heads
  static constexpr int STAGE = STAGE4 > STAGE8 ? STAGE4 : STAGE8;
  static constexpr int QBLOBS = GW * qblob_bytes(D);         // the group's 8 query blobs
};

// Per head group, written by the planner.
struct Group {
  int b, seq, hg;   // index into seq_ids, sequence id, head group (KV heads 8*hg .. 8*hg+7)
  int n4;           // INT4 stages (tiles t0 .. t0+n4-1)
  int t0, lo4, hi4; // first INT4 tile, valid INT4 positions [lo4, hi4)
  int n8;           // INT8 tiles (2 stages each), valid slots [0, nprot)
  int nprot;
  int start;        // first global stage index
  int segbase;      // first segment (partial slot / 8) of this group
  int c_first;      // first CTA whose range touches this group
};
static_assert(sizeof(Group) == 48, "group size");

struct SegQ {       // one queued segment
  Group g;
  int u0, n, k;     // local stages [u0, u0+n), segment index within the group
  int pad;
};

struct GHeader {
  int T;            // total stages
  int N;            // CTAs of the attention grid
  int n_groups;
  int pad[61];
};

__host__ __device__ inline int group_stages(const Group& g) { return g.n4 + 2 * g.n8; }

// CTA owning global stage j: the largest c with floor(c*T/N) <= j.
__device__ __forceinline__ int cta_of(long long j, long long T, long long N) {
  return static_cast<int>(((j + 1) * N - 1) / T);
}

template <int D>
__host__ __device__ inline size_t gattn_smem_bytes(int ns) {
  using C = GCfg<D>;
  return static_cast<size_t>(ns) * C::STAGE + static_cast<size_t>(GQD) * C::QBLOBS + GQD * sizeof(SegQ) +
         (2 * ns + 2 * GQD) * sizeof(uint64_t) + 16 + ns * sizeof(int);
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

// ---------------------------------------------------------------------------
// planner: blocks 0..nq-1 build the query blobs (one warp per (sequence, KV
// head)); the last block describes the head groups and the stream-K partition.

template <int D>
__global__ void __launch_bounds__(1024) gprep_kernel(AttnParams p, Group* groups, int* cta_first, GHeader* hdr,
                                                     int n_qblocks) {
  extern __shared__ float s_q[];   // [32][G][D] for the query blocks, scan scratch for the planner
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  if (static_cast<int>(blockIdx.x) < n_qblocks) {
    const int gw = blockIdx.x * (blockDim.x >> 5) + wib;
    if (gw >= p.n_seqs * p.Hkv) return;
    build_qblob<D, false>(p, gw / p.Hkv, gw % p.Hkv, lane, s_q + wib * p.G * D);
    return;
  }
  // ---- the planner block
  int* s_tmp = reinterpret_cast<int*>(s_q);
  const int HGN = p.Hkv / GW;
  const int n_groups = p.n_seqs * HGN;
  const int per = (n_groups + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per, i1 = min(i0 + per, n_groups);
  auto describe = [&](int i) -> Group {
    Group g{};
    g.b = i / HGN;
    g.hg = i % HGN;
    g.seq = p.seq_ids[g.b];
    int L = 0;
    if (g.seq >= 0 && g.seq < p.max_seqs) L = p.seq_lens[g.seq];
    else if (g.hg == 0) atomicOr(&p.state->status, KV4_DEV_BAD_SEQ);
    int lo4, hi4, nprot;
    if (p.mode & KV4_MODE_INT4_ONLY) { lo4 = 0; hi4 = L; nprot = 0; }
    else { nprot = min(L, p.S + p.W); lo4 = p.S; hi4 = L - p.W; }
    g.lo4 = lo4; g.hi4 = hi4; g.nprot = nprot;
    g.t0 = 0; g.n4 = 0;
    if (hi4 > lo4) { g.t0 = lo4 / TILE; g.n4 = (hi4 + TILE - 1) / TILE - g.t0; }
    g.n8 = (nprot + TILE - 1) / TILE;
    return g;
  };
  // pass 1: stage counts -> starts, total T
  int local = 0;
  for (int i = i0; i < i1; ++i) local += group_stages(describe(i));
  int T = 0;
  int start = block_exclusive_scan(local, s_tmp, &T);
  // partition over min(grid, T) CTAs: every active CTA owns at least one stage, so
  // the CTAs touching a group are exactly its consecutive segments
  const long long N = T < p.grid ? T : p.grid;
  // pass 2: segments per group -> segment bases
  int segs = 0;
  {
    int st = start;
    for (int i = i0; i < i1; ++i) {
      const int n = group_stages(describe(i));
      if (n > 0) segs += cta_of(st + n - 1, T, N) - cta_of(st, T, N) + 1;
      st += n;
    }
  }
  int n_segs = 0;
  int segbase = block_exclusive_scan(segs, s_tmp, &n_segs);
  // pass 3: write groups, the first group of every CTA, the per-(sequence, head) merge records
  {
    int st = start, sb = segbase;
    for (int i = i0; i < i1; ++i) {
      Group g = describe(i);
      const int n = group_stages(g);
      g.start = st;
      g.segbase = sb;
      g.c_first = n > 0 ? cta_of(st, T, N) : 0;
      const int nseg = n > 0 ? cta_of(st + n - 1, T, N) - g.c_first + 1 : 0;
      groups[i] = g;
      if (n > 0) {
        for (int c = g.c_first; c < g.c_first + nseg; ++c) {
          const long long b0 = static_cast<long long>(c) * T / N;   // first stage of CTA c
          if (b0 >= st && b0 < st + n) cta_first[c] = i;
        }
      }
      const int L = g.seq >= 0 && g.seq < p.max_seqs ? p.seq_lens[g.seq] : 0;
      for (int w = 0; w < GW; ++w) {
        SeqHead sh;
        sh.part_base = (sb * GW + w);
        sh.n_parts = nseg;
        sh.len = L;
        sh.pad = GW;   // stride between the segments' partials of one head
        p.seqhead[g.b * p.Hkv + g.hg * GW + w] = sh;
      }
      if ((sb + nseg) * GW > p.cap_parts) atomicOr(&p.state->status, KV4_DEV_WORKSPACE);
      st += n;
      sb += nseg;
    }
  }
  if (threadIdx.x == 0) {
    hdr->T = T;
    hdr->N = static_cast<int>(N);
    hdr->n_groups = n_groups;
  }
}

// ---------------------------------------------------------------------------
// the attention kernel

template <int D>
__device__ __forceinline__ const uint8_t* stage_source(const AttnParams& p, const Group& g, int u, uint32_t& bytes) {
  using C = GCfg<D>;
  if (u < g.n4) {
    const int pos = (g.t0 + u) * TILE;
    int page = p.block_table[static_cast<long long>(g.seq) * p.max_pages_per_seq + pos / p.P];
    if (page < 0 || page >= p.num_pages) {
      atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
      page = 0;
    }
    bytes = C::STAGE4;
    return p.pool + ((static_cast<long long>(page) * (p.P / TILE) + (pos % p.P) / TILE) * p.Hkv + g.hg * GW) *
                        tile4_bytes(D);
  }
  const int v = u - g.n4;
  bytes = C::STAGE8;
  return p.prot + ((static_cast<long long>(g.seq) * n_prot_tiles(p.S, p.W) + (v >> 1)) * p.Hkv + g.hg * GW +
                   (v & 1) * (GW / 2)) *
                      tile8_bytes(D);
}

// PAIR = INT4 tiles per iteration of a consumer warp: 2 (more independent work
// per warp, 1 CTA per SM) or 1 (fewer registers, 2 CTAs per SM).
template <int D, int PAIR>
__global__ void __launch_bounds__(GTHREADS, 3 - PAIR) gattn_kernel(AttnParams p, const Group* groups,
                                                                   const int* cta_first, const GHeader* hdr) {
  using C = GCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int NS = p.ns;
  uint8_t* ring = smem;
  uint8_t* qbuf = ring + static_cast<size_t>(NS) * C::STAGE;
  SegQ* segq = reinterpret_cast<SegQ*>(qbuf + GQD * C::QBLOBS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(segq + GQD);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NS + 2 * GQD);
  int* last_fill = const_cast<int*>(abort_flag) + 4;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * NS;
  const uint32_t iqf0 = full0 + 16 * NS, iqe0 = iqf0 + 8 * GQD;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* status = &p.state->status;

  const long long T = hdr->T, N = hdr->N;   // N = min(grid, T) active CTAs
  const long long c = blockIdx.x;
  if (c >= N) return;   // uniform over the CTA
  const int j0 = static_cast<int>(c * T / N), j1 = static_cast<int>((c + 1) * T / N);
  if (j0 >= j1) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, GW); }
    for (int s = 0; s < GQD; ++s) { mbar_init(iqf0 + 8 * s, 1); mbar_init(iqe0 + 8 * s, GW); }
    *abort_flag = 0;
    for (int s = 0; s < NS; ++s) last_fill[s] = -1;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == GW) {
    // ------------------------------------------------------------ producer
    const int nbatch = NS < 32 ? NS : 32;
    int gi = cta_first[c];
    Group g = groups[gi];
    int u = j0 - g.start;
    int j = j0;
    uint32_t jj = 0;   // CTA-local stage counter
    int q = 0;
    bool ok = true;
    while (j < j1 && ok) {
      const int n = min(g.start + group_stages(g) - j, j1 - j);
      const int slot = q % GQD;
      if (lane == 0) ok = mbar_wait(iqe0 + 8 * slot, ((q / GQD) & 1) ^ 1, abort_flag, status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        SegQ sq;
        sq.g = g; sq.u0 = u; sq.n = n; sq.k = static_cast<int>(c) - g.c_first; sq.pad = 0;
        segq[slot] = sq;
        mbar_arrive_expect_tx(iqf0 + 8 * slot, C::QBLOBS);
        bulk_g2s(smem_u32(qbuf + slot * C::QBLOBS),
                 p.qblob + static_cast<size_t>(g.b * p.Hkv + g.hg * GW) * qblob_bytes(D), C::QBLOBS, iqf0 + 8 * slot);
      }
      // the next group with stages (its descriptor load overlaps the copies below)
      int gn = gi + 1;
      Group nxt{};
      if (j + n < j1) nxt = groups[gn];
      // stages u .. u+n-1: one lane per stage, batches of at most NS stages
      for (int base = 0; base < n; base += nbatch) {
        bool lane_ok = true;
        if (lane < nbatch && base + lane < n) {
          uint32_t bytes;
          const uint8_t* src = stage_source<D>(p, g, u + base + lane, bytes);
          const uint32_t jl = jj + base + lane;
          const int s = jl % NS;
          lane_ok = mbar_wait(empty0 + 8 * s, ((jl / NS) & 1) ^ 1, abort_flag, status);
          if (lane_ok) {
            mbar_arrive_expect_tx(full0 + 8 * s, bytes);
            bulk_g2s(smem_u32(ring + static_cast<size_t>(s) * C::STAGE), src, bytes, full0 + 8 * s);
            last_fill[s] = static_cast<int>(jl);
          } else {
            *abort_flag = 1;
          }
        }
        ok = __all_sync(0xffffffffu, lane_ok);
        if (!ok) break;
      }
      jj += n;
      j += n;
      ++q;
      if (j < j1) {
        while (group_stages(nxt) == 0) nxt = groups[++gn];   // skip empty sequences
        gi = gn;
        g = nxt;
        u = 0;
      }
    }
    if (ok) {
      const int slot = q % GQD;
      if (lane == 0) ok = mbar_wait(iqe0 + 8 * slot, ((q / GQD) & 1) ^ 1, abort_flag, status);
      if (lane == 0 && ok) { segq[slot].n = -1; mbar_arrive(iqf0 + 8 * slot); }
    }
    if (!ok && lane == 0) {
      for (int st = 0; st < NS; ++st)
        if (last_fill[st] >= 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full0 + 8 * st, (last_fill[st] / NS) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
        }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int w = warp;   // KV head within the group
  const int g8 = lane >> 2, t = lane & 3;
  const int G = p.G;
  constexpr int HS = head_stride(D);
  ColSplit cs;
  cs.colsplit = (G == 1 || G == 2 || G == 4);
  cs.part0 = cs.colsplit ? (2 * t) / G : 0;
  cs.part1 = cs.colsplit ? (2 * t + 1) / G : 0;
  int s = 0;          // stage of the next CTA-local stage index
  uint32_t par = 0;   // its fill parity
  auto advance = [&]() {
    if (++s == NS) { s = 0; par ^= 1u; }
  };
  for (int q = 0;; ++q) {
    const int slot = q % GQD;
    if (!mbar_wait(iqf0 + 8 * slot, (q / GQD) & 1, abort_flag, status)) break;
    const SegQ sq = segq[slot];
    if (sq.n < 0) break;
    QFrag<D> qf;
    {
      const uint32_t qb = smem_u32(qbuf + slot * C::QBLOBS + w * qblob_bytes(D));
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        const uint4 v = lds128(qb + 16 * (32 * cc + lane));
        qf.b[2 * cc][0] = v.x; qf.b[2 * cc][1] = v.y; qf.b[2 * cc + 1][0] = v.z; qf.b[2 * cc + 1][1] = v.w;
      }
      const float* tail = reinterpret_cast<const float*>(qbuf + slot * C::QBLOBS + w * qblob_bytes(D) + 16 * D);
      qf.qs0 = tail[(2 * t) & 7];
      qf.qs1 = tail[(2 * t + 1) & 7];
      qf.kscale = tail[MAX_G];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(iqe0 + 8 * slot);

    WarpState<D> ws;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) ws.o[m][0] = ws.o[m][1] = ws.o[m][2] = ws.o[m][3] = 0.f;
    ws.m0 = ws.m1 = NEG_INF;
    ws.l0 = ws.l1 = ws.z0 = ws.z1 = 0.f;

    const Group& g = sq.g;
    const int u_end = sq.u0 + sq.n;
    bool ok = true;
    for (int u = sq.u0; u < u_end && ok;) {
      if (u < g.n4) {
        // one or two INT4 stages: the tiles of this warp's head
        const int nt = (PAIR == 2 && u + 1 < u_end && u + 1 < g.n4) ? 2 : 1;
        const int s0 = s;
        const uint32_t p0 = par;
        advance();
        const int s1 = nt == 2 ? s : s0;
        const uint32_t p1 = nt == 2 ? par : p0;
        if (nt == 2) advance();
        ok = mbar_wait(full0 + 8 * s0, p0, abort_flag, status);
        if (ok && nt == 2) ok = mbar_wait(full0 + 8 * s1, p1, abort_flag, status);
        if (!ok) break;
        const uint32_t tl[2] = {smem_u32(ring + static_cast<size_t>(s0) * C::STAGE + w * tile4_bytes(D)),
                                smem_u32(ring + static_cast<size_t>(s1) * C::STAGE + w * tile4_bytes(D))};
        const int pos0 = (g.t0 + u) * TILE;
        const bool inside = pos0 >= g.lo4 && pos0 + nt * TILE <= g.hi4;
        const uint32_t eb0 = empty0 + 8 * s0, eb1 = empty0 + 8 * s1;
        if (inside) {
          const int valid[2] = {3, 3};
          if (nt == 2) unit_int4<D, PAIR, false>(tl, qf, ws, lane, valid, eb0, eb1, cs);
          else unit_int4<D, 1, false>(tl, qf, ws, lane, valid, eb0, eb1, cs);
        } else {
          int valid[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int pg = pos0 + k * TILE + g8;
            valid[k] = (pg >= g.lo4 && pg < g.hi4 ? 1 : 0) | (pg + 8 >= g.lo4 && pg + 8 < g.hi4 ? 2 : 0);
          }
          if (nt == 2) unit_int4<D, PAIR, true>(tl, qf, ws, lane, valid, eb0, eb1, cs);
          else unit_int4<D, 1, true>(tl, qf, ws, lane, valid, eb0, eb1, cs);
        }
        u += nt;
      } else {
        // one INT8 stage: half (v & 1) of protected tile (v >> 1) holds heads 4*(v&1) .. +3
        const int v = u - g.n4;
        const int s0 = s;
        const uint32_t p0 = par;
        advance();
        ok = mbar_wait(full0 + 8 * s0, p0, abort_flag, status);
        if (!ok) break;
        const uint32_t eb = empty0 + 8 * s0;
        if ((v & 1) == (w >> 2)) {
          const uint32_t st = smem_u32(ring + static_cast<size_t>(s0) * C::STAGE + (w & 3) * tile8_bytes(D));
          const int slot0 = (v >> 1) * TILE;
          const bool vg = slot0 + g8 < g.nprot, vg8 = slot0 + g8 + 8 < g.nprot;
          if (slot0 + TILE <= g.nprot) tile_int8<D, false>(st, qf, ws, lane, true, true, eb, cs);
          else tile_int8<D, true>(st, qf, ws, lane, vg, vg8, eb, cs);
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(eb);
        }
        u += 1;
      }
    }
    if (!ok) break;

    // ---- this warp's partial for the segment
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
    const int slotp = (g.segbase + sq.k) * GW + w;
    if (slotp < p.cap_parts) {
      float* part = p.partials + static_cast<size_t>(slotp) * partial_stride(G, D);
      const int h0 = 2 * t, h1 = 2 * t + 1;
      if (h0 < G) {
        float* r = part + h0 * HS;
#pragma unroll
        for (int m = 0; m < D / 16; ++m) { r[16 * m + g8] = ws.o[m][0] + ws.z0; r[16 * m + g8 + 8] = ws.o[m][2] + ws.z0; }
        if (g8 == 0) { r[D] = ws.m0; r[D + 1] = ws.l0; }
      }
      if (h1 < G) {
        float* r = part + h1 * HS;
#pragma unroll
        for (int m = 0; m < D / 16; ++m) { r[16 * m + g8] = ws.o[m][1] + ws.z1; r[16 * m + g8 + 8] = ws.o[m][3] + ws.z1; }
        if (g8 == 0) { r[D] = ws.m1; r[D + 1] = ws.l1; }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host side

struct GLayout {
  size_t seqhead, qblob, hdr, groups, cta_first, partials, total;
  int cap_parts;
};

inline size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

GLayout g_layout(const kv4_cache* c, int n_seqs) {
  const kv4_config& cfg = c->cfg;
  const int G = cfg.num_q_heads / cfg.num_kv_heads, D = cfg.head_dim;
  const size_t nsh = static_cast<size_t>(n_seqs) * cfg.num_kv_heads;
  const size_t ngroups = static_cast<size_t>(n_seqs) * (cfg.num_kv_heads / GW);
  const size_t N = static_cast<size_t>(c->num_sms) * 2;   // upper bound of the grid over both variants
  GLayout l{};
  l.cap_parts = static_cast<int>((N + ngroups) * GW);
  size_t off = 0;
  l.seqhead = off; off = al256(off + nsh * sizeof(SeqHead));
  l.qblob = off; off = al256(off + nsh * qblob_bytes(D));
  l.hdr = off; off = al256(off + sizeof(GHeader));
  l.groups = off; off = al256(off + ngroups * sizeof(Group));
  l.cta_first = off; off = al256(off + N * sizeof(int));
  l.partials = off; off = al256(off + static_cast<size_t>(l.cap_parts) * partial_stride(G, D) * sizeof(float));
  l.total = off;
  return l;
}

// Ring depth for the kernel variant PAIR at its CTAs per SM (2 for PAIR 1, 1 for PAIR 2).
template <int D, int PAIR>
int g_choose_ring(int device) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess) return -1;
  if (cudaFuncSetAttribute(gattn_kernel<D, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess)
    return -1;
  const int want = PAIR == 1 ? 2 : 1;
  for (int ns = 16; ns >= 2; --ns) {
    const size_t smem = gattn_smem_bytes<D>(ns);
    if (smem > static_cast<size_t>(optin)) continue;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, gattn_kernel<D, PAIR>, GTHREADS, smem) != cudaSuccess)
      return -1;
    if (blocks >= want) return ns;
  }
  return -1;
}

template <int D>
int g_launch(kv4_cache* c, AttnParams p, void* ws, cudaStream_t stream, void (*merge)(const AttnParams&, cudaStream_t)) {
  const GLayout l = g_layout(c, p.n_seqs);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.seqhead = reinterpret_cast<SeqHead*>(wsb + l.seqhead);
  p.qblob = wsb + l.qblob;
  p.partials = reinterpret_cast<float*>(wsb + l.partials);
  p.cap_parts = l.cap_parts;
  const int per_sm = c->gattn_pair == 1 ? 2 : 1;
  p.grid = c->num_sms * per_sm;
  p.ns = c->gattn_ring;
  Group* groups = reinterpret_cast<Group*>(wsb + l.groups);
  int* cta_first = reinterpret_cast<int*>(wsb + l.cta_first);
  GHeader* hdr = reinterpret_cast<GHeader*>(wsb + l.hdr);
  const int nsh = p.n_seqs * p.Hkv;
  const int n_qblocks = (nsh + 31) / 32;
  const size_t prep_smem = static_cast<size_t>(32) * p.G * D * sizeof(float);
  if (prep_smem > 48 * 1024 &&
      cudaFuncSetAttribute(gprep_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(prep_smem)) !=
          cudaSuccess)
    return KV4_ERR_CUDA;
  gprep_kernel<D><<<n_qblocks + 1, 1024, prep_smem, stream>>>(p, groups, cta_first, hdr, n_qblocks);
  if (c->ev_before) cudaEventRecord(c->ev_before, stream);
  if (c->gattn_pair == 1)
    gattn_kernel<D, 1><<<p.grid, GTHREADS, gattn_smem_bytes<D>(p.ns), stream>>>(p, groups, cta_first, hdr);
  else
    gattn_kernel<D, 2><<<p.grid, GTHREADS, gattn_smem_bytes<D>(p.ns), stream>>>(p, groups, cta_first, hdr);
  if (c->ev_after) cudaEventRecord(c->ev_after, stream);
  merge(p, stream);
  return cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

}  // namespace

bool grouped_path(const kv4_cache* c) { return !c->bf16 && c->cfg.num_kv_heads % GW == 0; }

#ifndef KV4_GROUPED_PAIR
#define KV4_GROUPED_PAIR 2
#endif

int grouped_ring(kv4_cache* c) {
  c->gattn_pair = KV4_GROUPED_PAIR;
  if (c->cfg.head_dim == 128)
    return c->gattn_pair == 1 ? g_choose_ring<128, 1>(c->device) : g_choose_ring<128, 2>(c->device);
  return c->gattn_pair == 1 ? g_choose_ring<64, 1>(c->device) : g_choose_ring<64, 2>(c->device);
}

size_t grouped_workspace_bytes(const kv4_cache* c, int n_seqs) { return g_layout(c, n_seqs).total; }

int launch_grouped(kv4_cache* c, const AttnParams& p, void* ws, size_t ws_bytes, cudaStream_t stream,
                   void (*merge)(const AttnParams&, cudaStream_t)) {
  if (ws_bytes < g_layout(c, p.n_seqs).total) return KV4_ERR_WORKSPACE;
  if (c->gattn_ring <= 0) return KV4_ERR_UNSUPPORTED;
  return p.D == 128 ? g_launch<128>(c, p, ws, stream, merge) : g_launch<64>(c, p, ws, stream, merge);
}

}  // namespace kv4

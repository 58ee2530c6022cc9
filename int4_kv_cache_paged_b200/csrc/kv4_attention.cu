// Per-head split-K decode attention of the BF16 baseline cache.  (The INT4/INT8
// cache uses the page-major kernel of kv4_attention_grouped.cu for every head
// count; the INT4 branches of the templates below are not instantiated.)
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Abstract -- fused attention over a paged, token-wise INT4 cache whose
// keys were rotated by a block-diagonal Hadamard transform (the query receives the
// same rotation); "KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with
// INT4 KV Cache Quantization", Abstract -- sinks and recent positions are read
// from INT8.  Scale and zero point are folded out of the inner products, in the
// spirit of the folded-scale kernels of "KV Cache Quantization" (topic page),
// item 2:
//     q . k^  = s_k * (q . c_k) + z_k * sum(q)
//     sum_p a_p v^_p = sum_p (a_p s_p) c_p + sum_p a_p z_p
// so the tensor cores multiply raw integer codes (exact in fp16) by fp16 q
// (scaled by a power of two) and by fp16 a_p * s_p.
//
// Three kernels per call:
//   prep    one warp per (sequence, KV head): rotates the G queries (fp32 FWHT,
//           bf16 rounding), lays them out as B operands, and cuts the sequence
//           into work items (chunks of 16-token tiles plus one item for the INT8
//           store), appended to three lists by atomics: full chunks, tail chunks,
//           protected items -- largest first for the dynamic scheduler.
//   attn    persistent, 2 CTAs per SM, 7 consumer warps + 1 producer warp.  The
//           producer claims items with an atomic counter and streams their tiles
//           into a shared-memory ring with 1-D bulk copies (mbarrier completion);
//           consumer warp w takes the tiles j with j % 7 == w (j counts tiles over
//           the CTA's whole item stream), turns codes into
//           16x8x16 tensor-core operands in registers, keeps an online softmax per
//           query head, and the 7 warps merge into one partial (m, l, o) per item.
//   merge   one warp per (sequence, query head): log-sum-exp merge of the item
//           partials, inverse Hadamard rotation, store.
#include "kv4_attn_tiles.cuh"

#include <math.h>

namespace kv4 {


namespace {

using namespace tiles;

constexpr int NW = 7;                  // consumer warps (+1 producer: 16 warps per SM at 2 CTAs)
constexpr int THREADS = 32 * (NW + 1); // + producer warp
constexpr int QD = 2;                  // item queue depth
constexpr int PREP_WARPS = 4;

// Ring of shared-memory stages filled by the producer.  Stage s is always
// consumed by warp s % NW: global tile j goes to stage j % ns and warp j % NW,
// and ns is a multiple of NW.  A warp therefore waits on the phases of each of
// its stages strictly in order, which the mbarrier parity test needs (bulk
// copies may land out of order, so a stage must never be queried two phases
// ahead of the last fill its consumer has seen).
// A stage holds one unit: two INT4 tiles (32 tokens), one INT8 tile, or one BF16 tile.
template <int D, bool BF16>
struct KCfg {
  static constexpr int UNIT4 = 2;   // INT4 tiles per unit
  static constexpr int STAGE = BF16 ? tile16_bytes(D)
                                    : (UNIT4 * tile4_bytes(D) > tile8_bytes(D) ? UNIT4 * tile4_bytes(D) : tile8_bytes(D));
  static constexpr int QBLOB = qblob_bytes(D);
};
constexpr int NS_CHOICES[4] = {4 * NW, 3 * NW, 2 * NW, NW};


template <int D, bool BF16>
__host__ __device__ inline size_t attn_smem_bytes(int G, int ns) {
  using C = KCfg<D, BF16>;
  return static_cast<size_t>(ns) * C::STAGE + static_cast<size_t>(QD) * C::QBLOB +
         static_cast<size_t>(NW) * G * head_stride(D) * sizeof(float) + QD * sizeof(Item) +
         (2 * ns + 2 * QD) * sizeof(uint64_t) + 16 + ns * sizeof(int);
}

// ---------------------------------------------------------------------------
// prep: query rotation + work items

template <int D, bool BF16>
__global__ void __launch_bounds__(32 * PREP_WARPS) prep_kernel(AttnParams p) {
  extern __shared__ float s_q[];  // [PREP_WARPS][G][D]
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int gw = blockIdx.x * PREP_WARPS + wib;
  if (gw >= p.n_seqs * p.Hkv) return;
  const int b = gw / p.Hkv, h = gw % p.Hkv;
  const int G = p.G;
  const int seq = p.seq_ids[b];
  int L = 0;
  if (seq >= 0 && seq < p.max_seqs) {
    L = p.seq_lens[seq];
  } else if (lane == 0) {
    atomicOr(&p.state->status, KV4_DEV_BAD_SEQ);
  }

  // ---- work items
  int lo4, hi4, nprot;
  if (BF16 || (p.mode & KV4_MODE_INT4_ONLY)) {
    lo4 = 0; hi4 = L; nprot = 0;
  } else {
    nprot = min(L, p.S + p.W);
    lo4 = p.S; hi4 = L - p.W;
  }
  int t0 = 0, t1 = 0;
  if (hi4 > lo4) { t0 = lo4 / TILE; t1 = (hi4 + TILE - 1) / TILE; }
  const int C = p.chunk_tiles;
  const int tiles = t1 - t0;
  const int nfull = tiles / C, rem = (tiles % C) ? 1 : 0, prot = nprot > 0 ? 1 : 0;
  const int nparts = nfull + rem + prot;
  int base0 = 0, base1 = 0, base2 = 0, pbase = 0;
  if (lane == 0) {
    if (nfull) base0 = atomicAdd(&p.state->n_items[0], nfull);
    if (rem) base1 = atomicAdd(&p.state->n_items[1], 1);
    if (prot) base2 = atomicAdd(&p.state->n_items[2], 1);
    if (nparts) pbase = atomicAdd(&p.state->n_parts, nparts);
    if (base0 + nfull > p.cap[0] || base1 + rem > p.cap[1] || base2 + prot > p.cap[2] ||
        pbase + nparts > p.cap_parts)
      atomicOr(&p.state->status, KV4_DEV_WORKSPACE);
  }
  base0 = __shfl_sync(0xffffffffu, base0, 0);
  base1 = __shfl_sync(0xffffffffu, base1, 0);
  base2 = __shfl_sync(0xffffffffu, base2, 0);
  pbase = __shfl_sync(0xffffffffu, pbase, 0);
  const int kind4 = BF16 ? 2 : 0;
  for (int j = lane; j < nfull; j += 32) {
    if (base0 + j >= p.cap[0]) break;
    Item it{};
    it.b = b; it.seq = seq; it.h = h; it.kind = kind4;
    it.t_begin = t0 + j * C; it.t_end = t0 + (j + 1) * C;
    it.lo = lo4; it.hi = hi4; it.part = pbase + j;
    p.items[0][base0 + j] = it;
  }
  if (lane == 0) {
    if (rem && base1 < p.cap[1]) {
      Item it{};
      it.b = b; it.seq = seq; it.h = h; it.kind = kind4;
      it.t_begin = t0 + nfull * C; it.t_end = t1;
      it.lo = lo4; it.hi = hi4; it.part = pbase + nfull;
      p.items[1][base1] = it;
    }
    if (prot && base2 < p.cap[2]) {
      Item it{};
      it.b = b; it.seq = seq; it.h = h; it.kind = 1;
      it.t_begin = 0; it.t_end = (nprot + TILE - 1) / TILE;
      it.lo = 0; it.hi = nprot; it.part = pbase + nfull + rem;
      p.items[2][base2] = it;
    }
    SeqHead sh;
    sh.part_base = pbase; sh.n_parts = nparts; sh.len = L; sh.pad = 1;
    p.seqhead[gw] = sh;
  }

  // ---- queries: rotate (INT4 cache), round to bf16, lay out as B operands
  build_qblob<D, BF16>(p, b, h, lane, s_q + wib * G * D);
}

template <int D, bool BF16>
__device__ __forceinline__ const uint8_t* tile_source(const AttnParams& p, const Item& it, int tile) {
  if (it.kind == 1)
    return p.prot + ((static_cast<long long>(it.seq) * n_prot_tiles(p.S, p.W) + tile) * p.Hkv + it.h) *
                        tile8_bytes(D);
  const int pos = tile * TILE;
  int page = p.block_table[static_cast<long long>(it.seq) * p.max_pages_per_seq + pos / p.P];
  if (page < 0 || page >= p.num_pages) {
    atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
    page = 0;
  }
  constexpr int TB = BF16 ? tile16_bytes(D) : tile4_bytes(D);
  return p.pool + ((static_cast<long long>(page) * (p.P / TILE) + (pos % p.P) / TILE) * p.Hkv + it.h) * TB;
}

__device__ __forceinline__ void named_barrier_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * NW) : "memory");
}


// Bounded wait used only to drain this CTA's own bulk copies before exit.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 1000000000ull) return;
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(THREADS, 2) attn_kernel(AttnParams p) {
  using C = KCfg<D, BF16>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  const int NS = p.ns;
  uint8_t* qbuf = ring + NS * C::STAGE;
  float* merge = reinterpret_cast<float*>(qbuf + QD * C::QBLOB);
  Item* itemq = reinterpret_cast<Item*>(merge + NW * p.G * head_stride(D));
  uint64_t* bars = reinterpret_cast<uint64_t*>(itemq + QD);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NS + 2 * QD);
  volatile int* go_flag = abort_flag + 1;
  int* last_fill = const_cast<int*>(abort_flag) + 4;   // [NS]: global index of the last tile copied into each stage
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * NS;
  const uint32_t iqf0 = full0 + 16 * NS, iqe0 = iqf0 + 8 * QD;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
    for (int s = 0; s < QD; ++s) { mbar_init(iqf0 + 8 * s, 1); mbar_init(iqe0 + 8 * s, NW); }
    *abort_flag = 0;
    *go_flag = 0;
    for (int st = 0; st < NS; ++st) last_fill[st] = -1;
    fence_barrier_init();
  }
  __syncthreads();

  const int n0 = min(p.state->n_items[0], p.cap[0]);
  const int n1 = min(p.state->n_items[1], p.cap[1]);
  const int n2 = min(p.state->n_items[2], p.cap[2]);
  const int total = n0 + n1 + n2;
  int* status = &p.state->status;

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    // Claims run one item ahead: while the tiles of `cur` stream, the item
    // after it is loaded and the one after that is claimed.
    auto load_item = [&](int k) -> Item {
      if (k < n0) return p.items[0][k];
      if (k < n0 + n1) return p.items[1][k - n0];
      return p.items[2][k - n0 - n1];
    };
    int k_cur = 0, k_nxt = 0;
    if (lane == 0) { k_cur = atomicAdd(&p.state->work, 1); k_nxt = atomicAdd(&p.state->work, 1); }
    k_cur = __shfl_sync(0xffffffffu, k_cur, 0);
    k_nxt = __shfl_sync(0xffffffffu, k_nxt, 0);
    Item cur{};
    if (k_cur < total) cur = load_item(k_cur);
    const int nbatch = NS < 32 ? NS : 32;
    auto units_of = [&](const Item& itm) {
      const int UT = (BF16 || itm.kind == 1) ? 1 : C::UNIT4;
      return (itm.t_end - itm.t_begin + UT - 1) / UT;
    };
    auto source = [&](const Item& itm, int u, int k) -> const uint8_t* {   // tile k of unit u
      const int UT = (BF16 || itm.kind == 1) ? 1 : C::UNIT4;
      const int i = u * UT + k;
      const uint8_t* a = nullptr;
      if (lane < nbatch && k < UT && i < itm.t_end - itm.t_begin) {
        a = tile_source<D, BF16>(p, itm, itm.t_begin + i);
#ifdef KV4_DEBUG_CHECKS
        const uint8_t* lo = itm.kind == 1 ? p.prot : p.pool;
        const size_t ext = itm.kind == 1 ? p.prot_bytes : p.pool_bytes;
        const uint32_t tb = itm.kind == 1 ? tile8_bytes(D) : (BF16 ? tile16_bytes(D) : tile4_bytes(D));
        if (a < lo || a + tb > lo + ext) { dbg_fail(10, a - lo, ext); a = nullptr; }
#endif
      }
      return a;
    };
    const uint8_t* pre0 = nullptr;
    const uint8_t* pre1 = nullptr;
    bool have_pre = false;
    Item nxt{};
    uint32_t it = 0;
    int q = 0;
    bool ok = true;
    for (;; ++q) {
      const int slot = q % QD;
      if (lane == 0) ok = mbar_wait(iqe0 + 8 * slot, ((q / QD) & 1) ^ 1, abort_flag, status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (k_cur >= total) {
        if (lane == 0) { itemq[slot].kind = -1; mbar_arrive(iqf0 + 8 * slot); }
        break;
      }
      nxt = Item{};
      if (k_nxt < total) nxt = load_item(k_nxt);
      int k_new = total;
      if (lane == 0 && k_nxt < total) k_new = atomicAdd(&p.state->work, 1);
#ifdef KV4_DEBUG_CHECKS
      if (static_cast<size_t>(cur.b * p.Hkv + cur.h + 1) * C::QBLOB > p.qblob_total) dbg_fail(11, cur.b, cur.h);
      if (!KV4_SMEM_OK(smem_u32(itemq + slot), sizeof(Item), 4, 12)) { ok = false; }
#endif
      if (lane == 0) {
        itemq[slot] = cur;
        mbar_arrive_expect_tx(iqf0 + 8 * slot, C::QBLOB);
        bulk_g2s(smem_u32(qbuf + slot * C::QBLOB),
                 p.qblob + static_cast<size_t>(cur.b * p.Hkv + cur.h) * C::QBLOB, C::QBLOB, iqf0 + 8 * slot);
      }
      // a unit is UT tiles (2 for INT4 pages, 1 for INT8 and BF16 tiles) copied into one stage
      const int nunits = units_of(cur);
      const uint32_t tbytes = cur.kind == 1 ? tile8_bytes(D) : (BF16 ? tile16_bytes(D) : tile4_bytes(D));
      // Lanes issue in parallel, one unit each; a batch of at most NS units never
      // uses a stage twice, so every lane waits only for its own stage.  Source
      // addresses (block-table lookups) are loaded one batch ahead, and those of
      // the next item's first batch while this item streams.
      const uint8_t* nxt0 = have_pre ? pre0 : source(cur, lane, 0);
      const uint8_t* nxt1 = have_pre ? pre1 : source(cur, lane, 1);
      have_pre = false;
      for (int base = 0; base < nunits; base += nbatch) {
        const uint8_t* src0 = nxt0;
        const uint8_t* src1 = nxt1;
        nxt0 = source(cur, base + nbatch + lane, 0);
        nxt1 = source(cur, base + nbatch + lane, 1);
        bool lane_ok = true;
        if (lane < nbatch && base + lane < nunits) {
          const uint32_t j = it + base + lane;
          const int s = j % NS;
          lane_ok = src0 != nullptr && mbar_wait(empty0 + 8 * s, ((j / NS) & 1) ^ 1, abort_flag, status);
          if (lane_ok) {
            const uint32_t dst = smem_u32(ring + static_cast<size_t>(s) * C::STAGE);
            mbar_arrive_expect_tx(full0 + 8 * s, src1 ? 2 * tbytes : tbytes);
            bulk_g2s(dst, src0, tbytes, full0 + 8 * s);
            if (src1) bulk_g2s(dst + tbytes, src1, tbytes, full0 + 8 * s);
            last_fill[s] = static_cast<int>(j);
          } else {
            *abort_flag = 1;
          }
        }
        ok = __all_sync(0xffffffffu, lane_ok);
        if (!ok) break;
        if (base == 0 && k_nxt < total) {
          // the next item's descriptor has arrived by now: start its first block-table loads
          pre0 = source(nxt, lane, 0);
          pre1 = source(nxt, lane, 1);
          have_pre = true;
        }
      }
      it += nunits;
      if (!ok) break;
      cur = nxt;
      k_cur = k_nxt;
      k_nxt = __shfl_sync(0xffffffffu, k_new, 0);
    }
    if (!ok && lane == 0) {
      // aborted: let this CTA's copies land before the shared memory is released
      for (int st = 0; st < NS; ++st)
        if (last_fill[st] >= 0) mbar_drain(full0 + 8 * st, (last_fill[st] / NS) & 1);
      for (int j = q > QD ? q - QD : 0; j < q; ++j) mbar_drain(iqf0 + 8 * (j % QD), (j / QD) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int pstride = partial_stride(G, D);
  ColSplit cs;
  cs.colsplit = !BF16 && (G == 1 || G == 2 || G == 4);
  cs.part0 = cs.colsplit ? (2 * t) / G : 0;
  cs.part1 = cs.colsplit ? (2 * t + 1) / G : 0;
  uint32_t it = 0;
  for (int q = 0;; ++q) {
    const int slot = q % QD;
    const uint32_t iq_parity = (q / QD) & 1;
    if (warp == 0 && lane == 0) {
      const bool ok = mbar_wait(iqf0 + 8 * slot, iq_parity, abort_flag, status);
      *go_flag = ok && itemq[slot].kind >= 0;
    }
    named_barrier_consumers();  // uniform exit decision; also orders the previous combine before new merge writes
    if (!*go_flag) break;
    mbar_wait(iqf0 + 8 * slot, iq_parity, abort_flag, status);  // completed: acquire for this thread
    const Item cur = itemq[slot];
    QFrag<D> qf;
    {
      const uint32_t qb = smem_u32(qbuf + slot * C::QBLOB);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        const uint4 v = lds128(qb + 16 * (32 * c + lane));
        qf.b[2 * c][0] = v.x; qf.b[2 * c][1] = v.y; qf.b[2 * c + 1][0] = v.z; qf.b[2 * c + 1][1] = v.w;
      }
      const float* tail = reinterpret_cast<const float*>(qbuf + slot * C::QBLOB + 16 * D);
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

    const int ntiles = cur.t_end - cur.t_begin;
    const int UT = (BF16 || cur.kind == 1) ? 1 : C::UNIT4;
    const int nunits = (ntiles + UT - 1) / UT;
    // this warp's units: global unit index j = it + u with j % NW == warp (it owns stage j % NS)
    const int u0 = (warp - static_cast<int>(it % NW) + NW) % NW;
    for (int u = u0; u < nunits; u += NW) {
      const uint32_t j = it + u;
      const int s = j % NS;
      if (!mbar_wait(full0 + 8 * s, (j / NS) & 1, abort_flag, status)) break;
      const uint32_t st = smem_u32(ring + static_cast<size_t>(s) * C::STAGE);
      const int tile0 = cur.t_begin + u * UT;
      const int nt = min(UT, cur.t_end - tile0);
      const int pos0 = tile0 * TILE;
      const bool inside = pos0 >= cur.lo && pos0 + nt * TILE <= cur.hi;
      // bits 0-1: token g visible to both columns; bits 2-3: token g+8 (one query token per sequence here)
      auto valid_bits = [&](int k) {
        const int pg = pos0 + k * TILE + g;
        return (pg >= cur.lo && pg < cur.hi ? 3 : 0) | (pg + 8 >= cur.lo && pg + 8 < cur.hi ? 12 : 0);
      };
      const uint32_t eb = empty0 + 8 * s;
      if constexpr (BF16) {
        const int vb = valid_bits(0);
        if (inside) {
          tile_bf16<D, false>(st, qf, ws, lane, true, true, eb, 0u, 0u);
        } else {
          auto ok_pos = [&](int r) { return pos0 + r >= cur.lo && pos0 + r < cur.hi; };
          const uint32_t m01 = (ok_pos(2 * t) ? 0x0000FFFFu : 0u) | (ok_pos(2 * t + 1) ? 0xFFFF0000u : 0u);
          const uint32_t m89 = (ok_pos(2 * t + 8) ? 0x0000FFFFu : 0u) | (ok_pos(2 * t + 9) ? 0xFFFF0000u : 0u);
          tile_bf16<D, true>(st, qf, ws, lane, vb & 1, vb & 4, eb, m01, m89);
        }
      } else if (cur.kind == 1) {
        const int vb = valid_bits(0);
        if (inside) tile_int8<D, false>(st, qf, ws, lane, 15, eb, cs);
        else tile_int8<D, true>(st, qf, ws, lane, vb, eb, cs);
      } else {
        const int valid[2] = {valid_bits(0), valid_bits(1)};
        const uint32_t tl[2] = {st, st + static_cast<uint32_t>(tile4_bytes(D))};
        const uint32_t ebs[2] = {eb, eb};
        if (nt == 2) {
          if (inside) unit_int4<D, 2, false>(tl, qf, ws, lane, valid, ebs, cs);
          else unit_int4<D, 2, true>(tl, qf, ws, lane, valid, ebs, cs);
        } else {
          if (inside) unit_int4<D, 1, false>(tl, qf, ws, lane, valid, ebs, cs);
          else unit_int4<D, 1, true>(tl, qf, ws, lane, valid, ebs, cs);
        }
      }
    }
    it += nunits;

    // ---- merge the NW warps into one partial
    if (cs.colsplit) {
      // fold the low-part columns into the high-part ones (column c + G into column c)
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
    constexpr int HS = head_stride(D);
    float* mw = merge + warp * G * HS;
#ifdef KV4_DEBUG_CHECKS
    if (!KV4_SMEM_OK(smem_u32(mw), G * HS * 4, 4, 13)) continue;
#endif
    const int h0 = 2 * t, h1 = 2 * t + 1;
    if (h0 < G) {
      float* r = mw + h0 * HS;
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { r[16 * m + g] = ws.o[m][0] + ws.z0; r[16 * m + g + 8] = ws.o[m][2] + ws.z0; }
      if (g == 0) { r[D] = ws.m0; r[D + 1] = ws.l0; }
    }
    if (h1 < G) {
      float* r = mw + h1 * HS;
#pragma unroll
      for (int m = 0; m < D / 16; ++m) { r[16 * m + g] = ws.o[m][1] + ws.z1; r[16 * m + g + 8] = ws.o[m][3] + ws.z1; }
      if (g == 0) { r[D] = ws.m1; r[D + 1] = ws.l1; }
    }
    named_barrier_consumers();
    if (cur.part >= 0 && cur.part < p.cap_parts) {
      float* part = p.partials + static_cast<size_t>(cur.part) * pstride;
      for (int idx = warp * 32 + lane; idx < G * D; idx += NW * 32) {
        const int hq = idx / D, d = idx % D;
        float M = NEG_INF;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[(w * G + hq) * HS + D]);
        float acc = 0.f, lsum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float* r = merge + (w * G + hq) * HS;
          const float mwv = r[D];
          if (mwv > NEG_INF) {
            const float f = ex2(mwv - M);
            acc = fmaf(f, r[d], acc);
            lsum = fmaf(f, r[D + 1], lsum);
          }
        }
        part[hq * HS + d] = acc;
        if (d == 0) { part[hq * HS + D] = M; part[hq * HS + D + 1] = lsum; }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// merge: log-sum-exp over the item partials, inverse rotation, store

template <int D, bool BF16>
__global__ void __launch_bounds__(256) merge_kernel(AttnParams p) {
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    // the attention kernel has finished: re-arm the per-call counters
    p.state->n_items[0] = 0; p.state->n_items[1] = 0; p.state->n_items[2] = 0;
    p.state->n_parts = 0; p.state->work = 0;
  }
  if (gw >= p.n_seqs * p.Hq) return;
  const int b = gw / p.Hq, hq = gw % p.Hq, h = hq / p.G, gq = hq % p.G;
  const SeqHead sh = p.seqhead[b * p.Hkv + h];
  const int pstride = partial_stride(p.G, D);
  float o[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) o[i] = 0.f;
  const int stride = sh.pad;
  if (sh.n_parts > 0 && sh.part_base >= 0 && stride >= 1 && sh.part_base + (sh.n_parts - 1) * stride < p.cap_parts) {
    const float* base = p.partials + static_cast<size_t>(sh.part_base) * pstride + gq * head_stride(D);
    const size_t step = static_cast<size_t>(stride) * pstride;
    float M = NEG_INF;
    for (int j = 0; j < sh.n_parts; ++j) M = fmaxf(M, base[j * step + D]);
    float lsum = 0.f;
    for (int j = 0; j < sh.n_parts; ++j) {
      const float* r = base + j * step;
      const float f = ex2(r[D] - M);
      lsum = fmaf(f, r[D + 1], lsum);
      if constexpr (VPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(r + 4 * lane);
        o[0] = fmaf(f, v.x, o[0]); o[1] = fmaf(f, v.y, o[1]); o[2] = fmaf(f, v.z, o[2]); o[3] = fmaf(f, v.w, o[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(r + 2 * lane);
        o[0] = fmaf(f, v.x, o[0]); o[1] = fmaf(f, v.y, o[1]);
      }
    }
    const float inv = 1.f / lsum;
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[i] *= inv;
    if constexpr (!BF16) {
      fwht_row<VPL>(o, p.Bh_o, lane);   // o = H_blk o_rot (the normalised Hadamard matrix is its own inverse)
#pragma unroll
      for (int i = 0; i < VPL; ++i) o[i] *= p.rc_o;
    }
  }
  const size_t off = (static_cast<size_t>(b) * p.Hq + hq) * D + VPL * lane;
  if (p.mode & KV4_MODE_OUT_F32) {
    float* out = static_cast<float*>(p.out) + off;
#pragma unroll
    for (int i = 0; i < VPL; ++i) out[i] = o[i];
  } else {
    uint16_t* out = static_cast<uint16_t*>(p.out) + off;
#pragma unroll
    for (int i = 0; i < VPL; ++i) out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(o[i]));
  }
}

// ---------------------------------------------------------------------------
// host side

struct WsLayout {
  size_t seqhead, qblob, items0, items1, items2, partials, total;
  int cap0, cap_side, cap_parts;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline int chunk_tiles_for(const kv4_cache* c, int n_seqs) {
  const kv4_config& cfg = c->cfg;
  const long long cap_tiles = static_cast<long long>(cfg.max_pages_per_seq) * cfg.page_size / TILE + 1;
  const long long work = static_cast<long long>(n_seqs) * cfg.num_kv_heads * cap_tiles;
  const long long target = 4LL * c->num_sms * (c->attn_blocks_per_sm > 0 ? c->attn_blocks_per_sm : 2);
  long long ct = (work + target - 1) / target;
  if (ct < 8) ct = 8;
  if (ct > 64) ct = 64;
  return static_cast<int>(ct);
}

inline WsLayout ws_layout(const kv4_cache* c, int n_seqs, int cap0) {
  const kv4_config& cfg = c->cfg;
  const int G = cfg.num_q_heads / cfg.num_kv_heads, D = cfg.head_dim;
  const size_t nsh = static_cast<size_t>(n_seqs) * cfg.num_kv_heads;
  WsLayout w{};
  w.cap0 = cap0;
  w.cap_side = static_cast<int>(nsh);
  w.cap_parts = cap0 + 2 * static_cast<int>(nsh);
  size_t off = 0;
  w.seqhead = off; off = align256(off + nsh * sizeof(SeqHead));
  w.qblob = off; off = align256(off + nsh * qblob_bytes(D));
  w.items0 = off; off = align256(off + static_cast<size_t>(cap0) * sizeof(Item));
  w.items1 = off; off = align256(off + nsh * sizeof(Item));
  w.items2 = off; off = align256(off + nsh * sizeof(Item));
  w.partials = off; off = align256(off + static_cast<size_t>(w.cap_parts) * partial_stride(G, D) * sizeof(float));
  w.total = off;
  return w;
}

// Deepest ring (a multiple of NW) that keeps 2 CTAs per SM, else 1 CTA per SM.
template <int D, bool BF16>
int choose_ring(int device, int G, int* blocks_per_sm) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess) return -1;
  // the attribute is per kernel and process-wide: allow the device maximum once
  if (cudaFuncSetAttribute(attn_kernel<D, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess)
    return -1;
  for (int want = 2; want >= 1; --want) {
    for (int ns : NS_CHOICES) {
      const size_t smem = attn_smem_bytes<D, BF16>(G, ns);
      if (smem > static_cast<size_t>(optin)) continue;
      int blocks = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, attn_kernel<D, BF16>, THREADS, smem) != cudaSuccess)
        return -1;
      if (blocks >= want) {
        *blocks_per_sm = blocks > 2 ? 2 : blocks;
        return ns;
      }
    }
  }
  return -1;
}

template <int D, bool BF16>
int launch_attention_t(kv4_cache* c, AttnParams& p, cudaStream_t stream) {
  const int blocks_per_sm = c->attn_blocks_per_sm;
  if (blocks_per_sm <= 0) return KV4_ERR_UNSUPPORTED;
  const int nsh = p.n_seqs * p.Hkv;
  const size_t prep_smem = static_cast<size_t>(PREP_WARPS) * p.G * D * sizeof(float);
  prep_kernel<D, BF16><<<(nsh + PREP_WARPS - 1) / PREP_WARPS, 32 * PREP_WARPS, prep_smem, stream>>>(p);
  // no more CTAs than items can exist
  long long max_items = static_cast<long long>(p.cap[0]) + p.cap[1] + p.cap[2];
  long long grid = static_cast<long long>(c->num_sms) * blocks_per_sm;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  if (c->ev_before) cudaEventRecord(c->ev_before, stream);
  attn_kernel<D, BF16><<<static_cast<unsigned>(grid), THREADS, attn_smem_bytes<D, BF16>(p.G, p.ns), stream>>>(p);
  if (c->ev_after) cudaEventRecord(c->ev_after, stream);
  const int merge_warps = p.n_seqs * p.Hq;
  merge_kernel<D, BF16><<<(merge_warps + 7) / 8, 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

}  // namespace

#ifdef KV4_DEBUG_CHECKS
extern "C" int kv4_debug_read(unsigned long long* out4) {
  if (cudaMemcpyFromSymbol(out4, kv4_debug_slot, 4 * sizeof(unsigned long long)) != cudaSuccess) return KV4_ERR_CUDA;
  const unsigned long long zero[4] = {0, 0, 0, 0};
  return cudaMemcpyToSymbol(kv4_debug_slot, zero, sizeof(zero)) == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}
#endif

int attention_blocks_per_sm(kv4_cache* c) {
  if (!c->bf16) return -1;   // INT4 caches use the page-major kernel (kv4_attention_grouped.cu)
  const int G = c->cfg.num_q_heads / c->cfg.num_kv_heads;
  int blocks = 0;
  const int ns = c->cfg.head_dim == 128 ? choose_ring<128, true>(c->device, G, &blocks)
                                        : choose_ring<64, true>(c->device, G, &blocks);
  if (ns <= 0) return -1;
  c->attn_ring = ns;
  return blocks;
}

// Rotations the kernels apply to q and to the output: the cache's block
// Hadamard, unless the mode says the caller folded it into its projections.
void set_rotations(AttnParams& p, int mode) {
  const bool qr = (mode & KV4_MODE_Q_ROTATED) != 0, orot = (mode & KV4_MODE_OUT_ROTATED) != 0;
  p.Bh_q = qr ? 1 : p.Bh;
  p.rc_q = qr ? 1.f : p.rot_c;
  p.Bh_o = orot ? 1 : p.Bh;
  p.rc_o = orot ? 1.f : p.rot_c;
}

// Fields of AttnParams shared by both attention paths.
void fill_common(const kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* q, void* out,
                 float softmax_scale, int mode, AttnParams& p) {
  const kv4_config& cfg = c->cfg;
  const uint8_t* lbase = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  p.pool = lbase;
  p.prot = c->bf16 ? nullptr : lbase + c->pool_bytes;
  p.block_table = c->block_table;
  p.seq_lens = c->seq_lens + static_cast<size_t>(layer) * cfg.max_seqs;
  p.seq_ids = seq_ids;
  p.q = static_cast<const uint16_t*>(q);
  p.out = out;
  p.state = c->state;
  p.n_seqs = n_seqs;
  p.Hq = cfg.num_q_heads;
  p.Hkv = cfg.num_kv_heads;
  p.G = cfg.num_q_heads / cfg.num_kv_heads;
  p.Gh = p.G;
  p.qlen = 1;
  p.q0 = 0;
  p.qtot = 1;
  p.D = cfg.head_dim;
  p.P = cfg.page_size;
  p.S = cfg.sink_tokens;
  p.W = cfg.recent_window;
  p.Bh = c->bf16 ? 1 : cfg.hadamard_block;
  p.rot_c = static_cast<float>(1.0 / sqrt(static_cast<double>(p.Bh)));
  set_rotations(p, mode);
  if (mode & KV4_MODE_ROPE_Q) p.rope = c->rope;
  p.max_seqs = cfg.max_seqs;
  p.num_pages = cfg.num_pages;
  p.max_pages_per_seq = cfg.max_pages_per_seq;
  p.mode = mode;
  const double scale = softmax_scale > 0.f ? static_cast<double>(softmax_scale) : 1.0 / sqrt(static_cast<double>(p.D));
  p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  p.pool_bytes = c->pool_bytes;
  p.prot_bytes = c->prot_bytes;
  p.qblob_total = static_cast<size_t>(n_seqs) * cfg.num_kv_heads * qblob_bytes(p.D);
}

size_t attention_workspace_bytes(const kv4_cache* c, int n_seqs, int max_ctx) {
  if (grouped_path(c)) return grouped_workspace_bytes(c, n_seqs, 1);
  const kv4_config& cfg = c->cfg;
  const long long cap_ctx = static_cast<long long>(cfg.max_pages_per_seq) * cfg.page_size;
  const long long ctx = (max_ctx <= 0 || max_ctx > cap_ctx) ? cap_ctx : max_ctx;
  const long long tiles = (ctx + TILE - 1) / TILE + 1;
  const int ct = chunk_tiles_for(c, n_seqs);
  const long long cap0 = static_cast<long long>(n_seqs) * cfg.num_kv_heads * ((tiles + ct - 1) / ct);
  return ws_layout(c, n_seqs, static_cast<int>(cap0)).total;
}

// Query tokens of one pass of the multi-token path: as many as fit the
// 8 operand columns of a KV head.
int extend_chunk(const kv4_cache* c, int qlen) {
  const int per = MAX_G / (c->cfg.num_q_heads / c->cfg.num_kv_heads);
  return qlen < per ? qlen : per;
}

// Attention of the last qlen positions of every sequence (the page-major path
// with (tokens of a pass) * Hq/Hkv operand columns per KV head; token i of a
// sequence of length L sees the positions 0 .. L - qlen + i).  More tokens
// than one operand holds run as several passes over the cache, in stream
// order, sharing the workspace.
int launch_extend_attention(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, int qlen, const void* q,
                            void* out, float softmax_scale, int mode, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
  if (!grouped_path(c)) return KV4_ERR_UNSUPPORTED;
  AttnParams p{};
  fill_common(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, p);
  const int chunk = extend_chunk(c, qlen);
  p.qtot = qlen;
  for (int q0 = 0; q0 < qlen; q0 += chunk) {
    p.q0 = q0;
    p.qlen = qlen - q0 < chunk ? qlen - q0 : chunk;
    p.G = p.qlen * p.Gh;
    const int rc = launch_grouped(c, p, ws, ws_bytes, stream);
    if (rc != KV4_OK) return rc;
  }
  return KV4_OK;
}

int launch_attention(kv4_cache* c, int layer, const int32_t* seq_ids, int n_seqs, const void* q, void* out,
                     float softmax_scale, int mode, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const kv4_config& cfg = c->cfg;
  const int D = cfg.head_dim;
  const int G = cfg.num_q_heads / cfg.num_kv_heads;
  if (grouped_path(c)) {
    AttnParams p{};
    fill_common(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, p);
    return launch_grouped(c, p, ws, ws_bytes, stream);
  }
  // largest first-list capacity that fits the caller's workspace
  const WsLayout w0 = ws_layout(c, n_seqs, 0);
  const size_t per_item = sizeof(Item) + static_cast<size_t>(partial_stride(G, D)) * sizeof(float);
  if (ws_bytes < w0.total) return KV4_ERR_WORKSPACE;
  long long cap0 = static_cast<long long>((ws_bytes - w0.total) / per_item);
  if (cap0 > (1LL << 30)) cap0 = 1LL << 30;
  WsLayout w = ws_layout(c, n_seqs, static_cast<int>(cap0));
  while (w.total > ws_bytes && cap0 > 0) { --cap0; w = ws_layout(c, n_seqs, static_cast<int>(cap0)); }
  if (w.total > ws_bytes) return KV4_ERR_WORKSPACE;

  AttnParams p{};
  const uint8_t* lbase = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.pool = lbase;
  p.prot = c->bf16 ? nullptr : lbase + c->pool_bytes;
  p.block_table = c->block_table;
  p.seq_lens = c->seq_lens + static_cast<size_t>(layer) * cfg.max_seqs;
  p.seq_ids = seq_ids;
  p.q = static_cast<const uint16_t*>(q);
  p.out = out;
  p.state = c->state;
  p.items[0] = reinterpret_cast<Item*>(wsb + w.items0);
  p.items[1] = reinterpret_cast<Item*>(wsb + w.items1);
  p.items[2] = reinterpret_cast<Item*>(wsb + w.items2);
  p.cap[0] = w.cap0;
  p.cap[1] = w.cap_side;
  p.cap[2] = w.cap_side;
  p.seqhead = reinterpret_cast<SeqHead*>(wsb + w.seqhead);
  p.qblob = wsb + w.qblob;
  p.partials = reinterpret_cast<float*>(wsb + w.partials);
  p.pool_bytes = c->pool_bytes;
  p.prot_bytes = c->prot_bytes;
  p.qblob_total = static_cast<size_t>(n_seqs) * cfg.num_kv_heads * qblob_bytes(D);
  p.cap_parts = w.cap_parts;
  p.n_seqs = n_seqs;
  p.Hq = cfg.num_q_heads;
  p.Hkv = cfg.num_kv_heads;
  p.G = G;
  p.Gh = G;
  p.qlen = 1;
  p.q0 = 0;
  p.qtot = 1;
  p.D = D;
  p.P = cfg.page_size;
  p.S = cfg.sink_tokens;
  p.W = cfg.recent_window;
  p.Bh = c->bf16 ? 1 : cfg.hadamard_block;
  p.rot_c = static_cast<float>(1.0 / sqrt(static_cast<double>(p.Bh)));
  set_rotations(p, mode);
  if (mode & KV4_MODE_ROPE_Q) p.rope = c->rope;
  p.max_seqs = cfg.max_seqs;
  p.num_pages = cfg.num_pages;
  p.max_pages_per_seq = cfg.max_pages_per_seq;
  p.chunk_tiles = chunk_tiles_for(c, n_seqs);
  p.ns = c->attn_ring;
  p.mode = mode;
  const double scale = softmax_scale > 0.f ? static_cast<double>(softmax_scale) : 1.0 / sqrt(static_cast<double>(D));
  p.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  if (!c->bf16) return KV4_ERR_UNSUPPORTED;   // INT4 caches took the page-major path above
  return D == 128 ? launch_attention_t<128, true>(c, p, stream) : launch_attention_t<64, true>(c, p, stream);
}

}  // namespace kv4

// Fused rotate + quantize + pack + append, the BF16 append, debug dequantization
// and sequence reset.
//
// Method: "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving", Abstract -- a fused kernel rotates new K/V with a block-diagonal
// Hadamard transform, quantizes them token-wise to INT4 and writes them straight
// into the paged layout; "KV4-RL: Unlocking Faster Asynchronous Rollouts for
// RLVR with INT4 KV Cache Quantization", Abstract -- sinks and recent tokens are
// also kept in INT8.
//
// One warp handles one (token, KV head, K-or-V) group of D values, D/32 values
// per lane at dims VPL*lane .. VPL*lane+VPL-1.  The fp32 arithmetic follows a
// fixed order so the codes are reproducible bit for bit:
//   rotation: butterfly stages h = 1, 2, ..., Bh/2 (x_i, x_{i+h}) ->
//             (x_i + x_{i+h}, x_i - x_{i+h}), then one multiply by fp32(1/sqrt(Bh));
//   quantizer: clamp to +-65504; z = fp16 round-down(min); r = max - z;
//             s = fp16 round-up(r / Q) (1 when r == 0); code = rint((x - z) / s)
//             clamped to [0, Q]; every operation round-to-nearest-even fp32.
#include "kv4_append_ops.cuh"

namespace kv4 {

namespace {

constexpr int APPEND_WARPS = 8;

__device__ __forceinline__ int find_seq(const int* cu, int n_seqs, int n) {
  int lo = 0, hi = n_seqs;  // largest i with cu[i] <= n
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= n) lo = mid; else hi = mid;
  }
  return lo;
}

// Last block of an append launch: advance the sequence lengths (from the old
// lengths every block read at its start; not when the row offsets were
// invalid) and re-arm the counter.
__device__ void finish_append(const AppendParams& p, const int* s_cu, const int* s_seq, const int* s_len,
                              bool bad_cu) {
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = (atomicAdd(&p.state->append_done, 1) == static_cast<int>(gridDim.x) - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int cap = p.max_pages_per_seq * p.P;
  for (int i = threadIdx.x; i < (bad_cu ? 0 : p.n_seqs); i += blockDim.x) {
    const int seq = s_seq[i];
    if (seq < 0 || seq >= p.max_seqs) continue;
    const int n = s_cu[i + 1] - s_cu[i];
    const int L = s_len[i];
    if (n > 0 && L + n <= cap) p.seq_lens[seq] = L + n;
  }
  __syncthreads();
  if (threadIdx.x == 0) p.state->append_done = 0;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(32 * APPEND_WARPS) append_kernel(AppendParams p) {
  constexpr int VPL = D / 32;
  // cu_new [n+1], then the sequence ids [n], then their lengths before this append [n]
  extern __shared__ int s_meta[];
  int* s_cu = s_meta;
  int* s_seq = s_meta + p.n_seqs + 1;
  int* s_len = s_seq + p.n_seqs;
  __shared__ __align__(16) uint8_t s_codes[APPEND_WARPS][2][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i <= p.n_seqs; i += blockDim.x) {
    s_cu[i] = p.cu_new[i];
    if (i < p.n_seqs) s_seq[i] = p.seq_ids[i];
  }
  __syncthreads();
  // the row offsets must run 0 = cu[0] <= cu[1] <= ... <= cu[n] = total_new: otherwise a
  // row could land past its sequence's new length, so nothing is written
  int bad = 0;
  for (int i = threadIdx.x; i < p.n_seqs; i += blockDim.x) {
    const int seq = s_seq[i];
    s_len[i] = (seq >= 0 && seq < p.max_seqs) ? p.seq_lens[seq] : 0;
    bad |= s_cu[i] > s_cu[i + 1];
  }
  if (threadIdx.x == 0) bad |= s_cu[0] != 0 || s_cu[p.n_seqs] != p.total_new;
  const bool bad_cu = __syncthreads_or(bad) != 0;
  if (bad_cu && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&p.state->status, KV4_DEV_BAD_CU);

  const long long job = static_cast<long long>(blockIdx.x) * APPEND_WARPS + warp;
  const long long n_jobs = static_cast<long long>(p.total_new) * p.Hkv * 2;
  if (job < n_jobs && !bad_cu) {
    const int tensor = static_cast<int>(job & 1);
    const int h = static_cast<int>((job >> 1) % p.Hkv);
    const int n = static_cast<int>((job >> 1) / p.Hkv);
    // the row's values first: their load overlaps the dependent metadata loads below
    uint16_t raw[VPL];
    {
      const uint16_t* src = (tensor ? p.v_new : p.k_new) + (static_cast<long long>(n) * p.Hkv + h) * D;
      if constexpr (VPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(src + 4 * lane);
        raw[0] = u.x & 0xFFFF; raw[1] = u.x >> 16; raw[2] = u.y & 0xFFFF; raw[3] = u.y >> 16;
      } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(src + 2 * lane);
        raw[0] = u & 0xFFFF; raw[1] = u >> 16;
      }
    }
    const int i = find_seq(s_cu, p.n_seqs, n);
    const int seq = s_seq[i];
    const int cap = p.max_pages_per_seq * p.P;
    bool ok = true;
    if (seq < 0 || seq >= p.max_seqs) {
      if (lane == 0) atomicOr(&p.state->status, KV4_DEV_BAD_SEQ);
      ok = false;
    }
    int pos = 0, L_new = 0;
    if (ok) {
      const int L_old = s_len[i];
      L_new = L_old + (s_cu[i + 1] - s_cu[i]);
      pos = L_old + (n - s_cu[i]);
      if (L_new > cap) {
        if (lane == 0) atomicOr(&p.state->status, KV4_DEV_OVERFLOW);
        ok = false;
      }
    }
    if (ok && tensor == 0 && p.rope.cs != nullptr && pos >= p.rope.max_pos) {
      if (lane == 0) atomicOr(&p.state->status, KV4_DEV_ROPE_POS);
      ok = false;
    }
    int page = -1;
    if (ok) {
      page = p.block_table[static_cast<long long>(seq) * p.max_pages_per_seq + pos / p.P];
      if (page < 0 || page >= p.num_pages) {
        if (lane == 0) atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
        ok = false;
      }
    }
    if (ok) {
      const int r = pos & (TILE - 1);
      // head-innermost pool: [page][P/16][Hkv][tile]
      const long long tile_idx = (static_cast<long long>(page) * (p.P / TILE) + (pos % p.P) / TILE) * p.Hkv + h;
      if constexpr (BF16) {
        uint16_t* tile = reinterpret_cast<uint16_t*>(p.pool + tile_idx * tile16_bytes(D));
        // share the row through smem so each lane can store element pairs
        uint16_t* row = reinterpret_cast<uint16_t*>(s_codes[warp][0]);
#pragma unroll
        for (int k = 0; k < VPL; ++k) row[VPL * lane + k] = raw[k];
        __syncwarp();
        const int rowhi = r >> 3, g = r & 7;
        if (tensor == 0) {
          for (int q = lane; q < D / 2; q += 32) {   // q = (k, h8, t): dims 16k + 8h8 + 2t + {0,1}
            const int k = q >> 3, h8 = (q >> 2) & 1, t = q & 3;
            const int d = 16 * k + 8 * h8 + 2 * t;
            const uint32_t v = static_cast<uint32_t>(row[d]) | (static_cast<uint32_t>(row[d + 1]) << 16);
            *reinterpret_cast<uint32_t*>(tile + 8 * (32 * k + 4 * g + t) + 2 * (rowhi + 2 * h8)) = v;
          }
        } else {
          const int t = (r & 7) >> 1, e = r & 1, th = r >> 3;
          for (int d = lane; d < D; d += 32) {
            const int m = d >> 4, dh = (d >> 3) & 1, gg = d & 7;
            tile[16 * D + 8 * (32 * m + 4 * gg + t) + 2 * (dh + 2 * th) + e] = row[d];
          }
        }
      } else {
        encode_row<D>(p, raw, tensor, h, seq, pos, L_new, tile_idx, r, s_codes[warp][0], s_codes[warp][1], lane);
      }
    }
  }
  finish_append(p, s_cu, s_seq, s_len, bad_cu);
}

// ---------------------------------------------------------------------------

struct DequantParams {
  const uint8_t* pool;
  const uint8_t* prot;
  const int32_t* block_table;
  const int32_t* seq_lens;
  State* state;
  float* k_out;
  float* v_out;
  int seq, start, count, view;
  int Hkv, D, P, S, W, max_pages_per_seq, num_pages;
  int fmt;   // page format
};

__global__ void dequant_kernel(DequantParams p) {
  const int lane = threadIdx.x & 31;
  const long long job = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (job >= static_cast<long long>(p.count) * p.Hkv * 2) return;
  const int tensor = static_cast<int>(job & 1);
  const int h = static_cast<int>((job >> 1) % p.Hkv);
  const int j = static_cast<int>((job >> 1) / p.Hkv);
  const int pos = p.start + j;
  const int L = p.seq_lens[p.seq];
  const int D = p.D;
  float* out = (tensor ? p.v_out : p.k_out) + (static_cast<long long>(j) * p.Hkv + h) * D;
  const bool protect = p.view == KV4_VIEW_EFFECTIVE && (pos < p.S || pos >= L - p.W);
  if (protect) {
    const int slot = pos < p.S ? pos : p.S + (pos - p.S) % p.W;
    const int r = slot & 15;
    const uint8_t* tile = p.prot + ((static_cast<long long>(p.seq) * n_prot_tiles(p.S, p.W) + slot / 16) * p.Hkv + h) *
                                       tile8_bytes(D);
    const uint32_t sz = *reinterpret_cast<const uint32_t*>(tile + 32 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3)));
    const float s = half_lo(sz), z = half_hi(sz);
    for (int d = lane; d < D; d += 32) {
      int off;
      if (tensor == 0) {
        const int kk = d >> 5, hf = (d >> 4) & 1, t = (d >> 2) & 3, j = d & 3;
        off = r * D + (D / 4) * t + 4 * (2 * kk + hf) + j;
      } else {
        const int m = d >> 4, dh = (d >> 3) & 1, gg = d & 7, th = r >> 3, t = (r & 7) >> 1, e = r & 1;
        const int w = 2 * m + th;
        off = 16 * D + 16 * (32 * (w >> 2) + 4 * gg + t) + 4 * (w & 3) + dh + 2 * e;
      }
      out[d] = __fmaf_rn(static_cast<float>(tile[off]), s, z);
    }
  } else {
    const int page = p.block_table[static_cast<long long>(p.seq) * p.max_pages_per_seq + pos / p.P];
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) atomicOr(&p.state->status, KV4_DEV_BAD_PAGE);
      return;
    }
    const int r = pos & 15;
    if (p.fmt == KV4_FORMAT_NVFP4) {   // x^ = e2m1(code) * e4m3(scale of the 16-dim block)
      const uint8_t* tile = p.pool + ((static_cast<long long>(page) * (p.P / 16) + (pos % p.P) / 16) * p.Hkv + h) *
                                         tilef_bytes(D);
      const int g = r & 7, rh = r >> 3, th = r >> 3, t = (r & 7) >> 1, e = r & 1;
      for (int d = lane; d < D; d += 32) {
        int byte, half, sbyte;
        if (tensor == 0) {
          const int b = d >> 4, tt = (d >> 2) & 3, j = (d >> 1) & 1;
          byte = 16 * (4 * g + tt) + 4 * (b & 3) + 512 * (b >> 2) + rh + 2 * j;
          half = d & 1;
          sbyte = 16 * D + (D / 8) * g + 2 * b + rh;
        } else {
          const int m = d >> 4, dh = (d >> 3) & 1, gg = d & 7;
          byte = 8 * D + 16 * (4 * gg + t) + 4 * (m & 3) + 512 * (m >> 2) + dh + 2 * th;
          half = e;
          sbyte = 17 * D + (D / 4) * t + 4 * m + 2 * th + e;
        }
        const uint32_t code = (tile[byte] >> (4 * half)) & 15u;
        const uint32_t ee = (code >> 1) & 3u, mm = code & 1u;
        const float mag = ee == 0u ? 0.5f * static_cast<float>(mm) : ldexpf(1.f + 0.5f * static_cast<float>(mm), ee - 1);
        out[d] = (code & 8u ? -mag : mag) * e4m3_value(tile[sbyte]);
      }
      return;
    }
    if (p.fmt == KV4_FORMAT_INT2) {   // x^ = fma(code, s, z), 2-bit codes
      const uint8_t* tile = p.pool + ((static_cast<long long>(page) * (p.P / 16) + (pos % p.P) / 16) * p.Hkv + h) *
                                         tile2_bytes(D);
      const uint32_t sz = *reinterpret_cast<const uint32_t*>(tile + 8 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3)));
      const float s = half_lo(sz), z = half_hi(sz);
      const int th = r >> 3, t = (r & 7) >> 1, e = r & 1;
      for (int d = lane; d < D; d += 32) {
        int byte, c;
        if (tensor == 0) {
          const int kq = d >> 6, cc = (d >> 4) & 3, tt = (d >> 2) & 3, j = d & 3;
          byte = r * (D / 4) + tt * (D / 16) + 4 * kq + j;
          c = cc;
        } else {
          const int m = d >> 4, mp = m >> 1, mb = m & 1, dh = (d >> 3) & 1, g = d & 7;
          byte = 4 * D + (D / 8) * (4 * g + t) + 4 * mp + th + 2 * e;
          c = dh + 2 * mb;
        }
        const int code = (tile[byte] >> (2 * c)) & 3;
        out[d] = __fmaf_rn(static_cast<float>(code), s, z);
      }
      return;
    }
    const uint8_t* tile = p.pool + ((static_cast<long long>(page) * (p.P / 16) + (pos % p.P) / 16) * p.Hkv + h) *
                                       tile4_bytes(D);
    const uint32_t sz = *reinterpret_cast<const uint32_t*>(tile + 16 * D + 16 * (r & 7) + 4 * (2 * tensor + (r >> 3)));
    const float s = half_lo(sz), z = half_hi(sz);
    for (int d = lane; d < D; d += 32) {
      int byte, half;
      if (tensor == 0) {
        const int kk = d >> 5, hf = (d >> 4) & 1, t = (d >> 2) & 3, j = d & 3;
        byte = r * (D / 2) + t * (D / 8) + 4 * kk + j;
        half = hf;
      } else {
        const int m = d >> 4, dh = (d >> 3) & 1, g = d & 7, th = r >> 3, t = (r & 7) >> 1, e = r & 1;
        byte = 8 * D + 512 * (m >> 2) + 16 * (4 * g + t) + 4 * (m & 3) + th + 2 * e;
        half = dh;
      }
      const int code = (tile[byte] >> (4 * half)) & 15;
      out[d] = __fmaf_rn(static_cast<float>(code), s, z);
    }
  }
}

__global__ void seq_reset_kernel(int32_t* seq_lens, int num_layers, int max_seqs, int seq) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l < num_layers) seq_lens[static_cast<long long>(l) * max_seqs + seq] = 0;
}

}  // namespace

int launch_append(kv4_cache* c, int layer, const int32_t* seq_ids, const int32_t* cu_new, int n_seqs, int total_new,
                  const void* k_new, const void* v_new, bool rope, cudaStream_t stream) {
  const AppendParams p = append_params(c, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, rope);
  const long long jobs = static_cast<long long>(total_new) * p.Hkv * 2;
  const long long blocks = (jobs + APPEND_WARPS - 1) / APPEND_WARPS;
  if (blocks > 0x7fffffffLL) return KV4_ERR_UNSUPPORTED;
  const size_t smem = sizeof(int) * (3 * static_cast<size_t>(n_seqs) + 1);
  if (smem > 40 * 1024) return KV4_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(blocks)), block(32 * APPEND_WARPS);
  if (p.D == 128) {
    if (c->bf16) append_kernel<128, true><<<grid, block, smem, stream>>>(p);
    else append_kernel<128, false><<<grid, block, smem, stream>>>(p);
  } else {
    if (c->bf16) append_kernel<64, true><<<grid, block, smem, stream>>>(p);
    else append_kernel<64, false><<<grid, block, smem, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

int launch_dequantize_debug(kv4_cache* c, int layer, int seq_id, int start, int count, int view, float* k_out,
                            float* v_out, cudaStream_t stream) {
  const kv4_config& cfg = c->cfg;
  DequantParams p{};
  const uint8_t* lbase = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  p.pool = lbase;
  p.prot = lbase + c->pool_bytes;
  p.block_table = c->block_table;
  p.seq_lens = c->seq_lens + static_cast<size_t>(layer) * cfg.max_seqs;
  p.state = c->state;
  p.k_out = k_out;
  p.v_out = v_out;
  p.seq = seq_id;
  p.start = start;
  p.count = count;
  p.view = view;
  p.Hkv = cfg.num_kv_heads;
  p.D = cfg.head_dim;
  p.P = cfg.page_size;
  p.S = cfg.sink_tokens;
  p.W = cfg.recent_window;
  p.max_pages_per_seq = cfg.max_pages_per_seq;
  p.num_pages = cfg.num_pages;
  p.fmt = cfg.page_format;
  const long long threads = static_cast<long long>(count) * p.Hkv * 2 * 32;
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return KV4_ERR_UNSUPPORTED;
  dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

int launch_seq_reset(kv4_cache* c, int seq_id, cudaStream_t stream) {
  const int L = c->cfg.num_layers;
  seq_reset_kernel<<<(L + 127) / 128, 128, 0, stream>>>(c->seq_lens, L, c->cfg.max_seqs, seq_id);
  return cudaGetLastError() == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

}  // namespace kv4

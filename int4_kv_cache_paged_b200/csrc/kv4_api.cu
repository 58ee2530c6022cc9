// Host side of the kv4 C ABI: argument checks, carving of the caller's device
// buffer, launches.  No function here allocates device memory.
#include "kv4_common.cuh"

#include <math.h>
#include <new>

using kv4::State;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Validates the configuration; bf16 caches ignore the quantization fields.
int check_config(const kv4_config* c, bool bf16) {
  if (!c) return KV4_ERR_INVALID_ARG;
  if (c->num_layers < 1 || c->max_seqs < 1 || c->num_q_heads < 1 || c->num_kv_heads < 1 || c->num_pages < 1 ||
      c->max_pages_per_seq < 1)
    return KV4_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads) return KV4_ERR_INVALID_ARG;
  if (c->num_q_heads / c->num_kv_heads > kv4::MAX_G) return KV4_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return KV4_ERR_UNSUPPORTED;
  if (c->page_size < 16 || c->page_size % 16 || c->page_size > 1024) return KV4_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->max_pages_per_seq) * c->page_size > (1LL << 30)) return KV4_ERR_UNSUPPORTED;
  if (c->page_format != KV4_FORMAT_INT4 &&
      (bf16 || (c->page_format != KV4_FORMAT_NVFP4 && c->page_format != KV4_FORMAT_INT2)))
    return KV4_ERR_INVALID_ARG;
  if (!bf16) {
    if (!is_pow2(c->hadamard_block) || c->head_dim % c->hadamard_block) return KV4_ERR_INVALID_ARG;
    if (c->sink_tokens < 0 || c->recent_window < 1) return KV4_ERR_INVALID_ARG;
    if (c->sink_tokens + c->recent_window > 4096) return KV4_ERR_UNSUPPORTED;
  }
  return KV4_OK;
}

struct Sizes {
  size_t seq_lens, pool, prot, layer_stride, pool_offset, total;
};

Sizes sizes_of(const kv4_config* c, bool bf16) {
  Sizes s{};
  const size_t Hkv = c->num_kv_heads, D = c->head_dim;
  const size_t tiles_per_page = c->page_size / kv4::TILE;
  s.seq_lens = align_up(sizeof(int32_t) * static_cast<size_t>(c->num_layers) * c->max_seqs);
  const size_t tile = bf16 ? kv4::tile16_bytes(static_cast<int>(D))
                           : kv4::page_tile_bytes(static_cast<int>(D), c->page_format);
  s.pool = align_up(static_cast<size_t>(c->num_pages) * Hkv * tiles_per_page * tile);
  s.prot = bf16 ? 0
                : align_up(static_cast<size_t>(c->max_seqs) * Hkv * kv4::n_prot_tiles(c->sink_tokens, c->recent_window) *
                           kv4::tile8_bytes(static_cast<int>(D)));
  s.layer_stride = s.pool + s.prot;
  s.pool_offset = kv4::STATE_BYTES + s.seq_lens;
  s.total = s.pool_offset + s.layer_stride * c->num_layers;
  return s;
}

int create(const kv4_config* cfg, bool bf16, void* dev_buf, size_t bytes, int32_t* block_table,
           cudaStream_t stream, kv4_cache** out) {
  if (!out) return KV4_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_config(cfg, bf16);
  if (rc) return rc;
  if (!dev_buf || !block_table) return KV4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_buf) % kAlign || reinterpret_cast<uintptr_t>(block_table) % 4)
    return KV4_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg, bf16);
  if (bytes < s.total) return KV4_ERR_CAPACITY;
  kv4_cache* c = new (std::nothrow) kv4_cache();
  if (!c) return KV4_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->bf16 = bf16;
  c->test_stall = -1;
  // the cache lives on the device that owns its buffer
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, dev_buf) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    delete c;
    return KV4_ERR_INVALID_ARG;
  }
  c->device = attr.device;
  const kv4::DeviceScope dev(c->device);
  if (!dev.ok() || cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
    delete c;
    return KV4_ERR_CUDA;
  }
  c->base = static_cast<uint8_t*>(dev_buf);
  c->state = reinterpret_cast<State*>(c->base);
  c->seq_lens = reinterpret_cast<int32_t*>(c->base + kv4::STATE_BYTES);
  c->block_table = block_table;
  c->layer_stride = s.layer_stride;
  c->pool_offset = s.pool_offset;
  c->pool_bytes = s.pool;
  c->prot_bytes = s.prot;
  c->attn_blocks_per_sm = 0;
  if (bf16) {   // the BF16 baseline: per-head split-K kernel
    c->attn_blocks_per_sm = kv4::attention_blocks_per_sm(c);
    if (c->attn_blocks_per_sm <= 0) {
      delete c;
      return KV4_ERR_CUDA;
    }
  }
  c->gattn_ring = 0;
  if (kv4::grouped_path(c)) {
    c->gattn_ring = kv4::grouped_ring(c);
    if (c->gattn_ring <= 0) {
      delete c;
      return KV4_ERR_CUDA;
    }
  }
  if (cudaMemsetAsync(c->base, 0, s.pool_offset, stream) != cudaSuccess) {
    delete c;
    return KV4_ERR_CUDA;
  }
  *out = c;
  return KV4_OK;
}


int check_layer(const kv4_cache* c, int32_t layer) {
  return (layer < 0 || layer >= c->cfg.num_layers) ? KV4_ERR_INVALID_ARG : KV4_OK;
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

// Attention mode bits this cache accepts: RoPE of q needs a registered table
// and contradicts an already rotated query.
bool mode_ok(const kv4_cache* c, int32_t mode) {
  if (mode & ~(KV4_MODE_INT4_ONLY | KV4_MODE_OUT_F32 | KV4_MODE_Q_ROTATED | KV4_MODE_OUT_ROTATED | KV4_MODE_ROPE_Q))
    return false;
  if ((mode & KV4_MODE_ROPE_Q) && (c->rope.cs == nullptr || (mode & KV4_MODE_Q_ROTATED))) return false;
  return true;
}

int append(kv4_cache* c, int32_t layer, const int32_t* seq_ids, const int32_t* cu_new, int32_t n_seqs,
           int32_t total_new, const void* k_new, const void* v_new, cudaStream_t stream, bool rope = false) {
  if (!c || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (n_seqs < 0 || total_new < 0) return KV4_ERR_INVALID_ARG;
  if (n_seqs == 0 || total_new == 0) return KV4_OK;
  if (!seq_ids || !cu_new || !k_new || !v_new) return KV4_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_append(c, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, rope, stream);
}

int attention(kv4_cache* c, int32_t layer, const int32_t* seq_ids, int32_t n_seqs, const void* q, void* out,
              float softmax_scale, int32_t mode, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!c || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (n_seqs < 0 || n_seqs > c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  if (n_seqs == 0) return KV4_OK;
  if (!seq_ids || !q || !out || !ws) return KV4_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || reinterpret_cast<uintptr_t>(ws) % kAlign) return KV4_ERR_INVALID_ARG;
  if (!mode_ok(c, mode)) return KV4_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_attention(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, ws, ws_bytes, stream);
}

int extend_attention(kv4_cache* c, int32_t layer, const int32_t* seq_ids, int32_t n_seqs, int32_t q_len,
                     const void* q, void* out, float softmax_scale, int32_t mode, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  if (!c || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (n_seqs < 0 || n_seqs > c->cfg.max_seqs || q_len < 1) return KV4_ERR_INVALID_ARG;
  if (!kv4::grouped_path(c)) return KV4_ERR_UNSUPPORTED;
  if (n_seqs == 0) return KV4_OK;
  if (!seq_ids || !q || !out || !ws) return KV4_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || reinterpret_cast<uintptr_t>(ws) % kAlign) return KV4_ERR_INVALID_ARG;
  if (!mode_ok(c, mode)) return KV4_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_extend_attention(c, layer, seq_ids, n_seqs, q_len, q, out, softmax_scale, mode, ws, ws_bytes,
                                      stream);
}

int get_status(kv4_cache* c, cudaStream_t stream, int32_t* device_status) {
  if (!c || !device_status) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, &c->state->status, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return KV4_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KV4_ERR_CUDA;
  if (cudaMemsetAsync(&c->state->status, 0, sizeof(int32_t), stream) != cudaSuccess) return KV4_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KV4_ERR_CUDA;
  *device_status = v;
  return v ? KV4_ERR_DEVICE_FAULT : KV4_OK;
}

}  // namespace

extern "C" {

int kv4_cache_required_bytes(const kv4_config* cfg, size_t* bytes) {
  if (!bytes) return KV4_ERR_INVALID_ARG;
  const int rc = check_config(cfg, false);
  if (rc) return rc;
  *bytes = sizes_of(cfg, false).total;
  return KV4_OK;
}

int kv4_cache_create(const kv4_config* cfg, void* dev_buf, size_t bytes, int32_t* dev_block_table,
                     kv4_stream_t stream, kv4_cache** out) {
  return create(cfg, false, dev_buf, bytes, dev_block_table, reinterpret_cast<cudaStream_t>(stream), out);
}

int kv4_cache_destroy(kv4_cache* cache) {
  if (!cache) return KV4_ERR_INVALID_ARG;
  delete cache;
  return KV4_OK;
}

int kv4_cache_layout(const kv4_cache* c, int32_t layer, void** dev_pages, void** dev_protected,
                     int32_t** dev_seq_lens) {
  if (!c || c->bf16 || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  uint8_t* lbase = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  if (dev_pages) *dev_pages = lbase;
  if (dev_protected) *dev_protected = lbase + c->pool_bytes;
  if (dev_seq_lens) *dev_seq_lens = c->seq_lens;
  return KV4_OK;
}

int kv4_seq_reset(kv4_cache* c, int32_t seq_id, kv4_stream_t stream) {
  if (!c || seq_id < 0 || seq_id >= c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_seq_reset(c, seq_id, reinterpret_cast<cudaStream_t>(stream));
}

int kv4_rotate_quantize_append(kv4_cache* c, int32_t layer, const int32_t* seq_ids, const int32_t* cu_new,
                               int32_t n_seqs, int32_t total_new, const void* k_new, const void* v_new,
                               kv4_stream_t stream) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  return append(c, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, reinterpret_cast<cudaStream_t>(stream));
}

int kv4_set_rope(kv4_cache* c, const float* cos_sin, int32_t max_pos, int32_t rotary_dim, int32_t style) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  if (cos_sin == nullptr) {
    c->rope = kv4::RopeParams{nullptr, 0, 0, 0};
    return KV4_OK;
  }
  const int R = rotary_dim;
  if (max_pos < 1 || R < 32 || R > c->cfg.head_dim || (R & (R - 1)) != 0) return KV4_ERR_INVALID_ARG;
  if (style != KV4_ROPE_NEOX && style != KV4_ROPE_GPTJ) return KV4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(cos_sin) % alignof(float)) return KV4_ERR_INVALID_ARG;
  c->rope = kv4::RopeParams{cos_sin, max_pos, R, style};
  return KV4_OK;
}

int kv4_rope_rotate_quantize_append(kv4_cache* c, int32_t layer, const int32_t* seq_ids, const int32_t* cu_new,
                                    int32_t n_seqs, int32_t total_new, const void* k_new, const void* v_new,
                                    kv4_stream_t stream) {
  if (!c || c->bf16 || c->rope.cs == nullptr) return KV4_ERR_INVALID_ARG;
  return append(c, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, reinterpret_cast<cudaStream_t>(stream),
                true);
}

int kv4_attention_workspace_bytes(const kv4_cache* c, int32_t n_seqs, int32_t max_ctx, size_t* bytes) {
  if (!c || c->bf16 || !bytes || n_seqs < 0) return KV4_ERR_INVALID_ARG;
  *bytes = kv4::attention_workspace_bytes(c, n_seqs, max_ctx);
  return KV4_OK;
}

int kv4_decode_attention(kv4_cache* c, int32_t layer, const int32_t* seq_ids, int32_t n_seqs, const void* q,
                         void* out, float softmax_scale, int32_t mode, void* ws, size_t ws_bytes,
                         kv4_stream_t stream) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  return attention(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode, ws, ws_bytes,
                   reinterpret_cast<cudaStream_t>(stream));
}

int kv4_decode_step(kv4_cache* c, int32_t layer, const int32_t* seq_ids, int32_t n_seqs, const void* k_new,
                    const void* v_new, const void* q, void* out, float softmax_scale, int32_t mode, void* ws,
                    size_t ws_bytes, kv4_stream_t stream) {
  if (!c || c->bf16 || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (n_seqs < 0 || n_seqs > c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  if (n_seqs == 0) return KV4_OK;
  if (!seq_ids || !k_new || !v_new || !q || !out || !ws) return KV4_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out) ||
      reinterpret_cast<uintptr_t>(ws) % kAlign)
    return KV4_ERR_INVALID_ARG;
  if (!mode_ok(c, mode)) return KV4_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_decode_step(c, layer, seq_ids, n_seqs, k_new, v_new, q, out, softmax_scale, mode, ws, ws_bytes,
                                 reinterpret_cast<cudaStream_t>(stream));
}

int kv4_extend_workspace_bytes(const kv4_cache* c, int32_t n_seqs, int32_t q_len, size_t* bytes) {
  if (!c || c->bf16 || !bytes || n_seqs < 0 || q_len < 1) return KV4_ERR_INVALID_ARG;
  if (!kv4::grouped_path(c)) return KV4_ERR_UNSUPPORTED;
  *bytes = kv4::grouped_workspace_bytes(c, n_seqs, kv4::extend_chunk(c, q_len));
  return KV4_OK;
}

int kv4_extend_attention(kv4_cache* c, int32_t layer, const int32_t* seq_ids, int32_t n_seqs, int32_t q_len,
                         const void* q, void* out, float softmax_scale, int32_t mode, void* ws, size_t ws_bytes,
                         kv4_stream_t stream) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  return extend_attention(c, layer, seq_ids, n_seqs, q_len, q, out, softmax_scale, mode, ws, ws_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

int kv4_dequantize_debug(kv4_cache* c, int32_t layer, int32_t seq_id, int32_t start, int32_t count, int32_t view,
                         float* k_out, float* v_out, kv4_stream_t stream) {
  if (!c || c->bf16 || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (seq_id < 0 || seq_id >= c->cfg.max_seqs || start < 0 || count < 0) return KV4_ERR_INVALID_ARG;
  if (view != KV4_VIEW_EFFECTIVE && view != KV4_VIEW_INT4) return KV4_ERR_INVALID_ARG;
  if (static_cast<long long>(start) + count > static_cast<long long>(c->cfg.max_pages_per_seq) * c->cfg.page_size)
    return KV4_ERR_INVALID_ARG;
  if (count == 0) return KV4_OK;
  if (!k_out || !v_out) return KV4_ERR_INVALID_ARG;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  return kv4::launch_dequantize_debug(c, layer, seq_id, start, count, view, k_out, v_out,
                                      reinterpret_cast<cudaStream_t>(stream));
}

int kv4_get_status(kv4_cache* c, kv4_stream_t stream, int32_t* device_status) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  return get_status(c, reinterpret_cast<cudaStream_t>(stream), device_status);
}

int kv4_test_stall_next_attention(kv4_cache* c, int32_t stage) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  c->test_stall = stage < 0 ? -1 : stage;
  return KV4_OK;
}

int kv4_set_attention_events(kv4_cache* c, void* ev_before, void* ev_after) {
  if (!c || c->bf16) return KV4_ERR_INVALID_ARG;
  c->ev_before = static_cast<cudaEvent_t>(ev_before);
  c->ev_after = static_cast<cudaEvent_t>(ev_after);
  return KV4_OK;
}

const char* kv4_status_string(int status) {
  switch (status) {
    case KV4_OK: return "ok";
    case KV4_ERR_INVALID_ARG: return "invalid argument";
    case KV4_ERR_UNSUPPORTED: return "unsupported shape";
    case KV4_ERR_CAPACITY: return "buffer smaller than required";
    case KV4_ERR_CUDA: return "CUDA runtime error";
    case KV4_ERR_DEVICE_FAULT: return "device status bits set";
    case KV4_ERR_WORKSPACE: return "workspace too small";
    case KV4_ERR_SCRATCH: return "needs more scratch than the static no-alloc array holds";
    default: return "unknown status";
  }
}

const char* kv4_version(void) { return "kv4 0.1.0 sm_100a"; }

// ---- BF16 baseline

int kv4bf16_cache_required_bytes(const kv4_config* cfg, size_t* bytes) {
  if (!bytes) return KV4_ERR_INVALID_ARG;
  const int rc = check_config(cfg, true);
  if (rc) return rc;
  *bytes = sizes_of(cfg, true).total;
  return KV4_OK;
}

int kv4bf16_cache_create(const kv4_config* cfg, void* dev_buf, size_t bytes, int32_t* dev_block_table,
                         kv4_stream_t stream, kv4bf16_cache** out) {
  kv4_cache* c = nullptr;
  const int rc = create(cfg, true, dev_buf, bytes, dev_block_table, reinterpret_cast<cudaStream_t>(stream), &c);
  if (out) *out = reinterpret_cast<kv4bf16_cache*>(c);
  return rc;
}

int kv4bf16_cache_destroy(kv4bf16_cache* cache) {
  if (!cache) return KV4_ERR_INVALID_ARG;
  delete reinterpret_cast<kv4_cache*>(cache);
  return KV4_OK;
}

int kv4bf16_cache_layout(const kv4bf16_cache* cache, int32_t layer, void** dev_pages, int32_t** dev_seq_lens) {
  const kv4_cache* c = reinterpret_cast<const kv4_cache*>(cache);
  if (!c || !c->bf16 || check_layer(c, layer)) return KV4_ERR_INVALID_ARG;
  if (dev_pages) *dev_pages = c->base + c->pool_offset + static_cast<size_t>(layer) * c->layer_stride;
  if (dev_seq_lens) *dev_seq_lens = c->seq_lens;
  return KV4_OK;
}

int kv4bf16_append(kv4bf16_cache* cache, int32_t layer, const int32_t* seq_ids, const int32_t* cu_new,
                   int32_t n_seqs, int32_t total_new, const void* k_new, const void* v_new, kv4_stream_t stream) {
  kv4_cache* c = reinterpret_cast<kv4_cache*>(cache);
  if (!c || !c->bf16) return KV4_ERR_INVALID_ARG;
  return append(c, layer, seq_ids, cu_new, n_seqs, total_new, k_new, v_new, reinterpret_cast<cudaStream_t>(stream));
}

int kv4bf16_attention_workspace_bytes(const kv4bf16_cache* cache, int32_t n_seqs, int32_t max_ctx, size_t* bytes) {
  const kv4_cache* c = reinterpret_cast<const kv4_cache*>(cache);
  if (!c || !c->bf16 || !bytes || n_seqs < 0) return KV4_ERR_INVALID_ARG;
  *bytes = kv4::attention_workspace_bytes(c, n_seqs, max_ctx);
  return KV4_OK;
}

int kv4bf16_decode_attention(kv4bf16_cache* cache, int32_t layer, const int32_t* seq_ids, int32_t n_seqs,
                             const void* q, void* out, float softmax_scale, int32_t mode, void* ws, size_t ws_bytes,
                             kv4_stream_t stream) {
  kv4_cache* c = reinterpret_cast<kv4_cache*>(cache);
  if (!c || !c->bf16) return KV4_ERR_INVALID_ARG;
  return attention(c, layer, seq_ids, n_seqs, q, out, softmax_scale, mode & KV4_MODE_OUT_F32, ws, ws_bytes,
                   reinterpret_cast<cudaStream_t>(stream));
}

int kv4bf16_get_status(kv4bf16_cache* cache, kv4_stream_t stream, int32_t* device_status) {
  kv4_cache* c = reinterpret_cast<kv4_cache*>(cache);
  if (!c || !c->bf16) return KV4_ERR_INVALID_ARG;
  return get_status(c, reinterpret_cast<cudaStream_t>(stream), device_status);
}

int kv4bf16_set_attention_events(kv4bf16_cache* cache, void* ev_before, void* ev_after) {
  kv4_cache* c = reinterpret_cast<kv4_cache*>(cache);
  if (!c || !c->bf16) return KV4_ERR_INVALID_ARG;
  c->ev_before = static_cast<cudaEvent_t>(ev_before);
  c->ev_after = static_cast<cudaEvent_t>(ev_after);
  return KV4_OK;
}

}  // extern "C"

// kv4_decode_attention_noalloc: decode attention whose scratch lives in a
// static device array of this library instead of a caller-provided workspace.
// The method's pages have no counterpart of this call; it exists for callers
// that cannot allocate device memory per call (see include/kv4.h).
#include "kv4_common.cuh"

#include <mutex>

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(KV4_NOALLOC_SCRATCH_BYTES);

// One copy per device (a __device__ variable is instantiated in every device
// context that loads this module).  Nothing in it needs to start at zero: each
// call writes every scratch byte it reads before reading it.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of this device's scratch, looked up once per device with that
// device current (the caller's cache device, selected by the caller).
int scratch_of(int device, void** addr) {
  if (device < 0 || device >= kMaxDevices) return KV4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[device]) {
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != device) return KV4_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return KV4_ERR_CUDA;
    }
    g_scratch_addr[device] = p;
  }
  *addr = g_scratch_addr[device];
  return KV4_OK;
}

}  // namespace

extern "C" int kv4_decode_attention_noalloc(kv4_cache* c, int32_t layer, const int32_t* dev_seq_ids, int32_t n_seqs,
                                            const void* q, void* out, float softmax_scale, int32_t mode,
                                            kv4_stream_t stream) {
  if (!c || c->bf16 || n_seqs < 0 || n_seqs > c->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  if (n_seqs == 0) return KV4_OK;
  size_t need = 0;
  int rc = kv4_attention_workspace_bytes(c, n_seqs, 0, &need);
  if (rc != KV4_OK) return rc;
  if (need > kScratchBytes) return KV4_ERR_SCRATCH;
  const kv4::DeviceScope dev(c->device);   // the cache's device, restored on return
  if (!dev.ok()) return KV4_ERR_CUDA;
  void* scratch = nullptr;
  rc = scratch_of(c->device, &scratch);
  if (rc != KV4_OK) return rc;
  return kv4_decode_attention(c, layer, dev_seq_ids, n_seqs, q, out, softmax_scale, mode, scratch, kScratchBytes,
                              stream);
}

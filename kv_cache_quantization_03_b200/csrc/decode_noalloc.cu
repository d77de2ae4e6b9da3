// Decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run
// decode: a plug-in inside a serving process whose host owns every device
// allocation and offers no scratch hook, or a deployment that fixes its
// memory budget at start-up and forbids cudaMalloc afterwards.  For them this
// entry point keeps the split-KV partial results in a fixed array of this
// library (kNoAllocScratchBytes, allocated once per GPU when the library's
// device code is loaded and held until the process exits) instead of a
// workspace argument.  It allocates nothing and runs the same kernels as
// kvq_decode_attention.
#include <cuda_runtime.h>

#include <mutex>

#include "kvq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first
// call on a device looks it up (cudaGetSymbolAddress) and caches it; a
// device reset invalidates the cache, and a failed lookup or launch clears
// the entry so that the next call looks it up again.
kvq_status scratch_address(int* dev_out, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *dev_out = dev;
  *out = g_scratch_addr[dev];
  return KVQ_OK;
}

void forget_scratch_address(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_scratch_addr[dev] = nullptr;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache_view* cache,
                                                   int32_t layer, const void* q, const int32_t* block_table,
                                                   int32_t max_pages_per_seq, const int32_t* seq_lens,
                                                   int32_t batch, int32_t num_q_heads, float softmax_scale,
                                                   float* out, uint32_t* dev_error, void* stream) {
  if (!cfg || max_pages_per_seq < 0 || (int64_t)max_pages_per_seq * cfg->tile_tokens > INT32_MAX)
    return KVQ_ERR_INVALID_ARG;
  size_t need = 0;
  kvq_status st = kvq_decode_workspace_bytes(cfg, batch, num_q_heads,
                                             max_pages_per_seq * cfg->tile_tokens, &need);
  if (st != KVQ_OK) return st;
  if (need > kNoAllocScratchBytes) {
    // Too big for the scratch array.  The workspace call validates every
    // other argument first and launches nothing without a workspace, so a
    // bad argument is reported as such rather than as the size.
    return kvq_decode_attention(cfg, cache, layer, q, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                                softmax_scale, out, nullptr, 0, dev_error, stream);
  }
  void* scratch = nullptr;
  int dev = 0;
  if ((st = scratch_address(&dev, &scratch)) != KVQ_OK) return st;
  st = kvq_decode_attention(cfg, cache, layer, q, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                            softmax_scale, out, scratch, kNoAllocScratchBytes, dev_error, stream);
  if (st == KVQ_ERR_CUDA) forget_scratch_address(dev);
  return st;
}

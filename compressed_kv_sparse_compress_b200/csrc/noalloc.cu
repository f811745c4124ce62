// sparse_indexer_topk_noalloc: the scoring and top-k selection of sparse_indexer_topk, with the
// scratch memory taken from a fixed array that this library owns instead of from a workspace the
// caller allocates.
//
// Who needs it: callers that cannot allocate device memory. Examples are an extension loaded
// into a host program that owns all device memory and hands its extensions no allocator, and a
// latency-critical path where a device allocation would synchronize the whole device. Such a
// caller still passes every input and output buffer; only the scratch (query average, radix
// histograms, selection bitmap, boundary candidates and, when no score buffer is passed, the
// scores) comes from the array below.
//
// Cost and limits: the array is kNoAllocScratchBytes (16 MiB); every GPU that loads this library
// holds that much memory until the process exits. Sizes whose scratch would not fit are rejected
// with CKV_ERR_WORKSPACE before anything is enqueued. All calls share the one array and it keeps
// the last call's contents: the kernels reset what must start at zero (the histograms and the
// candidate counters) at the start of every call, and calls whose kernels overlap on the GPU
// (different streams, or different threads without ordering) race on the array.

#include <mutex>

#include "ckv_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device. In host code the array's name is a
// host-side stand-in, not a device address; the address a kernel can use comes from
// cudaGetSymbolAddress, asked once per device with that device current.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CKV_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CKV_OK;
}

}  // namespace

extern "C" int sparse_indexer_topk_noalloc(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache,
                                           int32_t batch, const int32_t* d_seq_len,
                                           int32_t max_seq_len, const float* d_q, int32_t top_k,
                                           int32_t* d_idx, int32_t* d_cnt, float* d_scores,
                                           uint32_t* d_status, void* stream) {
  // a bad configuration gets its own status from sparse_indexer_topk below (its size is 0 here)
  if (ckv_indexer_workspace_bytes(cfg, batch, max_seq_len, top_k) > kNoAllocScratchBytes)
    return CKV_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != CKV_OK) return st;
  return sparse_indexer_topk(cfg, cache, batch, d_seq_len, max_seq_len, d_q, top_k, d_idx, d_cnt,
                             d_scores, scratch, kNoAllocScratchBytes, d_status, stream);
}

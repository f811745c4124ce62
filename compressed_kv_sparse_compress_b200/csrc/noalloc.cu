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

#include <cuda.h>

#include <mutex>

#include "ckv_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchSlot {
  unsigned long long ctx_id;  // id of the context the address was looked up in (0: none yet)
  void* addr;
};

std::mutex g_scratch_mutex;
ScratchSlot g_scratch[kMaxDevices] = {};

template <typename Fn>
Fn driver_fn(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(f);
}

// Device address of g_noalloc_scratch in the current device's current context. In host code the
// array's name is a host-side stand-in, not a device address; the address a kernel can use comes
// from cudaGetSymbolAddress, asked with the device current. The answer is kept per device together
// with the id of the context it was asked in (ids are never reused within a process), and asked
// again when that context has been replaced (after cudaDeviceReset the module is loaded anew and
// the array may live elsewhere). Looking up the current context and its id are host-side driver
// queries that enqueue nothing.
int scratch_address(void** out) {
  static const CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_ctx || !get_id) return CKV_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return CKV_ERR_CUDA;
  void* p = nullptr;
  if (ctx == nullptr) {  // no context yet: the symbol lookup initialises the device's primary one
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CKV_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return CKV_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return CKV_ERR_CUDA;
  if (slot.ctx_id != id || slot.addr == nullptr) {
    if (p == nullptr && (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr))
      return CKV_ERR_CUDA;
    slot.ctx_id = id;
    slot.addr = p;
  }
  *out = slot.addr;
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

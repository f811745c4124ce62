// The C ABI of libckv (include/ckv.h): argument validation, block pools, workspace carving and
// dispatch to the kernels. Host code only; nothing here touches device memory directly.

#include <atomic>
#include <cmath>
#include <mutex>
#include <new>
#include <vector>

#include "ckv_internal.h"

namespace ckv {

static std::atomic<uint64_t> g_launches{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static cudaEvent_t g_prof[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};

void prof_begin(ProfPoint which, cudaStream_t stream) {
  if (g_prof[which][0]) cudaEventRecord(g_prof[which][0], stream);
}

void prof_end(ProfPoint which, cudaStream_t stream) {
  if (g_prof[which][1]) cudaEventRecord(g_prof[which][1], stream);
}

int sm_count() {
  static int cache[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Raises a kernel's dynamic shared-memory limit once per (device, kernel, larger size); later calls
// with the same or a smaller size make no CUDA call (so they are free inside graph capture too).
cudaError_t allow_smem(const void* kernel, int bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  struct Entry {
    int dev;
    const void* kernel;
    int bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& e : done)
    if (e.dev == dev && e.kernel == kernel && e.bytes >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({dev, kernel, bytes});
  return e;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int row_bytes_comp(int dtype, int D) {
  switch (dtype) {
    case CKV_F32: return 4 * D;
    case CKV_BF16: return 2 * D;
    case CKV_NVFP4: return D / 2;
    default: return -1;
  }
}

int row_bytes_win(int dtype, int D) {
  switch (dtype) {
    case CKV_F32: return 4 * D;
    case CKV_FP8_E4M3: return D;
    default: return -1;
  }
}

int check_cfg(const ckv_layer_cfg* c) {
  if (!c) return CKV_ERR_INVALID_ARG;
  if (c->num_heads < 1 || c->num_heads > 1024) return CKV_ERR_INVALID_ARG;
  if (c->ratio < 1 || c->ratio > 256 || !is_pow2(c->ratio)) return CKV_ERR_INVALID_ARG;
  if (c->window < 0 || c->window > 256) return CKV_ERR_INVALID_ARG;
  if (c->rope_dim < 0 || c->rope_dim > c->head_dim || (c->rope_dim & 1)) return CKV_ERR_INVALID_ARG;
  if (!(c->sm_scale >= 0.f) || !std::isfinite(c->sm_scale)) return CKV_ERR_INVALID_ARG;
  if (!(c->rope_base >= 0.f) || !std::isfinite(c->rope_base)) return CKV_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256 && c->head_dim != 512 &&
      c->head_dim != 1024)
    return CKV_ERR_UNSUPPORTED;
  if (row_bytes_comp(c->comp_dtype, c->head_dim) < 0) return CKV_ERR_UNSUPPORTED;
  if (row_bytes_win(c->win_dtype, c->head_dim) < 0) return CKV_ERR_UNSUPPORTED;
  return CKV_OK;
}

// Validates cfg + cache and fills the kernel parameter block. need_residue: the append path.
int make_params(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int batch, int max_seq_len,
                bool need_residue, LayerParams* p) {
  int st = check_cfg(cfg);
  if (st != CKV_OK) return st;
  if (!cache || batch < 1 || max_seq_len < 1) return CKV_ERR_INVALID_ARG;
  const int D = cfg->head_dim;
  if (!cache->comp_codes || !aligned16(cache->comp_codes)) return CKV_ERR_INVALID_ARG;
  if (cfg->comp_dtype == CKV_NVFP4 && (!cache->comp_scales || !aligned16(cache->comp_scales)))
    return CKV_ERR_INVALID_ARG;
  if (cfg->window > 0) {
    if (!cache->win_codes || !aligned16(cache->win_codes) || !cache->win_table ||
        !aligned16(cache->win_table) || cache->win_blocks < 1)
      return CKV_ERR_INVALID_ARG;
    if (cfg->win_dtype == CKV_FP8_E4M3 && (!cache->win_scales || !aligned16(cache->win_scales)))
      return CKV_ERR_INVALID_ARG;
  }
  if (!cache->comp_table || !aligned16(cache->comp_table) || cache->comp_blocks < 1)
    return CKV_ERR_INVALID_ARG;
  if (cache->table_stride < (static_cast<int64_t>(max_seq_len) + kBlockTokens - 1) / kBlockTokens)
    return CKV_ERR_INVALID_ARG;
  if (need_residue && (!cache->residue_kv || !aligned16(cache->residue_kv) || !cache->residue_logit ||
                       !aligned16(cache->residue_logit)))
    return CKV_ERR_INVALID_ARG;
  LayerParams& q = *p;
  q.H = cfg->num_heads;
  q.D = D;
  q.d_r = cfg->rope_dim;
  q.r = cfg->ratio;
  q.W = cfg->window;
  q.comp_dtype = cfg->comp_dtype;
  q.win_dtype = cfg->win_dtype;
  q.epb = kBlockTokens / cfg->ratio;
  q.comp_row_bytes = row_bytes_comp(cfg->comp_dtype, D);
  q.win_row_bytes = row_bytes_win(cfg->win_dtype, D);
  q.sm_scale = cfg->sm_scale > 0.f ? cfg->sm_scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  q.rope_base = cfg->rope_base > 0.f ? static_cast<double>(cfg->rope_base) : 10000.0;
  q.comp_codes = static_cast<uint8_t*>(cache->comp_codes);
  q.comp_scales = static_cast<uint8_t*>(cache->comp_scales);
  q.win_codes = static_cast<uint8_t*>(cache->win_codes);
  q.win_scales = cache->win_scales;
  q.res_kv = cache->residue_kv;
  q.res_logit = cache->residue_logit;
  q.comp_table = cache->comp_table;
  q.win_table = cache->win_table;
  q.table_stride = cache->table_stride;
  q.comp_blocks = cache->comp_blocks;
  q.win_blocks = cfg->window > 0 ? cache->win_blocks : 0;
  for (int i = 0; i < LayerParams::kRopeTable; ++i)
    q.inv_freq[i] = i < q.d_r / 2 ? std::pow(q.rope_base, -(2.0 * i) / static_cast<double>(q.d_r)) : 0.0;
  return CKV_OK;
}

// Validates the index config and plane. need_residue: the append path.
int make_index_params(const ckv_index_cfg* icfg, const ckv_index_cache* icache, bool need_residue,
                      IndexParams* ip) {
  if (!icfg || !icache) return CKV_ERR_INVALID_ARG;
  const int H = icfg->index_heads, d = icfg->index_dim;
  if (H < 16 || H > 128 || H % 16 != 0) return CKV_ERR_UNSUPPORTED;
  if (d != 128 && d != 256) return CKV_ERR_UNSUPPORTED;
  if (!icache->codes || !aligned16(icache->codes) || !icache->scales || !aligned16(icache->scales))
    return CKV_ERR_INVALID_ARG;
  if (need_residue && (!icache->residue_k || !aligned16(icache->residue_k) || !icache->residue_logit ||
                       !aligned16(icache->residue_logit)))
    return CKV_ERR_INVALID_ARG;
  ip->heads = H;
  ip->dim = d;
  ip->codes = static_cast<uint8_t*>(icache->codes);
  ip->scales = icache->scales;
  ip->res_k = icache->residue_k;
  ip->res_logit = icache->residue_logit;
  return CKV_OK;
}

// Workspace of the multi-head indexer: the query images, then the indexer's selection state.
size_t mh_ws_bytes(const LayerParams& p, const IndexParams& ip, int batch, int max_seq_len, IndexerWs* iw,
                   uint8_t** qimage, void* base) {
  const size_t img = mh_image_bytes(ip, batch);
  *iw = indexer_ws_layout(base ? static_cast<char*>(base) + img : nullptr, p, batch, max_seq_len);
  if (qimage) *qimage = static_cast<uint8_t*>(base);
  return img + iw->bytes;
}

}  // namespace
}  // namespace ckv

using namespace ckv;

struct ckv_pool {
  std::vector<int32_t> stack;    // free ids, top at the back
  std::vector<uint8_t> is_free;  // per id
};

extern "C" {

int kv_block_pool_create(int32_t num_blocks, ckv_pool** out) {
  if (!out || num_blocks < 1) return CKV_ERR_INVALID_ARG;
  ckv_pool* p = new (std::nothrow) ckv_pool;
  if (!p) return CKV_ERR_INVALID_ARG;
  p->stack.resize(num_blocks);
  for (int32_t i = 0; i < num_blocks; ++i) p->stack[i] = num_blocks - 1 - i;
  p->is_free.assign(num_blocks, 1);
  *out = p;
  return CKV_OK;
}

int kv_block_pool_destroy(ckv_pool* pool) {
  delete pool;
  return CKV_OK;
}

int kv_block_alloc(ckv_pool* pool, int32_t n, int32_t* out_ids) {
  if (!pool || n < 0 || (n > 0 && !out_ids)) return CKV_ERR_INVALID_ARG;
  if (static_cast<size_t>(n) > pool->stack.size()) return CKV_ERR_OUT_OF_BLOCKS;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = pool->stack.back();
    pool->stack.pop_back();
    pool->is_free[id] = 0;
    out_ids[i] = id;
  }
  return CKV_OK;
}

int kv_block_free(ckv_pool* pool, const int32_t* ids, int32_t n) {
  if (!pool || n < 0 || (n > 0 && !ids)) return CKV_ERR_INVALID_ARG;
  const int32_t nb = static_cast<int32_t>(pool->is_free.size());
  // validate everything first, so a bad call frees nothing
  std::vector<uint8_t> seen;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = ids[i];
    if (id < 0 || id >= nb || pool->is_free[id]) return CKV_ERR_INVALID_ARG;
  }
  seen.assign(nb, 0);
  for (int32_t i = 0; i < n; ++i) {
    if (seen[ids[i]]) return CKV_ERR_INVALID_ARG;
    seen[ids[i]] = 1;
  }
  for (int32_t i = 0; i < n; ++i) {
    pool->is_free[ids[i]] = 1;
    pool->stack.push_back(ids[i]);
  }
  return CKV_OK;
}

int32_t kv_block_pool_num_free(const ckv_pool* pool) {
  if (!pool) return CKV_ERR_INVALID_ARG;
  return static_cast<int32_t>(pool->stack.size());
}

int ckv_cache_row_bytes(const ckv_layer_cfg* cfg, size_t* comp_code_bytes, size_t* comp_scale_bytes,
                        size_t* win_code_bytes, size_t* win_scale_bytes) {
  const int st = check_cfg(cfg);
  if (st != CKV_OK) return st;
  const int D = cfg->head_dim;
  if (comp_code_bytes) *comp_code_bytes = static_cast<size_t>(row_bytes_comp(cfg->comp_dtype, D));
  if (comp_scale_bytes) *comp_scale_bytes = cfg->comp_dtype == CKV_NVFP4 ? static_cast<size_t>(D / 16) : 0;
  if (win_code_bytes) *win_code_bytes = static_cast<size_t>(row_bytes_win(cfg->win_dtype, D));
  if (win_scale_bytes) *win_scale_bytes = cfg->win_dtype == CKV_FP8_E4M3 ? sizeof(float) : 0;
  return CKV_OK;
}

int64_t ckv_score_stride(const ckv_layer_cfg* cfg, int32_t max_seq_len) {
  if (check_cfg(cfg) != CKV_OK || max_seq_len < 1) return 0;
  return score_stride(cfg->ratio, max_seq_len);
}

size_t ckv_indexer_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch, int32_t max_seq_len,
                                   int32_t top_k) {
  if (check_cfg(cfg) != CKV_OK || batch < 1 || max_seq_len < 1 || top_k < 1) return 0;
  LayerParams p{};
  p.D = cfg->head_dim;
  p.r = cfg->ratio;
  return indexer_ws_layout(nullptr, p, batch, max_seq_len).bytes;
}

size_t ckv_attention_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch, int32_t max_seq_len,
                                     int32_t max_selected) {
  if (check_cfg(cfg) != CKV_OK || batch < 1 || max_seq_len < 1 || max_selected < 0) return 0;
  LayerParams p{};
  p.H = cfg->num_heads;
  p.D = cfg->head_dim;
  p.r = cfg->ratio;
  p.W = cfg->window;
  p.comp_dtype = cfg->comp_dtype;
  p.win_dtype = cfg->win_dtype;
  p.d_r = cfg->rope_dim;
  return attention_ws_layout(nullptr, p, batch, max_seq_len, max_selected).bytes;
}

int kv_compress_append(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                       const int32_t* d_prev_len, const int32_t* d_cu_new, int32_t max_new,
                       int32_t max_seq_len, const float* d_kv_new, const float* d_logit_new,
                       uint32_t* d_status, void* stream) {
  LayerParams p{};
  const int st = make_params(cfg, cache, batch, max_seq_len, true, &p);
  if (st != CKV_OK) return st;
  if (!d_prev_len || !d_kv_new || !d_logit_new || !d_status || !aligned16(d_kv_new)) return CKV_ERR_INVALID_ARG;
  if (d_cu_new ? max_new < 1 : max_new != 1) return CKV_ERR_INVALID_ARG;
  cudaError_t e = launch_append(p, batch, d_prev_len, d_cu_new, max_new, max_seq_len, d_kv_new,
                                d_logit_new, d_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

int kv_window_replay(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                     const int32_t* d_seq_len, int32_t max_seq_len, const float* d_kv, const float* d_logit,
                     uint32_t* d_status, void* stream) {
  LayerParams p{};
  const int st = make_params(cfg, cache, batch, max_seq_len, true, &p);
  if (st != CKV_OK) return st;
  if (!d_seq_len || !d_status || (p.W > 0 && (!d_kv || !d_logit || !aligned16(d_kv)))) return CKV_ERR_INVALID_ARG;
  cudaError_t e = launch_window_replay(p, batch, d_seq_len, max_seq_len, d_kv, d_logit, d_status,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

int sparse_indexer_topk(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                        const int32_t* d_seq_len, int32_t max_seq_len, const float* d_q,
                        int32_t top_k, int32_t* d_idx, int32_t* d_cnt, float* d_scores,
                        void* d_ws, size_t ws_bytes, uint32_t* d_status, void* stream) {
  LayerParams p{};
  const int st = make_params(cfg, cache, batch, max_seq_len, false, &p);
  if (st != CKV_OK) return st;
  if (batch > 16384) return CKV_ERR_UNSUPPORTED;
  if (!d_seq_len || !d_q || !d_idx || !d_cnt || !d_status || top_k < 1 || !aligned16(d_q) ||
      !aligned16(d_idx) || !aligned16(d_cnt) || (d_scores && !aligned16(d_scores)))
    return CKV_ERR_INVALID_ARG;
  if (!d_ws || !aligned16(d_ws)) return CKV_ERR_WORKSPACE;
  IndexerWs ws = indexer_ws_layout(d_ws, p, batch, max_seq_len);
  if (ws_bytes < ws.bytes) return CKV_ERR_WORKSPACE;
  cudaError_t e = launch_indexer(p, batch, d_seq_len, max_seq_len, d_q, top_k, d_idx, d_cnt, d_scores,
                                 ws, d_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

int compressed_window_attention(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache,
                                int32_t batch, const int32_t* d_seq_len, int32_t max_seq_len,
                                const float* d_q, const int32_t* d_idx, const int32_t* d_cnt,
                                int32_t idx_stride, float* d_out, void* d_ws, size_t ws_bytes,
                                uint32_t* d_status, void* stream) {
  LayerParams p{};
  const int st = make_params(cfg, cache, batch, max_seq_len, false, &p);
  if (st != CKV_OK) return st;
  if (!d_seq_len || !d_q || !d_out || !d_status || !aligned16(d_q) || !aligned16(d_out))
    return CKV_ERR_INVALID_ARG;
  if (d_idx && (!d_cnt || idx_stride < 1)) return CKV_ERR_INVALID_ARG;
  if (!d_ws || !aligned16(d_ws)) return CKV_ERR_WORKSPACE;
  AttnWs ws = attention_ws_layout(d_ws, p, batch, max_seq_len, d_idx ? idx_stride : 0);
  if (ws_bytes < ws.bytes) return CKV_ERR_WORKSPACE;
  cudaError_t e = launch_attention(p, batch, d_seq_len, max_seq_len, d_q, d_idx, d_cnt,
                                   d_idx ? idx_stride : 0, d_out, ws, d_status,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

// Workspace of a fused step: the indexer's (sparse layers) followed by the attention's, each
// 256-byte aligned.
static size_t step_ws_bytes(const LayerParams& p, int batch, int max_seq_len, int top_k, IndexerWs* iw,
                            AttnWs* aw, void* base) {
  size_t off = 0;
  if (top_k > 0) {
    *iw = indexer_ws_layout(base, p, batch, max_seq_len);
    off = align_up(iw->bytes, 256);
  }
  *aw = attention_ws_layout(base ? static_cast<char*>(base) + off : nullptr, p, batch, max_seq_len,
                            top_k > 0 ? top_k : 0);
  return off + aw->bytes;
}

size_t ckv_decode_step_workspace_bytes(const ckv_layer_cfg* cfg, int32_t batch, int32_t max_seq_len,
                                       int32_t top_k) {
  if (check_cfg(cfg) != CKV_OK || batch < 1 || max_seq_len < 1 || top_k < 0) return 0;
  LayerParams p{};
  p.H = cfg->num_heads;
  p.D = cfg->head_dim;
  p.r = cfg->ratio;
  p.W = cfg->window;
  p.comp_dtype = cfg->comp_dtype;
  p.win_dtype = cfg->win_dtype;
  p.d_r = cfg->rope_dim;
  IndexerWs iw{};
  AttnWs aw{};
  return step_ws_bytes(p, batch, max_seq_len, top_k, &iw, &aw, nullptr);
}

int ckv_decode_step(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, int32_t batch,
                    const int32_t* d_seq_len, int32_t max_seq_len, const float* d_q,
                    const float* d_kv_new, const float* d_logit_new, int32_t top_k, int32_t* d_idx,
                    int32_t* d_cnt, float* d_out, void* d_ws, size_t ws_bytes, uint32_t* d_status,
                    void* stream) {
  LayerParams p{};
  const int st = make_params(cfg, cache, batch, max_seq_len, true, &p);
  if (st != CKV_OK) return st;
  if (batch > 16384) return CKV_ERR_UNSUPPORTED;
  if (!d_seq_len || !d_q || !d_kv_new || !d_logit_new || !d_out || !d_status || top_k < 0 ||
      !aligned16(d_q) || !aligned16(d_kv_new) || !aligned16(d_out))
    return CKV_ERR_INVALID_ARG;
  if (top_k > 0 && (!d_idx || !d_cnt || !aligned16(d_idx) || !aligned16(d_cnt))) return CKV_ERR_INVALID_ARG;
  if (!d_ws || !aligned16(d_ws)) return CKV_ERR_WORKSPACE;
  IndexerWs iw{};
  AttnWs aw{};
  if (ws_bytes < step_ws_bytes(p, batch, max_seq_len, top_k, &iw, &aw, d_ws)) return CKV_ERR_WORKSPACE;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // append of the token at seq_len[b] - 1 beside the query pass (q_bar and the cos/sin table of the
  // rotary pairs on sparse layers, the attention's query preparation on dense ones), then selection
  // (sparse layers) and attention
  const QueryPrepOut prep{aw.rope, aw.qimage, aw.qscale};  // the image only for tensor-core layers
  // Sparse layers keep the append and the q-bar pass as two kernels, the pass running beside the
  // append (qbar_kernel, early) and its CTAs leaving room for the next kernel's to become resident.
  // Dense layers with more (request, slice) CTAs than SMs run the append and the attention's query
  // preparation side by side in one front kernel; with fewer, the attention prepares its query
  // itself. Measured (us per step): at batch 8 sparse, 54.2 with two kernels against 57.5 with the
  // front kernel (before the pass ran beside the append); the 64-request mixed step (a sparse and a
  // dense layer) 248.9 against 253.5 with the front kernel for both layers; HCA 128K at batch 32,
  // 49.3 with the front kernel against 56.9 without.
  const bool front = top_k <= 0 && static_cast<int64_t>(batch) * 8 > sm_count();
  cudaError_t e = cudaSuccess;
  if (front) {
    e = launch_step_front(p, batch, d_seq_len, max_seq_len, d_kv_new, d_logit_new, d_q, prep, aw, d_status, s);
  } else {
    e = launch_append(p, batch, d_seq_len, nullptr, 1, max_seq_len, d_kv_new, d_logit_new, d_status, s, -1);
  }
  if (e != cudaSuccess) return CKV_ERR_CUDA;
  if (top_k > 0) {
    e = launch_indexer(p, batch, d_seq_len, max_seq_len, d_q, top_k, d_idx, d_cnt, nullptr, iw, d_status, s,
                       prep, true);
    if (e != cudaSuccess) return CKV_ERR_CUDA;
  }
  // the cos/sin table is written when the front kernel ran or the indexer's q-bar pass wrote it
  // (the tensor-core attention computes it itself either way); the step's first kernel waited for
  // the producers of q and seq_len, so the attention may read them early
  e = launch_attention(p, batch, d_seq_len, max_seq_len, d_q, top_k > 0 ? d_idx : nullptr,
                       top_k > 0 ? d_cnt : nullptr, top_k > 0 ? top_k : 0, d_out, aw, d_status, s,
                       front || top_k > 0, true);
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

int kv_index_append(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, const ckv_index_cfg* icfg,
                    const ckv_index_cache* icache, int32_t batch, const int32_t* d_prev_len,
                    const int32_t* d_cu_new, int32_t max_new, int32_t max_seq_len, const float* d_k_new,
                    const float* d_logit_new, uint32_t* d_status, void* stream) {
  LayerParams p{};
  int st = make_params(cfg, cache, batch, max_seq_len, false, &p);
  if (st != CKV_OK) return st;
  IndexParams ip{};
  st = make_index_params(icfg, icache, true, &ip);
  if (st != CKV_OK) return st;
  if (!d_prev_len || !d_k_new || !d_logit_new || !d_status || !aligned16(d_k_new)) return CKV_ERR_INVALID_ARG;
  if (d_cu_new ? max_new < 1 : max_new != 1) return CKV_ERR_INVALID_ARG;
  cudaError_t e = launch_index_append(p, ip, batch, d_prev_len, d_cu_new, max_new, max_seq_len, d_k_new,
                                      d_logit_new, d_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

size_t ckv_mh_indexer_workspace_bytes(const ckv_layer_cfg* cfg, const ckv_index_cfg* icfg, int32_t batch,
                                      int32_t max_seq_len, int32_t top_k) {
  if (check_cfg(cfg) != CKV_OK || !icfg || batch < 1 || max_seq_len < 1 || top_k < 1) return 0;
  const int H = icfg->index_heads, d = icfg->index_dim;
  if (H < 16 || H > 128 || H % 16 != 0 || (d != 128 && d != 256)) return 0;
  LayerParams p{};
  p.D = cfg->head_dim;
  p.r = cfg->ratio;
  IndexParams ip{};
  ip.heads = H;
  ip.dim = d;
  IndexerWs iw{};
  return mh_ws_bytes(p, ip, batch, max_seq_len, &iw, nullptr, nullptr);
}

int sparse_mh_indexer_topk(const ckv_layer_cfg* cfg, const ckv_layer_cache* cache, const ckv_index_cfg* icfg,
                           const ckv_index_cache* icache, int32_t batch, const int32_t* d_seq_len,
                           int32_t max_seq_len, const float* d_q_index, const float* d_weights, int32_t top_k,
                           int32_t* d_idx, int32_t* d_cnt, float* d_scores, void* d_ws, size_t ws_bytes,
                           uint32_t* d_status, void* stream) {
  LayerParams p{};
  int st = make_params(cfg, cache, batch, max_seq_len, false, &p);
  if (st != CKV_OK) return st;
  IndexParams ip{};
  st = make_index_params(icfg, icache, false, &ip);
  if (st != CKV_OK) return st;
  if (batch > 2048 || p.r > 4) return CKV_ERR_UNSUPPORTED;  // 64-entry runs within one pool block
  if (!d_seq_len || !d_q_index || !d_weights || !d_idx || !d_cnt || !d_status || top_k < 1 ||
      !aligned16(d_q_index) || !aligned16(d_idx) || !aligned16(d_cnt) || (d_scores && !aligned16(d_scores)))
    return CKV_ERR_INVALID_ARG;
  if (!d_ws || !aligned16(d_ws)) return CKV_ERR_WORKSPACE;
  IndexerWs iw{};
  uint8_t* qimage = nullptr;
  if (ws_bytes < mh_ws_bytes(p, ip, batch, max_seq_len, &iw, &qimage, d_ws)) return CKV_ERR_WORKSPACE;
  cudaError_t e = launch_mh_indexer(p, ip, batch, d_seq_len, max_seq_len, d_q_index, d_weights, top_k, d_idx,
                                    d_cnt, d_scores, iw, qimage, d_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

const char* ckv_status_str(int status) {
  switch (status) {
    case CKV_OK: return "ok";
    case CKV_ERR_INVALID_ARG: return "invalid argument";
    case CKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case CKV_ERR_OUT_OF_BLOCKS: return "block pool exhausted";
    case CKV_ERR_WORKSPACE: return "workspace too small";
    case CKV_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

uint64_t ckv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ckv_debug_force_timeout(int32_t request) {
  if (request < -1) return CKV_ERR_INVALID_ARG;
  return attention_force_timeout(request) == cudaSuccess ? CKV_OK : CKV_ERR_CUDA;
}

int ckv_profile_events(int which, void* ev_begin, void* ev_end) {
  if (which != CKV_PROF_SCORE && which != CKV_PROF_ATTENTION) return CKV_ERR_INVALID_ARG;
  if ((ev_begin == nullptr) != (ev_end == nullptr)) return CKV_ERR_INVALID_ARG;
  g_prof[which][0] = static_cast<cudaEvent_t>(ev_begin);
  g_prof[which][1] = static_cast<cudaEvent_t>(ev_end);
  return CKV_OK;
}

}  // extern "C"

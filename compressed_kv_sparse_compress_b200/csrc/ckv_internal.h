// Internal launch interface between the C ABI layer (capi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ckv_common.cuh"

namespace ckv {

// Bookkeeping of kernel launches (ckv_launch_count).
void note_launch();
// Multiprocessor count of the current device (cached per device).
int sm_count();
// Opt a kernel into more than 48 KB of dynamic shared memory on the current device, once.
cudaError_t allow_smem(const void* kernel, int bytes);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launches a library kernel with programmatic stream serialization (see griddep_wait) and counts
// it; returns the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Diagnostic events around one kernel (ckv_profile_events); no-ops when unset.
enum ProfPoint { kProfScore = 0, kProfAttention = 1 };
void prof_begin(ProfPoint which, cudaStream_t stream);
void prof_end(ProfPoint which, cudaStream_t stream);

// ---------------------------------------------------------------------------- append
// prev_offset is added to every prev_len[b] (-1 when prev_len holds the lengths after the append)
cudaError_t launch_append(const LayerParams& p, int batch, const int32_t* prev_len,
                          const int32_t* cu_new, int max_new, int max_seq_len, const float* kv_new,
                          const float* logit_new, uint32_t* status, cudaStream_t stream,
                          int prev_offset = 0);

// SWA bounded replay: rewrites the last min(W, L) window rows and the unfinished group's ring slots
// of every request from kv [batch][W][D] / logit [batch][W] (row i = position L - n_w + i).
cudaError_t launch_window_replay(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                                 const float* kv, const float* logit, uint32_t* status, cudaStream_t stream);

// ---------------------------------------------------------------------------- indexer
constexpr int kHistBins = 2048;  // first radix digit: the top 11 bits of the order key

// Carve-up of the indexer workspace.
struct IndexerWs {
  float* qbar;        // [B][D]   scaled, rotated, head-averaged query
  int32_t* n_c;       // [B]      candidate count (0 for an invalid length)
  uint32_t* hist;     // [B][2048]
  uint32_t* cand_cnt; // [B]
  uint32_t* bitmap;   // [B][stride/32]
  uint2* cand;        // [B][stride]  (order key, index) of boundary-bin candidates
  float* scores;      // [B][stride]  when the caller passes no score buffer
  size_t bytes;
};
int64_t score_stride(int ratio, int max_seq_len);
IndexerWs indexer_ws_layout(void* base, const LayerParams& p, int batch, int max_seq_len);

// Output of the query pass that the attention of the same layer and step can take over: the
// cos/sin table of the rotary pairs at the query position (null: not written).
struct QueryPrepOut {
  double* rope;        // [B][d_r/2 + 1][2] cos, sin of the rotary pairs at the query position
  uint8_t* qimage;     // [B][128 KB] the tensor-core attention's query operand (qimage.cuh), or null
  float* qscale;       // [B][64] its per-head power-of-two scales
};
// early_qbar: the q_bar pass follows the fused step's append, which has waited for the producers
// of q and the lengths, and may run beside it (qbar_kernel)
cudaError_t launch_indexer(const LayerParams& p, int batch, const int32_t* seq_len,
                           int max_seq_len, const float* q, int top_k, int32_t* idx, int32_t* cnt,
                           float* scores, const IndexerWs& ws, uint32_t* status,
                           cudaStream_t stream, QueryPrepOut prep = {nullptr}, bool early_qbar = false);

// Top-k of the scores a score pass wrote, with the candidate counts, the reset selection state
// and the first-digit histogram in ws (the kernels after the score pass).
cudaError_t launch_topk(const LayerParams& p, int batch, int max_seq_len, int top_k, const float* scores,
                        int64_t stride, const IndexerWs& ws, int32_t* idx, int32_t* cnt, cudaStream_t stream);

// ---------------------------------------------------------------------------- multi-head indexer
// The index plane of a layer: FP8 index entries in the rows of the compressed pool, and the
// index-key compressor's own residue ring.
struct IndexParams {
  int heads;           // H_I: a multiple of 16, 16 .. 128
  int dim;             // d_I: 128 or 256
  uint8_t* codes;      // [pool rows][d_I] e4m3
  float* scales;       // [pool rows] fp32
  float* res_k;        // [B][r][d_I] fp32
  float* res_logit;    // [B][r] fp32
};
// bytes of the fp16 query images of a batch (the head of the multi-head indexer's workspace)
size_t mh_image_bytes(const IndexParams& ip, int batch);
cudaError_t launch_index_append(const LayerParams& p, const IndexParams& ip, int batch, const int32_t* prev_len,
                                const int32_t* cu_new, int max_new, int max_seq_len, const float* k_new,
                                const float* logit_new, uint32_t* status, cudaStream_t stream);
cudaError_t launch_mh_indexer(const LayerParams& p, const IndexParams& ip, int batch, const int32_t* seq_len,
                              int max_seq_len, const float* q_index, const float* weights, int top_k,
                              int32_t* idx, int32_t* cnt, float* scores, const IndexerWs& ws,
                              uint8_t* qimage, uint32_t* status, cudaStream_t stream);

// ---------------------------------------------------------------------------- attention
struct AttnWs {
  float* part_o;     // [B][S][H][D]   un-normalised partial outputs (CUDA-core path)
  uint16_t* part_h;  // [B][S][D][H]   tensor-core path: fp16 partial outputs, rows of 64 heads per
                     //                dim, head h divided by part_sc (same memory as part_o)
  float* part_sc;    // [B][S][H]      tensor-core path: power-of-two scale of each partial
  bool half_parts;   // which of the two forms the splits write (the tensor-core form)
  float* part_ml;    // [B][S][H][2]   running max and sum of each split (max in nats on the
                     //                CUDA-core path, in base 2 on the tensor-core path)
  double* rope;      // [B][d_r/2][2]  cos, sin of each rotary pair at the query position
  uint8_t* qimage;   // [B][128 KB]    tensor-core path: the query operand, written by the step's
                     //                query pass (qimage.cuh); null for other layers
  float* qscale;     // [B][64]        its per-head scales
  int splits;        // S: splits per request
  int keys_per_split;
  size_t bytes;
};
bool attention_tc_supported(const LayerParams& p);  // the tensor-core path serves this layer
// Failure-path hook of the tensor-core attention (request index, -1: off); see ckv_debug_force_timeout.
cudaError_t attention_force_timeout(int request);
AttnWs attention_ws_layout(void* base, const LayerParams& p, int batch, int max_seq_len,
                           int max_selected);

// prep_done: the cos/sin table is already in ws (written by the indexer's query pass or the front
// kernel of the same step), so the CUDA-core path launches no prep kernel (the tensor-core kernel
// computes the table itself and writes it when it is not there). early: the call is part of a
// fused decode step whose first kernel has already waited for the producers of q and seq_len, so
// the tensor-core kernel may read them before waiting for its predecessor.
cudaError_t launch_attention(const LayerParams& p, int batch, const int32_t* seq_len,
                             int max_seq_len, const float* q, const int32_t* idx,
                             const int32_t* cnt, int idx_stride, float* out, const AttnWs& ws,
                             uint32_t* status, cudaStream_t stream, bool prep_done = false,
                             bool early = false);

// ---------------------------------------------------------------------------- fused step
// First kernel of ckv_decode_step on a dense layer: the append of the new token (at seq_len[b] - 1)
// side by side with the attention's query preparation (the cos/sin table and the query image).
cudaError_t launch_step_front(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                              const float* kv_new, const float* logit_new, const float* q,
                              QueryPrepOut prep, const AttnWs& aws, uint32_t* status, cudaStream_t stream);

}  // namespace ckv

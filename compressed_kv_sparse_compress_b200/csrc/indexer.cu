// Step 2 of the decode path: the sparse MQA indexer and top-k selection.
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": attention is restricted to the top-k compressed tokens;
// aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section "Vykon neprinesl jeden kernel": the
// "Sparse MQA logits" kernel scores only the candidate positions. Reading: the score of entry j is
// the head-average of the MQA logits, s_j = sm_scale/H * sum_h q~_h . k_j. All heads share k_j,
// so the sum over heads collapses into one query q_bar = sm_scale/H * sum_h q~_h, computed once
// per request, and scoring streams the compressed cache once with one fp32 dot per entry.
//
// Kernels, in stream order:
//   qbar_kernel     per (request, slice of dims): q_bar, candidate count, reset of the
//                   selection state
//   score_kernel    persistent, HBM-bound: streams every candidate entry with 16-byte
//                   non-allocating loads, writes its fp32 score, and counts the top 11 bits of
//                   its order key into a per-request histogram (first radix digit)
//   topk_small      per request, when every request has at most 16384 candidates: the whole
//                   selection in one CTA of 1024 threads with the scores in registers
//   topk_mark       per (request, 8192 scores): marks scores above the boundary bin in a
//                   bitmap and appends boundary-bin candidates to a list
//   topk_finish     per request: resolves the boundary bin with two more radix digits (and the
//                   lower-index tie rule), then compacts the bitmap into ascending indices.

#include "ckv_internal.h"
#include "query_prep.cuh"

namespace ckv {

int64_t score_stride(int ratio, int max_seq_len) {
  const int64_t n = static_cast<int64_t>(max_seq_len) / ratio;
  return (n + 63) / 64 * 64;
}

IndexerWs indexer_ws_layout(void* base, const LayerParams& p, int batch, int max_seq_len) {
  IndexerWs w{};
  const int64_t stride = score_stride(p.r, max_seq_len);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return static_cast<char*>(base) + o;
  };
  const bool have = base != nullptr;
  char* q = take(sizeof(float) * batch * p.D);
  char* nc = take(sizeof(int32_t) * batch);
  char* h = take(sizeof(uint32_t) * batch * kHistBins);
  char* cc = take(sizeof(uint32_t) * batch);
  char* bm = take(sizeof(uint32_t) * batch * (stride / 32));
  char* cd = take(sizeof(uint2) * batch * stride);
  char* sc = take(sizeof(float) * batch * stride);
  if (have) {
    w.qbar = reinterpret_cast<float*>(q);
    w.n_c = reinterpret_cast<int32_t*>(nc);
    w.hist = reinterpret_cast<uint32_t*>(h);
    w.cand_cnt = reinterpret_cast<uint32_t*>(cc);
    w.bitmap = reinterpret_cast<uint32_t*>(bm);
    w.cand = reinterpret_cast<uint2*>(cd);
    w.scores = reinterpret_cast<float*>(sc);
  }
  w.bytes = off;
  return w;
}

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMarkChunk = 4 * kThreads;  // scores per mark CTA
constexpr int kFinishThreads = 1024;
static_assert(kHistBins == 8 * kThreads && kHistBins == 2 * kFinishThreads, "first-digit bins per thread");

// ---------------------------------------------------------------------------- block scans

// inclusive scan of one value per thread across the block (blockDim.x multiple of 32)
template <typename T>
__device__ T block_inclusive_scan(T v, T* sh /* >= 32 */, T* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  __syncthreads();
  if (lane == 31) sh[w] = v;
  __syncthreads();
  if (w == 0) {
    T s = lane < nw ? sh[lane] : T(0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    if (lane < nw) sh[lane] = s;
  }
  __syncthreads();
  if (w > 0) v += sh[w - 1];
  if (total) *total = sh[nw - 1];
  __syncthreads();
  return v;
}

// Boundary of a histogram h[nbins] (shared or global) for selecting `need` items, scanning from
// the top bin down (descending) or from bin 0 up: the bin where the running count reaches need,
// and the count strictly before it in scan order. Result in out[0] (bin), out[1] (before).
__device__ void find_boundary(const uint32_t* h, int nbins, uint32_t need, bool descending,
                              uint32_t* sh /* >= 32 */, uint32_t* out) {
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  const int g0 = threadIdx.x * per;
  uint32_t s = 0;
  for (int i = 0; i < per; ++i) {
    const int k = g0 + i;
    if (k < nbins) s += h[descending ? nbins - 1 - k : k];
  }
  const uint32_t incl = block_inclusive_scan<uint32_t>(s, sh, nullptr);
  const uint32_t excl = incl - s;
  if (excl < need && incl >= need) {
    uint32_t cum = excl;
    for (int i = 0; i < per; ++i) {
      const int k = g0 + i;
      if (k >= nbins) break;
      const int bin = descending ? nbins - 1 - k : k;
      if (cum + h[bin] >= need) {
        out[0] = bin;
        out[1] = cum;
        break;
      }
      cum += h[bin];
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------- q_bar

// q_bar of one slice of one request: qbar_slice (query_prep.cuh).
// early: the call is part of a fused decode step whose first kernel (the append, which this pass
// follows) has already waited for the producers of q and the lengths, and nothing this pass reads
// or writes is touched by the append: the pass runs beside the append and waits for it only before
// it exits, so that its completion still implies the append's.
__global__ void __launch_bounds__(kQbarThreads) qbar_kernel(LayerParams p, const int32_t* seq_len,
                                                            int max_seq_len, const float* q,
                                                            IndexerWs ws, uint32_t* status,
                                                            QueryPrepOut prep, bool early) {
  if (!early) griddep_wait();
  griddep_launch();
  __shared__ double part[kQbarThreads][2];
  qbar_slice(p, seq_len, max_seq_len, q, ws, status, prep, blockIdx.x, blockIdx.y, threadIdx.x, part, 0);
  if (prep.qimage) {  // the attention's query image, heads 8 x .. 8 x + 7 (slices = 8)
    __shared__ double rope_tmp[2 * kQiMaxRopePairs];
    qimage_part(p, seq_len, max_seq_len, q, prep, blockIdx.x, blockIdx.y, threadIdx.x, rope_tmp, 0);
  }
  if (early) griddep_wait();
}

// ---------------------------------------------------------------------------- scoring

template <int DT>
struct VecFmt;  // elements decoded from one 16-byte vector of codes
template <> struct VecFmt<CKV_F32> { static constexpr int kElems = 4; };
template <> struct VecFmt<CKV_BF16> { static constexpr int kElems = 8; };
template <> struct VecFmt<CKV_NVFP4> { static constexpr int kElems = 32; };

// dot of one 16-byte code vector with the matching q_bar elements held in registers
template <int DT>
__device__ __forceinline__ float vec_dot(const float* qv, uint4 raw, uint32_t sc16) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  float acc = 0.f;
  if constexpr (DT == CKV_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc = fmaf(qv[i], __uint_as_float(w[i]), acc);
  } else if constexpr (DT == CKV_BF16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(qv[2 * i], __uint_as_float(w[i] << 16), acc);
      acc = fmaf(qv[2 * i + 1], __uint_as_float(w[i] & 0xffff0000u), acc);
    }
  } else {  // NVFP4: two 16-element blocks, each with its e4m3 scale
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t word = w[2 * blk + i];
#pragma unroll
        for (int by = 0; by < 4; ++by) {
          const float2 v = __half22float2(e2m1x2_to_half2(static_cast<uint8_t>(word >> (8 * by))));
          const int e = 16 * blk + 8 * i + 2 * by;
          part = fmaf(qv[e], v.x, part);
          part = fmaf(qv[e + 1], v.y, part);
        }
      }
      acc = fmaf(part, e4m3_to_f32(static_cast<uint8_t>(sc16 >> (8 * blk))), acc);
    }
  }
  return acc;
}

// NV: 16-byte code vectors per entry (a power of two); U: entries per lane group per chunk
// Before its wait for the previous kernel (the query pass) the kernel takes the candidate counts
// from the lengths (the query pass derives the same ones for the selection), partitions the
// chunks, resolves each warp's first chunk through the block tables and prefetches its entries into
// L2: the lengths and the block tables come from before the step and no kernel of the step writes
// them, while the entries (the step's append may complete one) are loaded only after the wait; a
// prefetch moves no data into registers, so a line the append writes later is read afresh.
template <int DT, int NV, int U>
__global__ void __launch_bounds__(kThreads, 2) score_kernel(LayerParams p, int batch, const int32_t* seq_len,
                                                         int max_seq_len, IndexerWs ws, float* scores,
                                                         int64_t stride, uint32_t* status) {
  constexpr int LPE = NV < 32 ? NV : 32;  // lanes per entry
  constexpr int VPL = NV / LPE;           // vectors per lane per entry
  constexpr int EPP = 32 / LPE;           // entries per warp pass
  constexpr int CH = U * EPP;             // entries per warp chunk
  constexpr int EPV = VecFmt<DT>::kElems;
  static_assert(U <= LPE, "one writer lane per entry of a pass");

  extern __shared__ int32_t chunk_prefix[];  // [batch + 1], then the candidate counts [batch]
  int32_t* n_c = chunk_prefix + batch + 1;
  __shared__ int32_t scan_sh[32];
  // chunks per request, exclusive prefix over the batch (one warp when the batch fits it)
  auto count = [&](int bb) {
    const int32_t L = __ldcg(seq_len + bb);
    return L >= 1 && L <= max_seq_len ? L / p.r : 0;
  };
  if (batch <= 32) {
    if (threadIdx.x < 32) {
      const int bb = threadIdx.x;
      const int32_t n = bb < batch ? count(bb) : 0;
      const int32_t s = (n + CH - 1) / CH;
      int32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (bb >= o) incl += t;
      }
      if (bb < batch) {
        n_c[bb] = n;
        chunk_prefix[bb] = incl - s;
      }
      if (bb == 31) chunk_prefix[batch] = incl;
    }
    __syncthreads();
  } else {
    const int per = (batch + blockDim.x - 1) / blockDim.x;
    int32_t s = 0;
    for (int i = 0; i < per; ++i) {
      const int bb = threadIdx.x * per + i;
      if (bb < batch) {
        const int32_t n = count(bb);
        n_c[bb] = n;
        s += (n + CH - 1) / CH;
      }
    }
    int32_t total;
    const int32_t incl = block_inclusive_scan<int32_t>(s, scan_sh, &total);
    int32_t run = incl - s;
    for (int i = 0; i < per; ++i) {
      const int bb = threadIdx.x * per + i;
      if (bb < batch) {
        chunk_prefix[bb] = run;
        run += (n_c[bb] + CH - 1) / CH;
      }
    }
    if (threadIdx.x == 0) chunk_prefix[batch] = total;
    __syncthreads();
  }
  const int64_t total = chunk_prefix[batch];
  const int64_t c_lo = total * blockIdx.x / gridDim.x;
  const int64_t c_hi = total * (blockIdx.x + 1) / gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPE, slot = lane / LPE;
  const int sc_bytes = p.D / 16;

  // A chunk's request, first entry and pool rows; resolving the next chunk (its block-table
  // loads) overlaps the data loads of the current one.
  struct Chunk {
    int b;
    int N;
    int64_t e_base;
    int64_t row[U];
  };
  auto resolve = [&](int64_t ch) {
    Chunk c;
    int lo = 0, hi = batch;   // last b with chunk_prefix[b] <= ch
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (chunk_prefix[mid] <= ch) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.N = n_c[lo];
    c.e_base = (ch - chunk_prefix[lo]) * CH;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t e = c.e_base + u * EPP + slot;
      c.row[u] = e < c.N ? comp_row(p, lo, e, status) : -1;
    }
    return c;
  };

  int cur_b = -1;
  float qreg[VPL][EPV];
  Chunk cur;
  if (c_lo + warp < c_hi) {
    cur = resolve(c_lo + warp);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = cur.row[u];
      if (row < 0) continue;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int v = sub + LPE * k;
        if ((v & 7) == 0) prefetch_l2(p.comp_codes + row * p.comp_row_bytes + v * 16);  // one per 128-byte line
      }
      if (DT == CKV_NVFP4 && sub == 0) prefetch_l2(p.comp_scales + row * sc_bytes);
    }
  }
  griddep_wait();
  griddep_launch();
  for (int64_t ch = c_lo + warp; ch < c_hi; ch += kWarps) {
    const int b = cur.b;
    if (b != cur_b) {
      const float* qb = ws.qbar + static_cast<int64_t>(b) * p.D;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
#pragma unroll
        for (int e = 0; e < EPV; e += 4) {
          const float4 v = *reinterpret_cast<const float4*>(qb + (sub + LPE * k) * EPV + e);
          qreg[k][e] = v.x; qreg[k][e + 1] = v.y; qreg[k][e + 2] = v.z; qreg[k][e + 3] = v.w;
        }
      }
      cur_b = b;
    }
    const int N = cur.N;
    const int64_t e_base = cur.e_base;
    uint4 raw[U][VPL];
    uint32_t sc[U][VPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = cur.row[u];
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int v = sub + LPE * k;
        if (row >= 0) {
          raw[u][k] = ldg_stream(p.comp_codes + row * p.comp_row_bytes + v * 16);
          sc[u][k] = (DT == CKV_NVFP4)
              ? static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p.comp_scales + row * sc_bytes + 2 * v))
              : 0u;
        } else {
          raw[u][k] = make_uint4(0, 0, 0, 0);
          sc[u][k] = 0u;
        }
      }
    }
    if (ch + kWarps < c_hi) cur = resolve(ch + kWarps);
    float acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      acc[u] = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k) acc[u] += vec_dot<DT>(qreg[k], raw[u][k], sc[u][k]);
#pragma unroll
      for (int o = LPE / 2; o > 0; o >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
    }
    // lane (slot, sub = u) writes the score of entry (pass u, slot) and counts its digit
    float mine = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (u == sub) mine = acc[u];
    const int64_t e = e_base + static_cast<int64_t>(sub) * EPP + slot;
    const bool writer = sub < U && e < N;
    uint32_t bin = 0xffffffffu - lane;
    if (writer) {
      scores[static_cast<int64_t>(b) * stride + e] = mine;
      bin = f32_order_key(mine) >> 21;
    }
    const uint32_t same = __match_any_sync(0xffffffffu, bin);
    if (writer && lane == __ffs(same) - 1)
      atomicAdd(ws.hist + static_cast<int64_t>(b) * kHistBins + bin, static_cast<uint32_t>(__popc(same)));
  }
}


// ---------------------------------------------------------------------------- selection

// Boundary of a block-distributed histogram (thread t owns bins [t * NBL, (t + 1) * NBL), NW warps)
// for selecting `need` items from the top bin down: returns (bin, items in the bins above it) to
// every thread. Two barriers.
template <int NBL, int NW>
__device__ __forceinline__ uint2 small_boundary(const uint32_t (&c)[NBL], uint32_t need, uint32_t* wsum,
                                                uint2* bnd) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < NBL; ++i) s += c[i];
  uint32_t suf = s;  // items in this lane's bins and those of the lanes above it
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += t;
  }
  if (lane == 0) wsum[w] = suf;
  __syncthreads();
  uint32_t above = (lane > w && lane < NW) ? wsum[lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  above += suf - s;  // items in all bins above this thread's bins
  if (above < need && above + s >= need) {
    uint32_t cum = above;
#pragma unroll
    for (int i = NBL - 1; i >= 0; --i) {
      if (cum + c[i] >= need) {
        *bnd = make_uint2(static_cast<uint32_t>(threadIdx.x * NBL + i), cum);
        break;
      }
      cum += c[i];
    }
  }
  __syncthreads();
  return *bnd;
}


// One CTA per 1024 scores of a request: each lane classifies 4 consecutive scores against the
// boundary bin of the first digit; the bitmap word of 32 scores is assembled from 8 lanes.
__global__ void __launch_bounds__(kThreads) topk_mark_kernel(const float* scores, int64_t stride,
                                                             int top_k, IndexerWs ws) {
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.y;
  const int64_t N = ws.n_c[b];
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kMarkChunk;
  if (j0 >= N) return;
  uint32_t* bm = ws.bitmap + static_cast<int64_t>(b) * (stride / 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j = j0 + 4 * static_cast<int64_t>(threadIdx.x);  // this lane's 4 scores
  const int64_t w0 = (j0 >> 5) + 4 * warp;                        // this warp's 4 words
  if (N <= top_k) {  // every candidate is selected
    if (threadIdx.x < kMarkChunk / 32) {
      const int64_t w = (j0 >> 5) + threadIdx.x;
      if (w * 32 < N) {
        const int64_t n = min(static_cast<int64_t>(32), N - w * 32);
        bm[w] = n == 32 ? 0xffffffffu : ((1u << n) - 1u);
      }
    }
    return;
  }
  // the lane's scores (stride is a multiple of 64 floats, so the float4 is in bounds)
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (j < N) v = __ldcg(reinterpret_cast<const float4*>(scores + static_cast<int64_t>(b) * stride + j));
  // first-digit boundary from the score kernel's histogram, eight bins per thread
  __shared__ uint32_t sh[32];
  __shared__ uint2 bnd;
  const uint4* hg = reinterpret_cast<const uint4*>(ws.hist + static_cast<int64_t>(b) * kHistBins) + 2 * threadIdx.x;
  const uint4 ha = __ldcg(hg), hb = __ldcg(hg + 1);
  const uint32_t c8[8] = {ha.x, ha.y, ha.z, ha.w, hb.x, hb.y, hb.z, hb.w};
  const uint32_t b1 = small_boundary<8, kWarps>(c8, static_cast<uint32_t>(top_k), sh, &bnd).x;
  const float vals[4] = {v.x, v.y, v.z, v.w};
  uint32_t keys[4];
  uint32_t sel = 0, cnd = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    keys[e] = f32_order_key(vals[e]);
    const bool in = j + e < N;
    const uint32_t bin = keys[e] >> 21;
    if (in && bin > b1) sel |= 1u << e;
    if (in && bin == b1) cnd |= 1u << e;
  }
  // bitmap: lanes 8k..8k+7 hold the 32 bits of word k of the warp
  uint32_t word = sel << (4 * (lane & 7));
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  word |= __shfl_xor_sync(0xffffffffu, word, 4);
  if ((lane & 7) == 0 && (w0 + (lane >> 3)) * 32 < N) bm[w0 + (lane >> 3)] = word;
  // boundary-bin candidates: one atomic per CTA (the request's counter is shared by all its
  // CTAs), then each lane writes its own
  __shared__ uint32_t wtot[kWarps + 1];
  const int mine = __popc(cnd);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = static_cast<uint32_t>(incl);
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t t = wtot[w];
      wtot[w] = run;
      run += t;
    }
    wtot[kWarps] = run ? atomicAdd(ws.cand_cnt + b, run) : 0u;
  }
  __syncthreads();
  if (mine) {
    uint2* cand = ws.cand + static_cast<int64_t>(b) * stride;
    uint32_t pos = wtot[kWarps] + wtot[warp] + static_cast<uint32_t>(incl - mine);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (cnd & (1u << e)) cand[pos++] = make_uint2(keys[e], static_cast<uint32_t>(j + e));
  }
}

// Radix digit pass over the candidate list: histogram of digit(key) among items matching
// `prefix` on the bits above `shift + width`, then the boundary for `need` from the top.
struct DigitSel {
  uint32_t bin, before;
};

template <bool kByIndex>
__device__ DigitSel candidate_digit_pass(const uint2* cand, uint32_t m, uint32_t* h, int shift,
                                         int width, uint32_t match_mask, uint32_t match_val,
                                         uint32_t eq_key, uint32_t need, uint32_t* sh) {
  const int nbins = 1 << width;
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < m; i += blockDim.x) {
    const uint2 c = cand[i];
    // by key: digits of the key, descending; by index: among key == eq_key, digits of the
    // index, ascending
    if (kByIndex && c.x != eq_key) continue;
    const uint32_t v = kByIndex ? c.y : c.x;
    if ((v & match_mask) != match_val) continue;
    atomicAdd(h + ((v >> shift) & (nbins - 1)), 1u);
  }
  __syncthreads();
  __shared__ uint2 sel;
  if (!kByIndex && nbins == 2 * kFinishThreads) {  // descending, 2 bins per thread
    const uint2 hv = reinterpret_cast<const uint2*>(h)[threadIdx.x];
    const uint32_t c2[2] = {hv.x, hv.y};
    const uint2 r = small_boundary<2, kFinishThreads / 32>(c2, need, sh, &sel);
    return DigitSel{r.x, r.y};
  }
  if (!kByIndex && nbins == kFinishThreads) {  // descending, 1 bin per thread
    const uint32_t c1[1] = {h[threadIdx.x]};
    const uint2 r = small_boundary<1, kFinishThreads / 32>(c1, need, sh, &sel);
    return DigitSel{r.x, r.y};
  }
  __shared__ uint32_t out[2];
  find_boundary(h, nbins, need, !kByIndex, sh, out);
  return DigitSel{out[0], out[1]};
}

// boundary-bin candidates that the finish kernel keeps in shared memory for its digit passes (the
// first digit's boundary bin holds about 1.5% of a request's candidates at 262144 of them)
constexpr uint32_t kFinishCandSmem = 16384;

__global__ void __launch_bounds__(kFinishThreads) topk_finish_kernel(int top_k, IndexerWs ws,
                                                                     int64_t stride, int32_t* idx,
                                                                     int32_t* cnt) {
  griddep_wait();
  griddep_launch();
  __shared__ uint32_t h[kHistBins];
  extern __shared__ uint2 cand_s[];  // up to kFinishCandSmem boundary-bin candidates
  __shared__ uint32_t sh[32];
  __shared__ uint2 bnd;
  const int b = blockIdx.x;
  const int64_t N = ws.n_c[b];
  const int64_t k_eff = min(static_cast<int64_t>(top_k), N);
  uint32_t* bm = ws.bitmap + static_cast<int64_t>(b) * (stride / 32);
  if (N > top_k) {
    // first digit from the score kernel's histogram, two bins per thread
    const uint2 hv = __ldcg(reinterpret_cast<const uint2*>(ws.hist + static_cast<int64_t>(b) * kHistBins) + threadIdx.x);
    const uint32_t c1[2] = {hv.x, hv.y};
    const uint2 r1 = small_boundary<2, kFinishThreads / 32>(c1, static_cast<uint32_t>(top_k), sh, &bnd);
    const uint32_t b1 = r1.x;
    uint32_t need = static_cast<uint32_t>(k_eff) - r1.y;
    const uint32_t m = ws.cand_cnt[b];
    const uint2* cand = ws.cand + static_cast<int64_t>(b) * stride;
    if (m <= kFinishCandSmem) {
      // four loads in flight per thread
      for (uint32_t i0 = threadIdx.x; i0 < m; i0 += 4 * blockDim.x) {
        uint2 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i0 + u * blockDim.x < m) v[u] = __ldcg(cand + i0 + u * blockDim.x);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i0 + u * blockDim.x < m) cand_s[i0 + u * blockDim.x] = v[u];
      }
      __syncthreads();
      cand = cand_s;
    }
    // digits 2 and 3 of the key: bits [20:10] and [9:0]
    const DigitSel dA = candidate_digit_pass<false>(cand, m, h, 10, 11, 0xffe00000u, b1 << 21, 0, need, sh);
    need -= dA.before;
    const uint32_t pA = (b1 << 21) | (dA.bin << 10);
    uint32_t T, n_eq;
    if (h[dA.bin] == need) {
      // every candidate of the boundary bin is taken: select key >= the bin's lower edge pA
      // (key == pA with any index)
      T = pA;
      n_eq = 0;
      need = 0;
    } else {
      __syncthreads();  // every thread has read h before the next pass clears it
      const DigitSel dB = candidate_digit_pass<false>(cand, m, h, 0, 10, 0xfffffc00u, pA, 0, need, sh);
      need -= dB.before;
      T = pA | dB.bin;
      n_eq = h[dB.bin];
    }
    // among key == T keep the `need` lowest indices: index threshold by three ascending digits
    uint32_t idx_thr = 0xffffffffu;
    if (need < n_eq) {
      const DigitSel i1 = candidate_digit_pass<true>(cand, m, h, 21, 11, 0u, 0u, T, need, sh);
      uint32_t nd = need - i1.before;
      const uint32_t q1 = i1.bin << 21;
      const DigitSel i2 = candidate_digit_pass<true>(cand, m, h, 10, 11, 0xffe00000u, q1, T, nd, sh);
      nd -= i2.before;
      const uint32_t q2 = q1 | (i2.bin << 10);
      const DigitSel i3 = candidate_digit_pass<true>(cand, m, h, 0, 10, 0xfffffc00u, q2, T, nd, sh);
      idx_thr = q2 | i3.bin;
    }
    for (uint32_t i = threadIdx.x; i < m; i += blockDim.x) {
      const uint2 c = cand[i];
      if (c.x > T || (c.x == T && c.y <= idx_thr)) atomicOr(bm + (c.y >> 5), 1u << (c.y & 31));
    }
    __threadfence_block();
    __syncthreads();
  }
  // compaction of the bitmap into ascending indices: thread t takes the words [w0, w1); when they
  // are at most kRegWords, all their loads are in flight at once and the words stay in registers
  // for the second pass
  constexpr int kRegWords = 8;
  const int64_t nw = (N + 31) / 32;
  const int64_t w0 = nw * threadIdx.x / blockDim.x, w1 = nw * (threadIdx.x + 1) / blockDim.x;
  const bool in_regs = w1 - w0 <= kRegWords;
  uint32_t wr[kRegWords];
  uint32_t c = 0;
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kRegWords; ++i) wr[i] = w0 + i < w1 ? __ldcg(bm + w0 + i) : 0u;
#pragma unroll
    for (int i = 0; i < kRegWords; ++i) c += __popc(wr[i]);
  } else {
    for (int64_t w = w0; w < w1; ++w) c += __popc(__ldcg(bm + w));
  }
  const uint32_t incl = block_inclusive_scan<uint32_t>(c, sh, nullptr);
  int64_t pos = incl - c;
  int32_t* out = idx + static_cast<int64_t>(b) * top_k;
  auto emit = [&](int64_t w, uint32_t word) {
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (pos < top_k) out[pos] = static_cast<int32_t>(w * 32 + bit);
      ++pos;
    }
  };
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kRegWords; ++i) emit(w0 + i, wr[i]);
  } else {
    for (int64_t w = w0; w < w1; ++w) emit(w, __ldcg(bm + w));
  }
  for (int64_t i = k_eff + threadIdx.x; i < top_k; i += blockDim.x) out[i] = -1;
  if (threadIdx.x == 0) cnt[b] = static_cast<int32_t>(k_eff);
}


// Whole selection of one request in one CTA, for up to kSmallMax candidates. Thread t holds the
// scores of the consecutive indices [t * per, (t + 1) * per) in registers, with per fixed by the
// largest candidate count of the launch so that the loads are issued before the request's own
// count has arrived. The three radix digits (11, 11, 10 bits of the order key) are resolved with
// the histogram split across the block (thread t owns bins [t * NBL, (t + 1) * NBL)), two
// barriers per digit; the first digit's histogram is the one the score kernel counted. Ties at
// the threshold key go to the lowest indices and the winners are written in ascending order, both
// from one block scan of the packed pair (count above the threshold, count equal to it).
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallPerThread = 16;
constexpr int kSmallMax = kSmallThreads * kSmallPerThread;

__global__ void __launch_bounds__(kSmallThreads) topk_small_kernel(const float* scores, int64_t stride,
                                                                   int nmax, int top_k, IndexerWs ws,
                                                                   int32_t* idx, int32_t* cnt) {
  griddep_wait();
  griddep_launch();
  __shared__ __align__(16) uint32_t h2[kHistBins];
  __shared__ __align__(16) uint32_t h3[kHistBins / 2];
  __shared__ uint32_t wsum[2][kSmallWarps];
  __shared__ uint2 bnd;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int per = (nmax + 4 * kSmallThreads - 1) / (4 * kSmallThreads) * 4;  // multiple of 4, <= 16
  const int j0 = tid * per;
  const float* sb = scores + static_cast<int64_t>(b) * stride;

  // every load first: scores (16-byte vectors inside the padded row), first-digit histogram, count
  float4 raw[kSmallPerThread / 4];
#pragma unroll
  for (int v = 0; v < kSmallPerThread / 4; ++v)
    raw[v] = (4 * v < per && j0 + 4 * v < nmax) ? __ldcg(reinterpret_cast<const float4*>(sb + j0) + v)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
  const uint2 c1v = __ldcg(reinterpret_cast<const uint2*>(ws.hist + static_cast<int64_t>(b) * kHistBins) + tid);
  const int N = ws.n_c[b];
  for (int i = tid; i < kHistBins; i += kSmallThreads) h2[i] = 0;
  for (int i = tid; i < kHistBins / 2; i += kSmallThreads) h3[i] = 0;

  uint32_t key[kSmallPerThread];
  uint32_t valid = 0;
#pragma unroll
  for (int v = 0; v < kSmallPerThread / 4; ++v) {
    key[4 * v + 0] = f32_order_key(raw[v].x);
    key[4 * v + 1] = f32_order_key(raw[v].y);
    key[4 * v + 2] = f32_order_key(raw[v].z);
    key[4 * v + 3] = f32_order_key(raw[v].w);
  }
#pragma unroll
  for (int u = 0; u < kSmallPerThread; ++u)
    if (u < per && j0 + u < N) valid |= 1u << u;

  const int k_eff = N < top_k ? N : top_k;
  const bool all = N <= top_k;
  uint32_t T = 0, quota = 0;  // selected: key > T, and the first `quota` keys == T in index order
  if (!all) {
    const uint32_t c1[2] = {c1v.x, c1v.y};
    const uint2 r1 = small_boundary<2, kSmallWarps>(c1, static_cast<uint32_t>(k_eff), wsum[0], &bnd);
    const uint32_t need2 = static_cast<uint32_t>(k_eff) - r1.y;
#pragma unroll
    for (int u = 0; u < kSmallPerThread; ++u)
      if (((valid >> u) & 1u) && (key[u] >> 21) == r1.x) atomicAdd(h2 + ((key[u] >> 10) & 2047u), 1u);
    __syncthreads();
    const uint2 c2v = reinterpret_cast<const uint2*>(h2)[tid];
    const uint32_t c2[2] = {c2v.x, c2v.y};
    const uint2 r2 = small_boundary<2, kSmallWarps>(c2, need2, wsum[1], &bnd);
    const uint32_t need3 = need2 - r2.y;
    const uint32_t p2 = (r1.x << 11) | r2.x;
    if (h2[r2.x] == need3 && p2 > 0) {
      // every key of the boundary bin is taken: the threshold is the bin's lower edge (the same
      // in every thread; the last digit is not needed)
      T = (p2 << 10) - 1;
      quota = 0;
    } else {
#pragma unroll
      for (int u = 0; u < kSmallPerThread; ++u)
        if (((valid >> u) & 1u) && (key[u] >> 10) == p2) atomicAdd(h3 + (key[u] & 1023u), 1u);
      __syncthreads();
      const uint32_t c3[1] = {h3[tid]};
      const uint2 r3 = small_boundary<1, kSmallWarps>(c3, need3, wsum[0], &bnd);
      T = (p2 << 10) | r3.x;
      quota = need3 - r3.y;
    }
  }

  // masks of this thread's keys above T and equal to T; one exclusive block scan of
  // (count above) << 16 | (count equal), both <= kSmallMax
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int u = 0; u < kSmallPerThread; ++u) {
    const bool v = (valid >> u) & 1u;
    gt |= (v && (all || key[u] > T)) ? (1u << u) : 0u;
    eq |= (v && !all && key[u] == T) ? (1u << u) : 0u;
  }
  const uint32_t packed = (static_cast<uint32_t>(__popc(gt)) << 16) | static_cast<uint32_t>(__popc(eq));
  const int lane = tid & 31, w = tid >> 5;
  uint32_t incl = packed;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[1][w] = incl;
  __syncthreads();
  uint32_t below = (lane < w) ? wsum[1][lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
  const uint32_t excl = below + incl - packed;
  const uint32_t eq_before = excl & 0xffffu;
  // the equal keys taken here: the first (quota - eq_before) of this thread's, in index order
  uint32_t take = gt;
  if (eq) {
    uint32_t rest = eq;
    const uint32_t n_take = quota > eq_before ? quota - eq_before : 0u;
    for (uint32_t i = 0; i < n_take && rest; ++i) rest &= rest - 1;  // drop the lowest n_take
    take |= eq & ~rest;
  }
  uint32_t pos = (excl >> 16) + (eq_before < quota ? eq_before : quota);
  int32_t* out = idx + static_cast<int64_t>(b) * top_k;
  while (take) {  // ascending index order
    const int u = __ffs(take) - 1;
    take &= take - 1;
    if (pos < static_cast<uint32_t>(top_k)) out[pos] = j0 + u;
    ++pos;
  }
  for (int i = k_eff + tid; i < top_k; i += kSmallThreads) out[i] = -1;
  if (tid == 0) cnt[b] = k_eff;
}

template <int DT, int NV, int U>
cudaError_t launch_score(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                         const IndexerWs& ws, float* scores, int64_t stride, uint32_t* status,
                         cudaStream_t stream) {
  constexpr int LPE = NV < 32 ? NV : 32;
  constexpr int CH = U * (32 / LPE);
  const int64_t per_req = (static_cast<int64_t>(max_seq_len) / p.r + CH - 1) / CH;
  const int64_t chunks = per_req * batch;
  const int smem = static_cast<int>(sizeof(int32_t) * (2 * batch + 1));
  auto kern = score_kernel<DT, NV, U>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // one wave of persistent CTAs: as many as fit on every SM at once
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  int64_t grid = static_cast<int64_t>(sm_count()) * (per_sm > 0 ? per_sm : 1);
  const int64_t useful = (chunks + kWarps - 1) / kWarps;
  if (grid > useful) grid = useful;
  if (grid < 1) grid = 1;
  prof_begin(kProfScore, stream);
  e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, stream, p, batch, seq_len,
                    max_seq_len, ws, scores, stride, status);
  prof_end(kProfScore, stream);
  return e;
}

template <int DT>
cudaError_t dispatch_score(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                           const IndexerWs& ws, float* scores, int64_t stride, uint32_t* status,
                           cudaStream_t stream) {
  // 16-byte vectors per entry for D = 64 .. 1024: f32 D/4, bf16 D/8, nvfp4 D/32
  const int nv = p.comp_row_bytes / 16;
  constexpr int kMin = DT == CKV_F32 ? 16 : DT == CKV_BF16 ? 8 : 2;
// entries per lane group and chunk: 8, fewer when an entry spans more than 64 vectors (the raw
// registers of a chunk stay at 16 vectors per lane)
#define CKV_SCORE_CASE(M)                                                                    \
  case kMin * M:                                                                             \
    return launch_score<DT, kMin * M,                                                        \
                        (kMin * M < 8 ? kMin * M : (kMin * M > 64 ? 512 / (kMin * M) : 8))>( \
        p, batch, seq_len, max_seq_len, ws, scores, stride, status, stream);
  switch (nv) {
    CKV_SCORE_CASE(1)
    CKV_SCORE_CASE(2)
    CKV_SCORE_CASE(4)
    CKV_SCORE_CASE(8)
    CKV_SCORE_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
#undef CKV_SCORE_CASE
}

}  // namespace

cudaError_t launch_indexer(const LayerParams& p, int batch, const int32_t* seq_len,
                           int max_seq_len, const float* q, int top_k, int32_t* idx, int32_t* cnt,
                           float* scores, const IndexerWs& ws, uint32_t* status,
                           cudaStream_t stream, QueryPrepOut prep, bool early_qbar) {
  const int64_t stride = score_stride(p.r, max_seq_len);
  float* sc = scores ? scores : ws.scores;
  cudaError_t e = cudaSuccess;
  static_assert(kQbarSlices * 8 == kQiHeads, "one query-image part (8 heads) per q_bar slice");
  e = launch_kernel(qbar_kernel, dim3(kQbarSlices, batch), dim3(kQbarThreads), 0, stream, p, seq_len,
                    max_seq_len, q, ws, status, prep, early_qbar);
  if (e != cudaSuccess) return e;
  switch (p.comp_dtype) {
    case CKV_F32: e = dispatch_score<CKV_F32>(p, batch, seq_len, max_seq_len, ws, sc, stride, status, stream); break;
    case CKV_BF16: e = dispatch_score<CKV_BF16>(p, batch, seq_len, max_seq_len, ws, sc, stride, status, stream); break;
    case CKV_NVFP4: e = dispatch_score<CKV_NVFP4>(p, batch, seq_len, max_seq_len, ws, sc, stride, status, stream); break;
    default: e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_topk(p, batch, max_seq_len, top_k, sc, stride, ws, idx, cnt, stream);
}

cudaError_t launch_topk(const LayerParams& p, int batch, int max_seq_len, int top_k, const float* sc,
                        int64_t stride, const IndexerWs& ws, int32_t* idx, int32_t* cnt, cudaStream_t stream) {
  const int64_t nmax = static_cast<int64_t>(max_seq_len) / p.r;
  if (nmax <= kSmallMax)   // every request's candidates fit one CTA's registers
    return launch_kernel(topk_small_kernel, dim3(batch), dim3(kSmallThreads), 0, stream, sc, stride,
                         static_cast<int>(nmax), top_k, ws, idx, cnt);
  dim3 mgrid(static_cast<unsigned>(nmax > 0 ? (nmax + kMarkChunk - 1) / kMarkChunk : 1), batch);
  cudaError_t e = launch_kernel(topk_mark_kernel, mgrid, dim3(kThreads), 0, stream, sc, stride, top_k, ws);
  if (e != cudaSuccess) return e;
  const int smem = static_cast<int>(kFinishCandSmem * sizeof(uint2));
  e = allow_smem(reinterpret_cast<const void*>(topk_finish_kernel), smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(topk_finish_kernel, dim3(batch), dim3(kFinishThreads), smem, stream, top_k, ws, stride,
                       idx, cnt);
}

}  // namespace ckv

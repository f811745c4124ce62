// Step 1 of the decode path: the KV compressor and cache append.
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": tokens are folded by a weighted sum (4x to 128x) and a local window
// keeps full vectors; section "Sto je vLLM morao rijesiti u integraciji?": the compressor
// remainder is held as sliding-window state. Readings: one scalar logit per token, softmax
// weights within the group, each token rotated at its own position before the sum.
//
// One CTA works on whole groups of one request (blockIdx.y). Block x = 0 owns the first group the
// call touches (the only one that reads the residue ring) and, after it, the trailing unfinished
// group (the only one that writes the ring), so ring reads happen before ring writes. Every other
// group of the call is made of new tokens only and is handled by any block, grid-strided.

#include "ckv_internal.h"
#include "query_prep.cuh"

namespace ckv {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kMaxPairsPerThread = 2;  // D <= 1024

struct AppendArgs {
  LayerParams p;
  const int32_t* prev_len;
  const int32_t* cu_new;
  int max_seq_len;
  const float* kv_new;
  const float* logit_new;
  uint32_t* status;
  int prev_offset;  // added to prev_len[b]
};

__device__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float m = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
  if (w == 0) m = warp_max(m);
  if (threadIdx.x == 0) red[0] = m;
  __syncthreads();
  return red[0];
}

// rotated fp32 value of dims (2*pr, 2*pr+1) of a raw token at position pos
__device__ __forceinline__ float2 rotate_raw_pair(const AppendArgs& a, const float* raw, int pr,
                                                  int64_t pos) {
  const LayerParams& p = a.p;
  const float x0 = raw[2 * pr], x1 = raw[2 * pr + 1];
  const int first_rope_pair = (p.D - p.d_r) / 2;
  if (pr < first_rope_pair) return make_float2(x0, x1);
  double o0, o1;
  rope_rotate_pair(x0, x1, static_cast<double>(pos),
                   rope_inv_freq(p, pr - first_rope_pair), false, &o0, &o1);
  return make_float2(static_cast<float>(o0), static_cast<float>(o1));
}

// Writes one rotated token (pairs held by this thread) into window pool row `row` (skipped when
// negative; the reduction still runs so that every thread reaches the same barriers).
__device__ void write_window_token(const AppendArgs& a, int64_t row,
                                   const float2 (&x)[kMaxPairsPerThread], float* red) {
  const LayerParams& p = a.p;
  const int npairs = p.D / 2;
  if (p.win_dtype == CKV_F32) {
    if (row < 0) return;
    float2* dst = reinterpret_cast<float2*>(p.win_codes + row * p.win_row_bytes);
    for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) dst[pr] = x[k];
    return;
  }
  // FP8 e4m3 with one fp32 scale per token: s = amax / 448 (1 when the token is zero)
  float amax = 0.f;
  for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x)
    amax = fmaxf(amax, fmaxf(fabsf(x[k].x), fabsf(x[k].y)));
  amax = block_max(amax, red);
  if (row < 0) return;
  const float s = amax > 0.f ? amax / 448.0f : 1.0f;
  uint16_t* dst = reinterpret_cast<uint16_t*>(p.win_codes + row * p.win_row_bytes);
  for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) {
    const uint32_t c0 = f32_to_e4m3_satfinite(x[k].x / s);
    const uint32_t c1 = f32_to_e4m3_satfinite(x[k].y / s);
    dst[pr] = static_cast<uint16_t>(c0 | (c1 << 8));
  }
  if (threadIdx.x == 0) p.win_scales[row] = s;
}

// Quantises entry c (fp32 in shared memory) into compressed pool row `row`.
__device__ void store_entry(const LayerParams& p, int64_t row, const float* c) {
  const int D = p.D;
  uint8_t* dst = p.comp_codes + row * p.comp_row_bytes;
  if (p.comp_dtype == CKV_F32) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) reinterpret_cast<float*>(dst)[d] = c[d];
  } else if (p.comp_dtype == CKV_BF16) {
    for (int d = threadIdx.x; d < D; d += blockDim.x)
      reinterpret_cast<uint16_t*>(dst)[d] = f32_to_bf16_rne(c[d]);
  } else {  // NVFP4: per 16 elements scale = e4m3(amax / 6), codes = e2m1(x / scale)
    uint8_t* sdst = p.comp_scales + row * (D / 16);
    for (int blk = threadIdx.x; blk < D / 16; blk += blockDim.x) {
      const float* v = c + 16 * blk;
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
      const uint8_t sc = f32_to_e4m3_satfinite(amax / 6.0f);
      const float s = e4m3_to_f32(sc);
      uint32_t lo = 0, hi = 0;
      if (s > 0.f) {
#pragma unroll
        for (int e = 0; e < 8; ++e) lo |= static_cast<uint32_t>(f32_to_e2m1_satfinite(v[e] / s)) << (4 * e);
#pragma unroll
        for (int e = 0; e < 8; ++e) hi |= static_cast<uint32_t>(f32_to_e2m1_satfinite(v[8 + e] / s)) << (4 * e);
      }
      reinterpret_cast<uint2*>(dst)[blk] = make_uint2(lo, hi);
      sdst[blk] = sc;
    }
  }
}

// Weighted sum of ring tokens [t0, t0 + n_ring) of one group, split across the CTA's warps: warp w
// takes a contiguous run of tokens, lane l the rotary-aligned pairs l + 32k (NPL of them), BT
// tokens' loads in flight; each warp writes its partial sums to part[w][D] (zeros if it has none).
template <int NPL, int BT>
__device__ void ring_partial(const float* ring, const float* w, int64_t t0, int r, int n_ring,
                             float* part) {
  constexpr int D = 64 * NPL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int per = (n_ring + nw - 1) / nw;
  const int tlo = warp * per, thi = min(n_ring, tlo + per);
  float2 acc[NPL];
#pragma unroll
  for (int k = 0; k < NPL; ++k) acc[k] = make_float2(0.f, 0.f);
  for (int tb = tlo; tb < thi; tb += BT) {
    float2 x[BT][NPL];
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const int t = tb + u;
      const float2* row = reinterpret_cast<const float2*>(ring + ((t0 + t) % r) * D);
#pragma unroll
      for (int k = 0; k < NPL; ++k) x[u][k] = t < thi ? row[lane + 32 * k] : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < BT; ++u) {
      const float wt = tb + u < thi ? w[tb + u] : 0.f;
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        acc[k].x = fmaf(wt, x[u][k].x, acc[k].x);
        acc[k].y = fmaf(wt, x[u][k].y, acc[k].y);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < NPL; ++k) reinterpret_cast<float2*>(part + warp * D)[lane + 32 * k] = acc[k];
}

// Handles group g of request b: writes the new tokens' window / ring slots and, when the group
// is complete, folds it into entry g.
__device__ void process_group(const AppendArgs& a, int b, int64_t g, int64_t prev, int64_t new_len,
                              int64_t row0, float* smem) {
  const LayerParams& p = a.p;
  const int r = p.r, D = p.D, npairs = D / 2;
  float* w = smem;            // [r] weights
  float* c = smem + 256;      // [D] entry
  float* red = c + 1024;      // [32] reductions
  const int64_t t0 = g * r;
  const int64_t t_end = min(t0 + r, new_len);
  const bool complete = (t0 + r) <= new_len;
  float* ring = p.res_kv + static_cast<int64_t>(b) * r * D;
  float* ring_logit = p.res_logit + static_cast<int64_t>(b) * r;

  // loads that do not depend on the new tokens first: the entry's pool row and the logits
  int64_t crow = -1;
  if (complete) {
    crow = comp_row(p, b, g, a.status);
    if (threadIdx.x < 32)
      for (int t = threadIdx.x; t < r; t += 32) {
        const int64_t pos = t0 + t;
        w[t] = pos < prev ? ring_logit[pos % r] : a.logit_new[row0 + (pos - prev)];
      }
  }

  // new tokens of the group: window and (unfinished group) residue ring
  float2 xlast[kMaxPairsPerThread];
  int64_t pos_last = -1;
  for (int64_t pos = max(t0, prev); pos < t_end; ++pos) {
    const bool to_window = p.W > 0 && pos >= new_len - p.W;
    if (!to_window && complete && pos != t_end - 1) continue;
    const int64_t wrow = to_window ? win_row(p, b, pos, a.status) : -1;
    const float* raw = a.kv_new + (row0 + (pos - prev)) * D;
    float2 x[kMaxPairsPerThread];
    for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) x[k] = rotate_raw_pair(a, raw, pr, pos);
    if (!complete) {
      float2* dst = reinterpret_cast<float2*>(ring + (pos % r) * D);
      for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) dst[pr] = x[k];
      if (threadIdx.x == 0) ring_logit[pos % r] = a.logit_new[row0 + (pos - prev)];
    }
    if (to_window) write_window_token(a, wrow, x, red);
#pragma unroll
    for (int k = 0; k < kMaxPairsPerThread; ++k) xlast[k] = x[k];
    pos_last = pos;
  }
  if (!complete) return;

  // softmax of the group's logits
  __syncthreads();
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    for (int t = threadIdx.x; t < r; t += 32) m = fmaxf(m, w[t]);
    m = warp_max(m);
    float s = 0.f;
    for (int t = threadIdx.x; t < r; t += 32) {
      const float e = expf(w[t] - m);
      w[t] = e;
      s += e;
    }
    s = warp_sum(s);
    for (int t = threadIdx.x; t < r; t += 32) w[t] = w[t] / s;
  }
  __syncthreads();
  // entry = sum over the group's tokens of w_t * rotated token t: the tokens already in the ring
  // are split across the warps (partial sums reduced in shared memory), then the new tokens are
  // added in token order
  const int64_t ring_end = min(prev, t0 + r);
  const int n_ring = ring_end > t0 ? static_cast<int>(ring_end - t0) : 0;
  float* part = smem + 256 + 1024 + 32;  // [warps][D]
  switch (D) {
    case 64: ring_partial<1, 4>(ring, w, t0, r, n_ring, part); break;
    case 128: ring_partial<2, 4>(ring, w, t0, r, n_ring, part); break;
    case 256: ring_partial<4, 4>(ring, w, t0, r, n_ring, part); break;
    case 512: ring_partial<8, 4>(ring, w, t0, r, n_ring, part); break;
    default: ring_partial<16, 2>(ring, w, t0, r, n_ring, part); break;
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) {
    float2 acc = make_float2(0.f, 0.f);
    for (int ww = 0; ww < nw; ++ww) {
      acc.x += part[ww * D + 2 * pr];
      acc.y += part[ww * D + 2 * pr + 1];
    }
    for (int64_t pos = max(t0, prev); pos < t0 + r; ++pos) {
      const float2 x = pos == pos_last ? xlast[k]
                                       : rotate_raw_pair(a, a.kv_new + (row0 + (pos - prev)) * D, pr, pos);
      acc.x = fmaf(w[pos - t0], x.x, acc.x);
      acc.y = fmaf(w[pos - t0], x.y, acc.y);
    }
    c[2 * pr] = acc.x;
    c[2 * pr + 1] = acc.y;
  }
  __syncthreads();
  if (crow >= 0) store_entry(p, crow, c);
  __syncthreads();
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendArgs a) {
  griddep_wait();
  griddep_launch();
  __shared__ float smem[256 + 1024 + 32 + (kAppendThreads / 32) * 1024];
  const int b = blockIdx.y;
  const int64_t prev = static_cast<int64_t>(a.prev_len[b]) + a.prev_offset;
  int64_t row0, n;
  if (a.cu_new) {
    row0 = a.cu_new[b];
    n = static_cast<int64_t>(a.cu_new[b + 1]) - row0;
  } else {
    row0 = b;
    n = 1;
  }
  if (n <= 0) return;
  if (prev < 0 || prev + n > a.max_seq_len) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.status, CKV_DEV_BAD_LENGTH);
    return;
  }
  const int r = a.p.r;
  const int64_t new_len = prev + n;
  const int64_t gA = prev / r, gB = (new_len - 1) / r;
  const bool trailing_unfinished = (new_len % r) != 0;
  if (blockIdx.x == 0) {
    process_group(a, b, gA, prev, new_len, row0, smem);
    __syncthreads();
    if (gB != gA && trailing_unfinished) process_group(a, b, gB, prev, new_len, row0, smem);
  }
  const int64_t mid_end = trailing_unfinished ? gB : gB + 1;
  for (int64_t g = gA + 1 + blockIdx.x; g < mid_end; g += gridDim.x) {
    __syncthreads();
    process_group(a, b, g, prev, new_len, row0, smem);
  }
}

// ---------------------------------------------------------------------------- one new token

// Decode form: every request appends at most one token, so a call either writes one ring slot
// (group unfinished) or folds one group (the token completes it), never both, and no group is
// shared by two calls' ring reads and writes. The fold is split across CTAs by 64-dim slices
// (blockIdx.x): slice s owns the rotary-aligned pairs [32 s, 32 s + 32) of the entry, the ring
// and the window row, so r ring tokens are read by D/64 CTAs instead of one. Each slice rotates
// the whole new token, because the window token's FP8 scale needs the amax of all its dims.
constexpr int kSlicePairs = 32;
constexpr int kRingPreload = 16;  // ring tokens per warp whose loads are issued at the start

// Shared memory of one append_decode_slice group.
struct AppendDecodeSmem {
  float w[256];
  float2 part[kAppendThreads / 32][kSlicePairs];
  float2 xs[kSlicePairs];
  float c[2 * kSlicePairs];
  float red[32];
};

// max over a group of 256 threads (ids tid) synchronising through barrier bar_id
__device__ float group_max(float v, float* red, int tid, int bar_id) {
  v = warp_max(v);
  const int w = tid >> 5, l = tid & 31;
  group_sync(bar_id);
  if (l == 0) red[w] = v;
  group_sync(bar_id);
  float m = (tid < kAppendThreads / 32) ? red[tid] : 0.f;
  if (w == 0) m = warp_max(m);
  if (tid == 0) red[0] = m;
  group_sync(bar_id);
  return red[0];
}

// Slice `slice` of request b, on a group of 256 threads (ids tid, barrier bar_id).
__device__ void append_decode_slice(const AppendArgs& a, int slice, int b, int tid, int bar_id,
                                    AppendDecodeSmem& sm) {
  float* w = sm.w;
  float2 (*part)[kSlicePairs] = sm.part;
  float2* xs = sm.xs;
  float* c = sm.c;
  float* red = sm.red;
  const LayerParams& p = a.p;
  const int warp = tid >> 5, lane = tid & 31, nw = kAppendThreads / 32;
  const int npairs = p.D / 2;
  const int sp = npairs < kSlicePairs ? npairs : kSlicePairs;
  const int pr_lo = slice * sp;
  const int64_t prev = static_cast<int64_t>(a.prev_len[b]) + a.prev_offset;
  int64_t row0 = b, n = 1;
  if (a.cu_new) {
    row0 = a.cu_new[b];
    n = static_cast<int64_t>(a.cu_new[b + 1]) - row0;
  }
  if (n <= 0) return;
  if (n != 1 || prev < 0 || prev + 1 > a.max_seq_len) {
    if (tid == 0 && slice == 0) atomicOr(a.status, CKV_DEV_BAD_LENGTH);
    return;
  }
  const int r = p.r;
  const int64_t pos = prev, t0 = pos / r * r;
  const bool complete = pos == t0 + r - 1;
  const float* ring = p.res_kv + static_cast<int64_t>(b) * r * p.D;
  float* ring_logit = p.res_logit + static_cast<int64_t>(b) * r;

  // every load first: table rows, logits, the new token, this warp's first ring tokens
  int64_t crow = -1;
  const int n_ring = r - 1;  // ring tokens of a completed group: slots 0 .. r - 2
  const int per = (n_ring + nw - 1) / nw;
  const int tlo = warp * per, thi = min(n_ring, tlo + per);
  float2 rx[kRingPreload];
  if (complete) {
    crow = comp_row(p, b, pos / r, a.status);
    for (int t = tid; t < r; t += kAppendThreads) w[t] = t < r - 1 ? ring_logit[t] : a.logit_new[row0];
#pragma unroll
    for (int u = 0; u < kRingPreload; ++u) {
      const int t = tlo + u;
      rx[u] = (t < thi && lane < sp) ? reinterpret_cast<const float2*>(ring + static_cast<int64_t>(t) * p.D)[pr_lo + lane]
                                     : make_float2(0.f, 0.f);
    }
  }
  const int64_t wrow = p.W > 0 ? win_row(p, b, pos, a.status) : -1;
  const float* raw = a.kv_new + row0 * p.D;
  float2 x[kMaxPairsPerThread];
  #pragma unroll
  for (int k = 0; k < kMaxPairsPerThread; ++k) {
    const int pr = tid + k * kAppendThreads;
    x[k] = pr < npairs ? rotate_raw_pair(a, raw, pr, pos) : make_float2(0.f, 0.f);
  }

  // this slice's pairs of the rotated token: ring slot or fold input
#pragma unroll
  for (int k = 0; k < kMaxPairsPerThread; ++k) {
    const int pr = tid + k * kAppendThreads;
    if (pr < pr_lo || pr >= pr_lo + sp) continue;
    if (complete) xs[pr - pr_lo] = x[k];
    else reinterpret_cast<float2*>(p.res_kv + (static_cast<int64_t>(b) * r + pos % r) * p.D)[pr] = x[k];
  }
  if (!complete && slice == 0 && tid == 0) ring_logit[pos % r] = a.logit_new[row0];

  // window row (the new token is always inside the window when W > 0)
  if (p.W > 0) {
    if (p.win_dtype == CKV_F32) {
      if (wrow >= 0)
#pragma unroll
        for (int k = 0; k < kMaxPairsPerThread; ++k) {
          const int pr = tid + k * kAppendThreads;
          if (pr >= pr_lo && pr < pr_lo + sp) reinterpret_cast<float2*>(p.win_codes + wrow * p.win_row_bytes)[pr] = x[k];
        }
    } else {
      float amax = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxPairsPerThread; ++k)
        amax = fmaxf(amax, fmaxf(fabsf(x[k].x), fabsf(x[k].y)));  // zero beyond npairs
      amax = group_max(amax, red, tid, bar_id);
      if (wrow >= 0) {
        const float sc = amax > 0.f ? amax / 448.0f : 1.0f;
        uint16_t* dst = reinterpret_cast<uint16_t*>(p.win_codes + wrow * p.win_row_bytes);
#pragma unroll
        for (int k = 0; k < kMaxPairsPerThread; ++k) {
          const int pr = tid + k * kAppendThreads;
          if (pr < pr_lo || pr >= pr_lo + sp) continue;
          const uint32_t c0 = f32_to_e4m3_satfinite(x[k].x / sc);
          const uint32_t c1 = f32_to_e4m3_satfinite(x[k].y / sc);
          dst[pr] = static_cast<uint16_t>(c0 | (c1 << 8));
        }
        if (slice == 0 && tid == 0) p.win_scales[wrow] = sc;
      }
    }
  }
  if (!complete) return;

  // softmax weights of the group
  group_sync(bar_id);
  if (warp == 0) {
    float m = -INFINITY;
    for (int t = lane; t < r; t += 32) m = fmaxf(m, w[t]);
    m = warp_max(m);
    float sum = 0.f;
    for (int t = lane; t < r; t += 32) {
      const float e = expf(w[t] - m);
      w[t] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    for (int t = lane; t < r; t += 32) w[t] = w[t] / sum;
  }
  group_sync(bar_id);
  // ring tokens: warp partial sums over its run of tokens, lane = pair of the slice
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kRingPreload; ++u) {
    const float wt = tlo + u < thi ? w[tlo + u] : 0.f;
    acc.x = fmaf(wt, rx[u].x, acc.x);
    acc.y = fmaf(wt, rx[u].y, acc.y);
  }
  for (int t = tlo + kRingPreload; t < thi; ++t) {  // r > 8 * kRingPreload + 1 only
    const float2 v = lane < sp ? reinterpret_cast<const float2*>(ring + static_cast<int64_t>(t) * p.D)[pr_lo + lane]
                               : make_float2(0.f, 0.f);
    acc.x = fmaf(w[t], v.x, acc.x);
    acc.y = fmaf(w[t], v.y, acc.y);
  }
  if (lane < sp) part[warp][lane] = acc;
  group_sync(bar_id);
  if (tid < sp) {
    float2 e = make_float2(0.f, 0.f);
    for (int ww = 0; ww < nw; ++ww) {
      e.x += part[ww][tid].x;
      e.y += part[ww][tid].y;
    }
    e.x = fmaf(w[r - 1], xs[tid].x, e.x);
    e.y = fmaf(w[r - 1], xs[tid].y, e.y);
    c[2 * tid] = e.x;
    c[2 * tid + 1] = e.y;
  }
  group_sync(bar_id);
  if (crow < 0) return;
  // this slice's dims of the entry
  const int d_lo = 2 * pr_lo, nd = 2 * sp;
  uint8_t* dst = p.comp_codes + crow * p.comp_row_bytes;
  if (p.comp_dtype == CKV_F32) {
    if (tid < nd) reinterpret_cast<float*>(dst)[d_lo + tid] = c[tid];
  } else if (p.comp_dtype == CKV_BF16) {
    if (tid < nd) reinterpret_cast<uint16_t*>(dst)[d_lo + tid] = f32_to_bf16_rne(c[tid]);
  } else if (tid < nd / 16) {  // NVFP4: one 16-element block per thread
    const float* v = c + 16 * tid;
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(v[e]));
    const uint8_t sc = f32_to_e4m3_satfinite(amax / 6.0f);
    const float s = e4m3_to_f32(sc);
    uint32_t lo = 0, hi = 0;
    if (s > 0.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e) lo |= static_cast<uint32_t>(f32_to_e2m1_satfinite(v[e] / s)) << (4 * e);
#pragma unroll
      for (int e = 0; e < 8; ++e) hi |= static_cast<uint32_t>(f32_to_e2m1_satfinite(v[8 + e] / s)) << (4 * e);
    }
    const int blk = d_lo / 16 + tid;
    reinterpret_cast<uint2*>(dst)[blk] = make_uint2(lo, hi);
    p.comp_scales[crow * (p.D / 16) + blk] = sc;
  }
}

__global__ void __launch_bounds__(kAppendThreads) append_decode_kernel(AppendArgs a) {
  griddep_wait();
  griddep_launch();
  __shared__ AppendDecodeSmem sm;
  append_decode_slice(a, blockIdx.x, blockIdx.y, threadIdx.x, 0, sm);
}

// ---------------------------------------------------------------------------- window replay

// SWA bounded replay (aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section "Proc je obnova
// sliding-window cache draha": after a prefix-cache hit only the last window is replayed and its
// dependence on older positions is cut). One CTA per (window token i, request b): the caller's raw
// token of position L - n_w + i (n_w = min(W, L)) is rotated at that position and written to the
// window cache; if the position belongs to the unfinished group [floor(L/r) r, L) it also goes
// to its residue ring slot with its logit. Compressed entries are not touched. kv_new rows are
// [batch][W][D] (row i of request b), logit_new [batch][W]; prev_len holds L.
__global__ void __launch_bounds__(kAppendThreads) window_replay_kernel(AppendArgs a) {
  griddep_wait();
  griddep_launch();
  __shared__ float red[32];
  const LayerParams& p = a.p;
  const int i = blockIdx.x, b = blockIdx.y;
  const int64_t L = a.prev_len[b];
  if (L < 1 || L > a.max_seq_len) {
    if (i == 0 && threadIdx.x == 0) atomicOr(a.status, CKV_DEV_BAD_LENGTH);
    return;
  }
  const int64_t n_w = min(static_cast<int64_t>(p.W), L);
  if (i >= n_w) return;
  const int64_t pos = L - n_w + i;
  const float* raw = a.kv_new + (static_cast<int64_t>(b) * p.W + i) * p.D;
  const int npairs = p.D / 2;
  float2 x[kMaxPairsPerThread];
  for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) x[k] = rotate_raw_pair(a, raw, pr, pos);
  write_window_token(a, win_row(p, b, pos, a.status), x, red);
  if (pos >= (L / p.r) * p.r) {
    float* dst = p.res_kv + (static_cast<int64_t>(b) * p.r + pos % p.r) * p.D;
    for (int k = 0, pr = threadIdx.x; pr < npairs; ++k, pr += blockDim.x) reinterpret_cast<float2*>(dst)[pr] = x[k];
    if (threadIdx.x == 0) p.res_logit[static_cast<int64_t>(b) * p.r + pos % p.r] = a.logit_new[static_cast<int64_t>(b) * p.W + i];
  }
}

// ---------------------------------------------------------------------------- fused step front

// First kernel of a fused decode step on a dense layer: the append of one slice (threads 0..255)
// and, on the other 256 threads, the attention's query preparation of the same step (the cos/sin
// table of the rotary pairs and, for the tensor-core path, the query image), which reads only the
// query. The two halves synchronise on barriers 1 and 2 and never wait for each other.
__global__ void __launch_bounds__(2 * kAppendThreads, 1) step_front_kernel(
    AppendArgs a, int app_slices, const float* q, QueryPrepOut prep, AttnWs aws, int prep_parts) {
  griddep_wait();
  griddep_launch();
  __shared__ AppendDecodeSmem sm;
  __shared__ double rope_tmp[2 * kQiMaxRopePairs];
  const int x = blockIdx.x, b = blockIdx.y;
  if (threadIdx.x < kAppendThreads) {
    if (x < app_slices) append_decode_slice(a, x, b, threadIdx.x, 1, sm);
  } else if (x < prep_parts) {
    prep_part(a.p, a.prev_len, a.max_seq_len, aws, x, b, threadIdx.x - kAppendThreads);
    if (prep.qimage)
      qimage_part(a.p, a.prev_len, a.max_seq_len, q, prep, x, b, threadIdx.x - kAppendThreads, rope_tmp, 2);
  }
}

}  // namespace

cudaError_t launch_step_front(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                              const float* kv_new, const float* logit_new, const float* q,
                              QueryPrepOut prep, const AttnWs& aws, uint32_t* status, cudaStream_t stream) {
  // the new token of request b is at position seq_len[b] - 1
  const AppendArgs a{p, seq_len, nullptr, max_seq_len, kv_new, logit_new, status, -1};
  const int app_slices = p.D / 2 < kSlicePairs ? 1 : p.D / 2 / kSlicePairs;
  const int prep_parts = prep.qimage ? kQiHeads / 8 : 1;  // the rotary table; the query image by 8 heads
  const dim3 grid(app_slices > prep_parts ? app_slices : prep_parts, batch);
  return launch_kernel(step_front_kernel, grid, dim3(2 * kAppendThreads), 0, stream, a, app_slices, q, prep, aws,
                       prep_parts);
}

cudaError_t launch_append(const LayerParams& p, int batch, const int32_t* prev_len,
                          const int32_t* cu_new, int max_new, int max_seq_len, const float* kv_new,
                          const float* logit_new, uint32_t* status, cudaStream_t stream,
                          int prev_offset) {
  AppendArgs a{p, prev_len, cu_new, max_seq_len, kv_new, logit_new, status, prev_offset};
  if (max_new == 1) {  // one token per request: the fold split across 64-dim slices
    const int slices = p.D / 2 < kSlicePairs ? 1 : p.D / 2 / kSlicePairs;
    return launch_kernel(append_decode_kernel, dim3(slices, batch), dim3(kAppendThreads), 0, stream, a);
  }
  const int64_t groups = static_cast<int64_t>(max_new) / p.r + 2;
  const int gx = static_cast<int>(groups < 512 ? groups : 512);
  dim3 grid(gx, batch);
  return launch_kernel(append_kernel, grid, dim3(kAppendThreads), 0, stream, a);
}

cudaError_t launch_window_replay(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                                 const float* kv, const float* logit, uint32_t* status, cudaStream_t stream) {
  if (p.W < 1) return cudaSuccess;
  AppendArgs a{p, seq_len, nullptr, max_seq_len, kv, logit, status, 0};
  return launch_kernel(window_replay_kernel, dim3(p.W, batch), dim3(kAppendThreads), 0, stream, a);
}

}  // namespace ckv

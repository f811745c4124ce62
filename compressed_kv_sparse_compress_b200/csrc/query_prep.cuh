// Query passes shared by the kernels of the indexer, the attention and the fused decode step's
// front kernel: the head-averaged query q_bar of the indexer's q-bar pass (one slice of dim pairs
// per call), the cos/sin table of the rotary pairs at the query position (for the combine's
// inverse rotation; attention prep and the dense front kernel) and a part of the attention's query
// image (the q-bar pass and the dense front kernel). Each runs on a group of 256 threads (ids tid)
// that synchronise through barrier bar_id (0 when the group is the whole CTA).
#pragma once

#include "ckv_internal.h"
#include "qimage.cuh"

namespace ckv {

constexpr int kQbarThreads = 256;
constexpr int kQbarSlices = 8;
constexpr int kPrepThreads = 256;

__device__ __forceinline__ void group_sync(int bar_id) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(256) : "memory");
}

// kQbarSlices CTAs of 256 threads per request, CTA s owning the rotary-aligned dim pairs
// [s * P, (s + 1) * P) with P = D / 2 / kQbarSlices: thread (pair k, head group g) sums its heads of
// one pair in fp64 with all its loads in flight at once; the head groups are added in shared
// memory, the sum rotated and scaled. The slices also reset the request's selection state.
// With `prep` set (a fused decode step), the same pass writes the cos/sin table of the rotary
// pairs that the attention's query preparation would write.

__device__ __forceinline__ void qbar_slice(const LayerParams& p, const int32_t* seq_len, int max_seq_len,
                                           const float* q, const IndexerWs& ws, uint32_t* status,
                                           const QueryPrepOut& prep, int slice, int b, int tid,
                                           double (*part)[2], int bar_id) {
  const int L = seq_len[b];
  const bool ok = L >= 1 && L <= max_seq_len;
  if (slice == 0 && tid == 0) {
    if (!ok) atomicOr(status, CKV_DEV_BAD_LENGTH);
    ws.n_c[b] = ok ? L / p.r : 0;
    ws.cand_cnt[b] = 0;
  }
  constexpr int kBinsPerSlice = kHistBins / kQbarSlices;
  for (int i = tid; i < kBinsPerSlice; i += kQbarThreads)
    ws.hist[static_cast<int64_t>(b) * kHistBins + slice * kBinsPerSlice + i] = 0;
  const int P = p.D / 2 / kQbarSlices;  // 4 .. 64 pairs (D = 64 .. 1024)
  const int G = kQbarThreads / P;       // head groups
  const int k = tid % P, g = tid / P;
  const int pr = slice * P + k, first_rope = (p.D - p.d_r) / 2;
  const float* qb = q + static_cast<int64_t>(b) * p.H * p.D;
  const int h_lo = (p.H * g) / G, h_hi = (p.H * (g + 1)) / G;
  const bool rope_pair = pr >= first_rope && ok;
  const bool rotate = rope_pair && g == 0;
  double s0 = 0.0, s1 = 0.0, rsn = 0.0, rcs = 1.0;
  bool have_angle = false;
  for (int h0 = h_lo; h0 < h_hi; h0 += 16) {
    float2 v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
      v[u] = h0 + u < h_hi ? __ldg(reinterpret_cast<const float2*>(qb + static_cast<int64_t>(h0 + u) * p.D) + pr)
                           : make_float2(0.f, 0.f);
    if (rotate && !have_angle) {  // rotation angle while the loads fly
      sincos(static_cast<double>(L - 1) * rope_inv_freq(p, pr - first_rope), &rsn, &rcs);
      have_angle = true;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      s0 += v[u].x;
      s1 += v[u].y;
    }
  }
  if (rotate && !have_angle)  // head group 0 holds no heads when H < G
    sincos(static_cast<double>(L - 1) * rope_inv_freq(p, pr - first_rope), &rsn, &rcs);
  if (prep.rope && rope_pair && g == 0) {
    double* rope_g = prep.rope + static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2;
    rope_g[2 * (pr - first_rope)] = rcs;
    rope_g[2 * (pr - first_rope) + 1] = rsn;
  }
  part[tid][0] = s0;
  part[tid][1] = s1;
  group_sync(bar_id);
  if (g == 0) {
    double a = 0.0, c = 0.0;
    for (int gg = 0; gg < G; ++gg) {
      a += part[gg * P + k][0];
      c += part[gg * P + k][1];
    }
    if (rope_pair) {
      const double x = a;
      a = x * rcs - c * rsn;
      c = x * rsn + c * rcs;
    }
    const double scale = static_cast<double>(p.sm_scale) / p.H;
    reinterpret_cast<float2*>(ws.qbar + static_cast<int64_t>(b) * p.D)[pr] =
        make_float2(static_cast<float>(a * scale), static_cast<float>(c * scale));
  }
}

// Per request: cos/sin of every rotary pair at the query position L-1 (fp64 angles), for the
// inverse rotation in the combine, by kPrepThreads threads with ids tid (part 0 of request b).
__device__ __forceinline__ void prep_part(const LayerParams& p, const int32_t* seq_len, int max_seq_len,
                                          const AttnWs& ws, int part, int b, int tid) {
  if (part != 0) return;
  const int L = seq_len[b];
  if (L < 1 || L > max_seq_len) return;
  const int n_pairs = p.d_r / 2;
  double* rope_g = ws.rope + static_cast<int64_t>(b) * (n_pairs + 1) * 2;
  for (int i = tid; i < n_pairs; i += kPrepThreads) {
    double sn, cs;
    sincos(static_cast<double>(L - 1) * rope_inv_freq(p, i), &sn, &cs);
    rope_g[2 * i] = cs;
    rope_g[2 * i + 1] = sn;
  }
}

// Per request: the query image of heads 8 part .. 8 part + 7 (qimage.cuh) for the tensor-core
// attention, one warp per head, by 256 threads with ids tid that synchronise through barrier
// bar_id; rope_tmp is shared memory for the cos/sin table (2 * d_r/2 doubles). Only for layers of
// 64 heads of dimension 512 (the caller checks); a bad length leaves the image unwritten.
__device__ __forceinline__ void qimage_part(const LayerParams& p, const int32_t* seq_len, int max_seq_len,
                                            const float* q, const QueryPrepOut& prep, int part, int b, int tid,
                                            double* rope_tmp, int bar_id) {
  const int L = seq_len[b];
  if (L < 1 || L > max_seq_len) return;
  const int w = tid >> 5, lane = tid & 31, h = 8 * part + w;
  float x[16];
  const float4* src = reinterpret_cast<const float4*>(q + (static_cast<int64_t>(b) * kQiHeads + h) * kQiDim + 16 * lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 v = __ldg(src + k);
    x[4 * k] = v.x;
    x[4 * k + 1] = v.y;
    x[4 * k + 2] = v.z;
    x[4 * k + 3] = v.w;
  }
  for (int i = tid; i < p.d_r / 2; i += kPrepThreads)
    rope_sincos(static_cast<double>(L - 1) * rope_inv_freq(p, i), &rope_tmp[2 * i + 1], &rope_tmp[2 * i]);
  group_sync(bar_id);
  uint4 hi[2], lo[2];
  const float sc = qimage_head(x, lane, (kQiDim - p.d_r) / 2, rope_tmp, hi, lo);
  uint8_t* img = prep.qimage + static_cast<int64_t>(b) * kQImageBytes;
  const int rh = qimage_row(h, 0), rl = qimage_row(h, 1);
  *reinterpret_cast<uint4*>(img + qimage_offset(rh, 2 * lane)) = hi[0];
  *reinterpret_cast<uint4*>(img + qimage_offset(rh, 2 * lane + 1)) = hi[1];
  *reinterpret_cast<uint4*>(img + qimage_offset(rl, 2 * lane)) = lo[0];
  *reinterpret_cast<uint4*>(img + qimage_offset(rl, 2 * lane + 1)) = lo[1];
  if (lane == 0) prep.qscale[static_cast<int64_t>(b) * kQiHeads + h] = sc;
}

}  // namespace ckv

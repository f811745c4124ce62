// The query operand of the tensor-core attention (H = 64 heads, D = 512): every head's rotated
// query, scaled by a power of two and split into fp16 hi and lo parts, laid out exactly as the
// attention kernel's shared memory holds it (so that a plain bulk copy brings it in):
//   8 chunks of 64 dims, 16 KB each; in a chunk, 128 rows of 128 bytes with the 128-byte swizzle
//   (16-byte granule g of row r at ((g ^ r) & 7) * 16); row 32 j + i holds the hi part (i < 16)
//   or the lo part (i >= 16) of head 16 j + i % 16.
// The logit of head h and key x is then (Q'hi[h] + Q'lo[h]) . x times the head's scale 2^-s_h.
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": rotary embedding on the last d_r dims of the query, before the dot
// product with the shared K=V vectors.
//
// Built by one warp per head, either by the attention kernel itself or, in a fused decode step,
// once per request by the step's query pass (into the attention workspace).
#pragma once

#include <cuda_fp16.h>

#include "ckv_common.cuh"

namespace ckv {

constexpr int kQiHeads = 64;
constexpr int kQiDim = 512;
constexpr uint32_t kQiChunk = 2 * kQiHeads * 128;                      // 16 KB
constexpr uint32_t kQImageBytes = kQiChunk * (kQiDim / 64);            // 128 KB
constexpr int kQiMaxRopePairs = 256;

// row of (head h, part): hi part 0, lo part 1
__host__ __device__ constexpr int qimage_row(int h, int part) { return 32 * (h >> 4) + 16 * part + (h & 15); }

// byte offset of the 16-byte granule g (dims 8 g .. 8 g + 7) of row `row`
__device__ __forceinline__ uint32_t qimage_offset(int row, int g) {
  return static_cast<uint32_t>(g >> 3) * kQiChunk + static_cast<uint32_t>(row) * 128u +
         (static_cast<uint32_t>((g & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t qi_pack(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One head, one warp: lane l holds dims 16 l .. 16 l + 15 of the head's query in x (modified).
// The rotary pairs (first_rope .. D/2 - 1) are rotated at the query position with the fp64 cos,
// sin table `rope` (pair i - first_rope at rope[2 i], rope[2 i + 1]); the head is scaled by the
// power of two that puts its largest magnitude in [2^8, 2^9) (within the range where the power
// and its inverse are normal) and split into fp16 hi and lo parts. Returns the granules 2 l and
// 2 l + 1 of the hi row (hi[0], hi[1]) and of the lo row, and the head's scale 2^-s (the same in
// every lane).
__device__ __forceinline__ float qimage_head(float (&x)[16], int lane, int first_rope, const double* rope,
                                             uint4 (&hi)[2], uint4 (&lo)[2]) {
  if (8 * lane + 7 >= first_rope) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int pr = 8 * lane + k;
      if (pr >= first_rope) {
        const double rc = rope[2 * (pr - first_rope)], rs = rope[2 * (pr - first_rope) + 1];
        const double a0 = x[2 * k], a1 = x[2 * k + 1];
        x[2 * k] = static_cast<float>(a0 * rc - a1 * rs);
        x[2 * k + 1] = static_cast<float>(a0 * rs + a1 * rc);
      }
    }
  }
  uint32_t mb = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) mb = max(mb, __float_as_uint(x[k]) & 0x7fffffffu);
  mb = __reduce_max_sync(0xffffffffu, mb);
  int sh = 0;
  if (mb != 0u) sh = max(-126, min(126, 8 - (static_cast<int>(mb >> 23) - 127)));
  const float up = __int_as_float((127 + sh) << 23);
  uint32_t h[8], l[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float a = x[2 * k] * up, c = x[2 * k + 1] * up;
    const __half2 h16 = __floats2half2_rn(a, c);
    const float2 back = __half22float2(h16);
    h[k] = *reinterpret_cast<const uint32_t*>(&h16);
    l[k] = qi_pack(a - back.x, c - back.y);
  }
  hi[0] = make_uint4(h[0], h[1], h[2], h[3]);
  hi[1] = make_uint4(h[4], h[5], h[6], h[7]);
  lo[0] = make_uint4(l[0], l[1], l[2], l[3]);
  lo[1] = make_uint4(l[4], l[5], l[6], l[7]);
  return __int_as_float((127 - sh) << 23);
}

}  // namespace ckv

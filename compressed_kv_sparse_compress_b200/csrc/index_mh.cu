// Multi-head indexer: its own compressed index keys, H_I index heads with one weight each, scored
// as one FP8 contraction on the tensor cores.
//
// aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section "Vykon neprinesl jeden kernel": the
// "Sparse MQA logits" kernel scores only the candidate positions. Reading (the multi-head form of
// that indexer): per token the caller supplies an index key of d_I dims; the keys of a group are
// folded with the softmax of the group's compressor logits (24-ai.news "vLLM uveo DeepSeek V4 s
// 8,7x manjim KV cacheom", section "Kako funkcionira optimizacija KV cachea?": compression by a
// weighted sum of tokens) and stored as FP8 e4m3 with one fp32 scale per entry, in an index plane
// that shares the compressed pool's blocks, rows and table. At decode time each head's index
// query is stored by the same FP8 rule (codes q~_h, scale t_h) and, with w_h the head's weight,
// candidate j (codes c_j, scale s_j) scores
//     score_j = s_j * sum_h (w_h t_h) * max(0, q~_h . c_j)
// which equals sum_h w_h max(0, q^_h . k_j) for the decoded query and entry (both scales > 0).
//
// Kernels:
//   index_append_kernel  the index-key compressor (same grouping and ring rules as the K=V
//                        append: block 0 owns the first group of the call, the only one that
//                        reads the ring, and then the trailing unfinished group, the only one
//                        that writes it)
//   mh_prep_kernel       per request: candidate count, reset of the selection state, the FP8
//                        query image (128-byte swizzled rows) and the scaled head weights
//   mh_score_kernel      persistent, warp-specialised: TMA loads of 64-entry runs of index rows
//                        (one pool block each) into a ring of shared-memory stages with the
//                        128-byte swizzle of the MMA operand; S^T[128 entries, H_I] = C . Q~^T as
//                        tcgen05 kind::f8f6f4 (e4m3 x e4m3, fp32 accumulation) into one of two
//                        tensor-memory accumulators; an epilogue of one thread per entry (TMEM
//                        lane) forms the weighted ReLU sum over heads, applies the entry scale,
//                        stores the score and counts the first radix digit of its order key,
//                        while the next tile's MMAs run
// after which the top-k kernels of the head-averaged indexer select from the scores.

#include <cuda.h>

#include "ckv_internal.h"
#include "ckv_ptx.cuh"

namespace ckv {

size_t mh_image_bytes(const IndexParams& ip, int batch) {
  // FP8 query images [B][H_I][d_I], then the scaled head weights [B][H_I] fp32
  return align_up(static_cast<size_t>(batch) * ip.heads * ip.dim, 256) +
         align_up(static_cast<size_t>(batch) * ip.heads * 4, 256);
}

namespace {

// ---------------------------------------------------------------------------- index append

constexpr int kIdxAppendThreads = 128;

struct IndexAppendArgs {
  LayerParams p;
  IndexParams ip;
  const int32_t* prev_len;
  const int32_t* cu_new;
  int max_seq_len;
  const float* k_new;
  const float* logit_new;
  uint32_t* status;
};

__device__ float block_max128(float v, float* red) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  const float m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return m;
}

// Group g of request b: ring writes of the new tokens of an unfinished group, or the fold and the
// FP8 store of a complete one. w: [256] shared weights, red: [4] shared.
__device__ void index_group(const IndexAppendArgs& a, int b, int64_t g, int64_t prev, int64_t new_len,
                            int64_t row0, float* w, float* red) {
  const int r = a.p.r, dI = a.ip.dim;
  const int64_t t0 = g * r;
  const int64_t t_end = min(t0 + r, new_len);
  const bool complete = t0 + r <= new_len;
  float* ring = a.ip.res_k + static_cast<int64_t>(b) * r * dI;
  float* ring_logit = a.ip.res_logit + static_cast<int64_t>(b) * r;
  if (!complete) {
    for (int64_t pos = max(t0, prev); pos < t_end; ++pos) {
      const float* src = a.k_new + (row0 + (pos - prev)) * dI;
      for (int d = threadIdx.x; d < dI; d += kIdxAppendThreads) ring[(pos % r) * dI + d] = src[d];
      if (threadIdx.x == 0) ring_logit[pos % r] = a.logit_new[row0 + (pos - prev)];
    }
    return;
  }
  for (int t = threadIdx.x; t < r; t += kIdxAppendThreads) {
    const int64_t pos = t0 + t;
    w[t] = pos < prev ? ring_logit[pos % r] : a.logit_new[row0 + (pos - prev)];
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // softmax of the group's logits, fp32
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
  // entry = sum over the group's tokens, in token order, of w_t * key_t (d_I <= 256: two dims
  // per thread at most)
  float c[2] = {0.f, 0.f};
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int d = threadIdx.x + kIdxAppendThreads * k;
    if (d >= dI) break;
    float acc = 0.f;
    for (int t = 0; t < r; ++t) {
      const int64_t pos = t0 + t;
      const float x = pos < prev ? ring[(pos % r) * dI + d] : a.k_new[(row0 + (pos - prev)) * dI + d];
      acc = fmaf(w[t], x, acc);
    }
    c[k] = acc;
    amax = fmaxf(amax, fabsf(acc));
  }
  amax = block_max128(amax, red);
  const int64_t row = comp_row(a.p, b, g, a.status);
  if (row >= 0) {
    const float s = amax > 0.f ? amax / 448.0f : 1.0f;  // the window's FP8 rule, per entry
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int d = threadIdx.x + kIdxAppendThreads * k;
      if (d < dI) a.ip.codes[row * dI + d] = f32_to_e4m3_satfinite(c[k] / s);
    }
    if (threadIdx.x == 0) a.ip.scales[row] = s;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kIdxAppendThreads) index_append_kernel(IndexAppendArgs a) {
  griddep_wait();
  griddep_launch();
  __shared__ float w[256];
  __shared__ float red[4];
  const int b = blockIdx.y;
  const int64_t prev = a.prev_len[b];
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
    index_group(a, b, gA, prev, new_len, row0, w, red);
    __syncthreads();
    if (gB != gA && trailing_unfinished) index_group(a, b, gB, prev, new_len, row0, w, red);
  }
  const int64_t mid_end = trailing_unfinished ? gB : gB + 1;
  for (int64_t g = gA + 1 + blockIdx.x; g < mid_end; g += gridDim.x) {
    __syncthreads();
    index_group(a, b, g, prev, new_len, row0, w, red);
  }
}

// ---------------------------------------------------------------------------- query image

constexpr int kMhPrepThreads = 256;

// One CTA per (8 heads, request), one warp per head, so that every head's loads are in flight at
// once: the index query of each head stored by the FP8 rule (s_h = amax_h / 448, 1 for a zero
// head; codes e4m3 of q / s_h) as the K-major operand image (chunk c = dims 128c .. 128c+127 holds
// H_I rows of 128 bytes, 16-byte granule g of row h stored at slot g ^ (h % 8)) and the head
// weights scaled by s_h (wq). The CTAs of head group 0 also set the candidate count and reset the
// selection state.
__global__ void __launch_bounds__(kMhPrepThreads) mh_prep_kernel(LayerParams p, IndexParams ip,
                                                                 const int32_t* seq_len, int max_seq_len,
                                                                 const float* q_index, const float* weights,
                                                                 IndexerWs ws, uint8_t* qimage, float* wq,
                                                                 uint32_t* status) {
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (blockIdx.x == 0) {
    const int L = seq_len[b];
    const bool ok = L >= 1 && L <= max_seq_len;
    if (tid == 0) {
      if (!ok) atomicOr(status, CKV_DEV_BAD_LENGTH);
      ws.n_c[b] = ok ? L / p.r : 0;
      ws.cand_cnt[b] = 0;
    }
    for (int i = tid; i < kHistBins; i += kMhPrepThreads) ws.hist[static_cast<int64_t>(b) * kHistBins + i] = 0;
  }
  const int dI = ip.dim;  // 128 or 256: lane l holds dims [e l, e l + e), e = dI / 32
  const int e = dI / 32;
  uint8_t* img = qimage + static_cast<int64_t>(b) * ip.heads * dI;
  const int h = blockIdx.x * (kMhPrepThreads / 32) + warp;
  if (h < ip.heads) {
    const float* qh = q_index + (static_cast<int64_t>(b) * ip.heads + h) * dI + e * lane;
    float x[8];
    const float4 v0 = __ldg(reinterpret_cast<const float4*>(qh));
    x[0] = v0.x; x[1] = v0.y; x[2] = v0.z; x[3] = v0.w;
    if (e == 8) {
      const float4 v1 = __ldg(reinterpret_cast<const float4*>(qh) + 1);
      x[4] = v1.x; x[5] = v1.y; x[6] = v1.z; x[7] = v1.w;
    } else {
      x[4] = x[5] = x[6] = x[7] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(x[k]));
    amax = warp_max(amax);
    const float s = amax > 0.f ? amax / 448.0f : 1.0f;
    uint32_t c[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) c[k >> 2] |= static_cast<uint32_t>(f32_to_e4m3_satfinite(x[k] / s)) << (8 * (k & 3));
    const int d0 = e * lane;                       // first dim of this lane
    const int chunk = d0 >> 7, g = (d0 & 127) >> 4;  // 128-dim chunk, 16-byte granule in its row
    uint8_t* dst = img + chunk * (ip.heads * 128) + h * 128 + ((g ^ (h & 7)) << 4) + (d0 & 15);
    if (e == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(c[0], c[1]);
    else *reinterpret_cast<uint32_t*>(dst) = c[0];
    if (lane == 0) wq[static_cast<int64_t>(b) * ip.heads + h] = weights[static_cast<int64_t>(b) * ip.heads + h] * s;
  }
}

// ---------------------------------------------------------------------------- scoring

// Warp roles of the score kernel (128 + 128 G threads, G = 1 or 2 epilogue groups): warp 0 lane 0
// loads (TMA for the index rows, bulk copies for the entry scales and the query images), warp 1
// lane 0 issues the MMAs, warps 4..4G+3 (TMEM lane quarters 0..3, one entry per thread) run the
// epilogue; with G = 2 the first group takes the tiles of accumulator 0 and the second those of
// accumulator 1, so that two tiles' epilogues overlap. Warp 2 allocates and frees the tensor
// memory; otherwise warps 2, 3 and the other lanes only take part in the set-up and the final
// barrier. G = 1 runs 3 CTAs per SM with 3 stages, G = 2 runs 2 CTAs per SM (the register file
// holds no third) with 4 stages.
constexpr int kMaxScoreThreads = 384;
constexpr int kEpiWarps = 8;    // weight slots for the largest G
constexpr int kTile = 128;      // entries per tile = MMA M
constexpr int kBoxRows = 64;    // entries per TMA box (one pool block holds 256 / r >= 64 of them)
constexpr int kMeta = 8;        // slots of per-tile entry scales (> stages + 2 tiles in flight)

__host__ __device__ constexpr int score_threads(int groups) { return 128 + 128 * groups; }
__host__ __device__ constexpr int score_ctas(int groups) { return groups == 2 ? 2 : 3; }
// shared-memory stages of index rows: d_I = 128 as above, 2 for d_I = 256
__host__ __device__ constexpr int score_stages(int dim, int groups) { return dim == 128 ? (groups == 2 ? 4 : 3) : 2; }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T, both e4m3 (kind::f8f6f4, fp32 accumulation)
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// K-major operand with 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;            // leading byte offset 16 (unused when swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;    // stride byte offset 1024
  d |= static_cast<uint64_t>(1) << 46;            // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;            // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA load of box (x, y) of `map` into shared memory, completing on bar (no multicast)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Shared memory of the score kernel, byte offsets from a 1024-aligned base.
struct MhSmem {
  uint32_t stage_bytes, stages, a, q, q_bytes, w, meta, mask, bars, tmem, flag, scan, prefix, end_fixed;
  __host__ __device__ MhSmem(int heads, int dim, int groups) {
    stage_bytes = kTile * dim;                         // 128 entries x d_I e4m3
    stages = score_stages(dim, groups);
    a = 0;
    q = a + stages * stage_bytes;                      // 2 query slots of H_I x d_I e4m3
    q_bytes = static_cast<uint32_t>(heads) * dim;
    w = q + 2 * ((q_bytes + 1023) / 1024 * 1024);      // float[8 warps][2][H] scaled weights
    meta = w + (kEpiWarps * 2 * 4 * heads + 1023) / 1024 * 1024;  // float[kMeta][128] entry scales
    mask = meta + kMeta * 512;                         // int[kMeta] valid 64-entry runs
    bars = mask + 4 * kMeta;                           // uint64: full[8], empty[8], qfull[2],
                                                       // qempty[2], tfull[2], tempty[2], drain,
                                                       // mfull[kMeta], mempty[kMeta]
    tmem = bars + 8 * (25 + 2 * kMeta);
    flag = tmem + 8;                                   // int abort flag
    scan = flag + 8;                                   // int32[kMaxScoreThreads / 32]
    prefix = scan + 4 * (kMaxScoreThreads / 32);       // int32[batch + 1], then n_c [batch]
    end_fixed = prefix;
  }
};

// Position of tile t in the flattened (request, tile) list: request b, first entry e0, entries
// n_valid.
struct TileInfo {
  int b;
  int64_t e0;
  int n_valid;
};

// Walks a CTA's consecutive tiles: one binary search for the first, then the request index only
// moves forward.
struct TileWalk {
  const int32_t* prefix;
  const int32_t* n_c;
  int b;
  __device__ TileWalk(const int32_t* pf, const int32_t* nc, int batch, int64_t t0) : prefix(pf), n_c(nc) {
    int lo = 0, hi = batch;  // last b with prefix[b] <= t0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= t0) lo = mid; else hi = mid;
    }
    b = lo;
  }
  __device__ __forceinline__ TileInfo at(int64_t t) {  // t never decreases between calls
    while (prefix[b + 1] <= t) ++b;
    TileInfo ti;
    ti.b = b;
    ti.e0 = (t - prefix[b]) * kTile;
    ti.n_valid = static_cast<int>(min(static_cast<int64_t>(kTile), static_cast<int64_t>(n_c[b]) - ti.e0));
    return ti;
  }
};

template <int DI, int G>
__global__ void __launch_bounds__(score_threads(G), score_ctas(G)) mh_score_kernel(const __grid_constant__ CUtensorMap rows_map,
                                                                     LayerParams p, IndexParams ip, int batch,
                                                                     IndexerWs ws, const uint8_t* qimage,
                                                                     const float* wq, float* scores, int64_t stride,
                                                                     uint32_t tmem_cols, uint32_t* status) {
  constexpr int kScoreThreads = score_threads(G);
  const MhSmem S(ip.heads, DI, G);
  constexpr int kNS = score_stages(DI, G);
  constexpr int kChunks = DI / 128;  // 128-byte column chunks of a row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  float* w_sh = reinterpret_cast<float*>(base + S.w);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + S.flag);
  int32_t* scan_sh = reinterpret_cast<int32_t*>(base + S.scan);
  int32_t* prefix = reinterpret_cast<int32_t*>(base + S.prefix);
  int32_t* n_c = prefix + batch + 1;
  const uint32_t bar0 = sb + S.bars;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (8 + s); };
  auto qfull = [&](int s) { return bar0 + 8u * (16 + s); };
  auto qempty = [&](int s) { return bar0 + 8u * (18 + s); };
  auto tfull = [&](int s) { return bar0 + 8u * (20 + s); };
  auto tempty = [&](int s) { return bar0 + 8u * (22 + s); };
  const uint32_t drain = bar0 + 8u * 24;
  auto mfull = [&](int s) { return bar0 + 8u * (25 + s); };
  auto mempty = [&](int s) { return bar0 + 8u * (25 + kMeta + s); };
  float* meta_sc = reinterpret_cast<float*>(base + S.meta);
  volatile int* meta_mask = reinterpret_cast<volatile int*>(base + S.mask);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = ip.heads;
  const uint32_t qslot_bytes = (S.q_bytes + 1023) / 1024 * 1024;
  // fp32 accumulator, e4m3 A and B (both K-major), M = 128, N = H
  const uint32_t idesc = (1u << 4) | ((static_cast<uint32_t>(H) >> 3) << 17) | ((128u >> 4) << 24);

  // set-up that reads no global memory, before waiting for the previous kernel
  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(qfull(s), 1);
      mbar_init(qempty(s), 1);
      mbar_init(tfull(s), 1);
      mbar_init(tempty(s), 128);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kMeta; ++s) {
      mbar_init(mfull(s), 1);
      mbar_init(mempty(s), 128);
    }
    *abort_flag = 0;
    fence_proxy_async();
  }
  if (warp == 2) tmem_alloc(sb + S.tmem, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<uint32_t*>(base + S.tmem);
  griddep_wait();
  griddep_launch();

  // tiles per request and their exclusive prefix (thread t sums requests [t*per, (t+1)*per))
  {
    const int per = (batch + kScoreThreads - 1) / kScoreThreads;
    int32_t s = 0;
    for (int i = 0; i < per; ++i) {
      const int bb = tid * per + i;
      if (bb < batch) {
        const int32_t n = ws.n_c[bb];
        n_c[bb] = n;
        s += (n + kTile - 1) / kTile;
      }
    }
    int32_t v = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) scan_sh[warp] = v;
    __syncthreads();
    int32_t before = 0, total = 0;
    for (int ww = 0; ww < kScoreThreads / 32; ++ww) {
      if (ww < warp) before += scan_sh[ww];
      total += scan_sh[ww];
    }
    int32_t run = before + v - s;
    for (int i = 0; i < per; ++i) {
      const int bb = tid * per + i;
      if (bb < batch) {
        prefix[bb] = run;
        run += (n_c[bb] + kTile - 1) / kTile;
      }
    }
    if (tid == 0) prefix[batch] = total;
    __syncthreads();
  }
  const int64_t total = prefix[batch];
  const int64_t t_lo = total * blockIdx.x / gridDim.x;
  const int64_t t_hi = total * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0 && lane == 0) {
    // ---------------- loads: query image per request switch; per tile the index rows (TMA) and
    //                  the entry scales (bulk copies into the scale ring); the block-table entries
    //                  of the next tile are loaded while the current one is issued
    auto table_runs = [&](const TileInfo& ti, int32_t (&ph)[2]) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int64_t e = ti.e0 + kBoxRows * j;
        ph[j] = e < n_c[ti.b] ? p.comp_table[static_cast<int64_t>(ti.b) * p.table_stride + ((e * p.r) >> 8)] : -2;
      }
    };
    int prev_b = -1, ns = 0;       // request switches so far
    int64_t it = 0;
    TileWalk walk(prefix, n_c, batch, t_lo);
    TileInfo tn{};
    int32_t phn[2] = {-2, -2};
    if (t_lo < t_hi) {
      tn = walk.at(t_lo);
      table_runs(tn, phn);
    }
    for (int64_t t = t_lo; t < t_hi && !*abort_flag; ++t, ++it) {
      const TileInfo ti = tn;
      const int32_t ph[2] = {phn[0], phn[1]};
      if (t + 1 < t_hi) {
        tn = walk.at(t + 1);
        table_runs(tn, phn);
      }
      if (ti.b != prev_b) {
        const int qs = ns & 1, k = ns >> 1;
        if (!mbar_wait(qempty(qs), (k & 1) ^ 1)) { *abort_flag = 1; break; }
        const uint8_t* img = qimage + static_cast<int64_t>(ti.b) * S.q_bytes;
        mbar_expect_tx(qfull(qs), S.q_bytes);
        for (uint32_t off = 0; off < S.q_bytes; off += 16384)
          bulk_g2s(sb + S.q + qs * qslot_bytes + off, img + off, S.q_bytes - off < 16384 ? S.q_bytes - off : 16384,
                   qfull(qs));
        prev_b = ti.b;
        ++ns;
      }
      // valid 64-entry runs (one pool block each); an unmapped block is flagged and skipped
      int mask = 0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (ph[j] >= 0 && ph[j] < p.comp_blocks) mask |= 1 << j;
        else if (ph[j] != -2) atomicOr(status, CKV_DEV_BAD_BLOCK);
      }
      const uint32_t nbox = static_cast<uint32_t>(__popc(mask));
      // entry scales into slot it % kMeta, index rows into stage it % kNS (the mask is written
      // before the arrive that releases the slot)
      const int m = static_cast<int>(it % kMeta);
      const int st = static_cast<int>(it % kNS);
      if (!mbar_wait(mempty(m), (static_cast<uint32_t>(it / kMeta) & 1) ^ 1) ||
          !mbar_wait(empty(st), (static_cast<uint32_t>(it / kNS) & 1) ^ 1)) {
        *abort_flag = 1;
        break;
      }
      meta_mask[m] = mask;
      mbar_expect_tx(mfull(m), nbox * (kBoxRows * 4));
      mbar_expect_tx(full(st), nbox * (kBoxRows * DI));
      const uint32_t dst = sb + S.a + st * S.stage_bytes;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (!(mask >> j & 1)) continue;
        const int64_t row = static_cast<int64_t>(ph[j]) * p.epb + ((ti.e0 + kBoxRows * j) & (p.epb - 1));
        bulk_g2s(sb + S.meta + m * 512 + j * (kBoxRows * 4), ip.scales + row, kBoxRows * 4, mfull(m));
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(dst + c * (kTile * 128) + j * (kBoxRows * 128), &rows_map, 128 * c, static_cast<int>(row),
                      full(st));
      }
    }
    // nothing may land in shared memory after the CTA exits: wait for the last loads of every
    // stage, scale slot and query slot (already complete unless a wait above gave up)
    for (int64_t j = it > kNS ? it - kNS : 0; j < it; ++j)
      if (!mbar_wait(full(static_cast<int>(j % kNS)), static_cast<uint32_t>(j / kNS) & 1)) *abort_flag = 1;
    for (int64_t j = it > kMeta ? it - kMeta : 0; j < it; ++j)
      if (!mbar_wait(mfull(static_cast<int>(j % kMeta)), static_cast<uint32_t>(j / kMeta) & 1)) *abort_flag = 1;
    for (int j = ns > 2 ? ns - 2 : 0; j < ns; ++j)
      if (!mbar_wait(qfull(j & 1), (j >> 1) & 1)) *abort_flag = 1;
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMAs: S^T[entries, heads] into accumulator it % 2
    int prev_b = -1, ns = 0, qs = 0;
    int64_t it = 0;
    bool issued = false;
    TileWalk walk(prefix, n_c, batch, t_lo);
    for (int64_t t = t_lo; t < t_hi && !*abort_flag; ++t, ++it) {
      const TileInfo ti = walk.at(t);
      if (ti.b != prev_b) {
        qs = ns & 1;
        if (!mbar_wait(qfull(qs), (ns >> 1) & 1)) { *abort_flag = 1; break; }
        prev_b = ti.b;
        ++ns;
      }
      const int st = static_cast<int>(it % kNS);
      if (!mbar_wait(full(st), static_cast<uint32_t>(it / kNS) & 1)) { *abort_flag = 1; break; }
      const int acc = static_cast<int>(it & 1);
      if (!mbar_wait(tempty(acc), (static_cast<uint32_t>(it >> 1) & 1) ^ 1)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t a0 = sb + S.a + st * S.stage_bytes;
      const uint32_t b0 = sb + S.q + qs * qslot_bytes;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_e4m3(tmem + static_cast<uint32_t>(acc) * (tmem_cols / 2), sdesc_sw128(a0 + c * (kTile * 128) + ks * 32),
                   sdesc_sw128(b0 + c * (H * 128) + ks * 32), idesc, (c | ks) != 0);
      }
      mma_commit(empty(st));
      mma_commit(tfull(acc));
      issued = true;
      const bool last_of_request = t + 1 == t_hi || prefix[ti.b + 1] <= t + 1;
      if (last_of_request) mma_commit(qempty(qs));
    }
    if (issued) {  // every MMA issued has completed before the tensor memory is released
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) *abort_flag = 1;
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: entry j = 32 (warp % 4) + lane = TMEM lane; score, digit count.
    //                  Group eg takes the CTA's tiles it = eg, eg + G, ...
    const int q4 = warp & 3;
    const int eg = (warp - 4) >> 2;
    const int j = q4 * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    float* w_warp = w_sh + (warp - 4) * 2 * H;  // this warp's two weight slots
    int prev_b = -1, ns = 0, qs = 0;
    int64_t it = eg;
    TileWalk walk(prefix, n_c, batch, t_lo);
    for (int64_t t = t_lo + eg; t < t_hi && !*abort_flag; t += G, it += G) {
      const TileInfo ti = walk.at(t);
      if (ti.b != prev_b) {  // this request's scaled head weights into the warp's slot qs
        qs = ns & 1;
        __syncwarp();
        for (int h = lane; h < H; h += 32) w_warp[qs * H + h] = wq[static_cast<int64_t>(ti.b) * H + h];
        __syncwarp();
        prev_b = ti.b;
        ++ns;
      }
      // the entry's scale from the scale ring (0 for an absent entry or an unmapped block)
      const int m = static_cast<int>(it % kMeta);
      const bool mok = __all_sync(0xffffffffu, mbar_wait(mfull(m), static_cast<uint32_t>(it / kMeta) & 1));
      const float scale = mok && j < ti.n_valid && (meta_mask[m] >> (j / kBoxRows) & 1) ? meta_sc[m * 128 + j] : 0.f;
      bar_arrive(mempty(m));
      if (!mok) {
        *abort_flag = 1;
        break;
      }
      const int acc = static_cast<int>(it & 1);
      // one decision per warp, so that the warp's TMEM loads stay converged
      const bool ok = __all_sync(0xffffffffu, mbar_wait(tfull(acc), static_cast<uint32_t>(it >> 1) & 1));
      if (!ok) *abort_flag = 1;
      tc_fence_after();
      float sum = 0.f;
      if (ok) {
        const uint32_t taddr = tmem + lane_base + static_cast<uint32_t>(acc) * (tmem_cols / 2);
        const float4* wv = reinterpret_cast<const float4*>(w_warp + qs * H);
        for (int g = 0; g < H; g += 16) {  // H is a multiple of 16
          uint32_t v[16];
          tmem_ld16(taddr + g, v);
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            const float4 wk = wv[(g + k) >> 2];
            sum = fmaf(wk.x, fmaxf(__uint_as_float(v[k]), 0.f), sum);
            sum = fmaf(wk.y, fmaxf(__uint_as_float(v[k + 1]), 0.f), sum);
            sum = fmaf(wk.z, fmaxf(__uint_as_float(v[k + 2]), 0.f), sum);
            sum = fmaf(wk.w, fmaxf(__uint_as_float(v[k + 3]), 0.f), sum);
          }
        }
      }
      tc_fence_before();
      bar_arrive(tempty(acc));
      if (!ok) break;
      const bool writer = j < ti.n_valid;
      uint32_t bin = 0xffffffffu - lane;
      if (writer) {
        const float s = scale > 0.f ? sum * scale : 0.f;
        scores[static_cast<int64_t>(ti.b) * stride + ti.e0 + j] = s;
        bin = f32_order_key(s) >> 21;
      }
      const uint32_t same = __match_any_sync(0xffffffffu, bin);
      if (writer && lane == __ffs(same) - 1)
        atomicAdd(ws.hist + static_cast<int64_t>(ti.b) * kHistBins + bin, static_cast<uint32_t>(__popc(same)));
    }
  }
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicOr(status, CKV_DEV_TIMEOUT);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// cuTensorMapEncodeTiled from the driver, looked up once (no link-time dependency on libcuda)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

template <int DI>
cudaError_t launch_mh_score(const LayerParams& p, const IndexParams& ip, int batch, int max_seq_len,
                            const IndexerWs& ws, const uint8_t* qimage, const float* wq, float* scores,
                            int64_t stride, uint32_t* status, cudaStream_t stream) {
  // the index rows as a 2-D tensor [pool rows][d_I] of bytes, loaded in boxes of 64 rows x 128
  // bytes with the 128-byte swizzle of the MMA operand
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(DI), static_cast<cuuint64_t>(p.comp_blocks) * p.epb};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(DI)};
  const cuuint32_t box[2] = {128, kBoxRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ip.codes, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // Two epilogue groups while the grid gets few tiles per CTA (per 256 K-token request and below:
  // 32K 14.1 -> 13.2 us, 256K 20.1 -> 18.2 us per launch); one group and 3 CTAs per SM for long
  // streams (1M: 39.6 against 43.0 us)
  const int64_t tiles = static_cast<int64_t>(batch) * ((static_cast<int64_t>(max_seq_len) / p.r + kTile - 1) / kTile);
  const int groups = tiles < static_cast<int64_t>(sm_count()) * 3 * 8 ? 2 : 1;
  const MhSmem S(ip.heads, DI, groups);
  auto kern = groups == 2 ? mh_score_kernel<DI, 2> : mh_score_kernel<DI, 1>;
  const uint32_t cols = 2 * ip.heads <= 32 ? 32u : 2 * ip.heads <= 64 ? 64u : 2 * ip.heads <= 128 ? 128u : 256u;
  const int smem = static_cast<int>(S.end_fixed + sizeof(int32_t) * (2 * batch + 1)) + 1024;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // CTAs resident per SM: by shared memory (228 KB per SM, 1 KB reserved per CTA), by tensor
  // memory (512 columns) and by registers; a persistent grid of that many per SM
  int per_sm = 233472 / (smem + 1024);
  if (per_sm > static_cast<int>(512 / cols)) per_sm = static_cast<int>(512 / cols);
  if (per_sm > score_ctas(groups)) per_sm = score_ctas(groups);
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(sm_count()) * per_sm;
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  prof_begin(kProfScore, stream);
  e = launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(score_threads(groups)), static_cast<size_t>(smem), stream,
                    map, p, ip, batch, ws, qimage, wq, scores, stride, cols, status);
  prof_end(kProfScore, stream);
  return e;
}

}  // namespace

cudaError_t launch_index_append(const LayerParams& p, const IndexParams& ip, int batch, const int32_t* prev_len,
                                const int32_t* cu_new, int max_new, int max_seq_len, const float* k_new,
                                const float* logit_new, uint32_t* status, cudaStream_t stream) {
  IndexAppendArgs a{p, ip, prev_len, cu_new, max_seq_len, k_new, logit_new, status};
  // block 0 takes the first and the trailing group; the others the groups between, grid-strided
  const int64_t groups = static_cast<int64_t>(max_new) / p.r + 2;
  const int gx = static_cast<int>(groups < 512 ? groups : 512);
  return launch_kernel(index_append_kernel, dim3(gx, batch), dim3(kIdxAppendThreads), 0, stream, a);
}

cudaError_t launch_mh_indexer(const LayerParams& p, const IndexParams& ip, int batch, const int32_t* seq_len,
                              int max_seq_len, const float* q_index, const float* weights, int top_k,
                              int32_t* idx, int32_t* cnt, float* scores, const IndexerWs& ws,
                              uint8_t* qimage, uint32_t* status, cudaStream_t stream) {
  const int64_t stride = score_stride(p.r, max_seq_len);
  float* sc = scores ? scores : ws.scores;
  float* wq = reinterpret_cast<float*>(qimage + align_up(static_cast<size_t>(batch) * ip.heads * ip.dim, 256));
  const int head_groups = (ip.heads + kMhPrepThreads / 32 - 1) / (kMhPrepThreads / 32);
  cudaError_t e = launch_kernel(mh_prep_kernel, dim3(head_groups, batch), dim3(kMhPrepThreads), 0, stream, p, ip,
                                seq_len, max_seq_len, q_index, weights, ws, qimage, wq, status);
  if (e != cudaSuccess) return e;
  switch (ip.dim) {
    case 128: e = launch_mh_score<128>(p, ip, batch, max_seq_len, ws, qimage, wq, sc, stride, status, stream); break;
    case 256: e = launch_mh_score<256>(p, ip, batch, max_seq_len, ws, qimage, wq, sc, stride, status, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_topk(p, batch, max_seq_len, top_k, sc, stride, ws, idx, cnt, stream);
}

}  // namespace ckv

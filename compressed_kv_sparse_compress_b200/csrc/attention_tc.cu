// Tensor-core attention path (tcgen05, kind::f16, fp32 accumulation in tensor memory) for
// H = 64 query heads sharing one K=V vector of D = 512 (multi-query attention).
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": every head reads the same shared K=V vector, so the heads x keys
// contractions are dense matrix products; aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section
// "Vykon neprinesl jeden kernel": attention over an NVFP4 compressed cache.
//
// Orientation: keys are the MMA's M dimension (128 keys per tile) and heads its N dimension (64),
// so every MMA runs at M = 128:
//     S^T[keys, heads]  = X[keys, D]  . Q~^T[D, heads]        A = X   (K-major), B = Q~ (K-major)
//     O^T[D, heads]    += X^T[D, keys] . P^T[keys, heads]     A = X^T (MN-major), B = P (MN-major)
// One fp16 copy of the key tile X in shared memory (128-byte swizzled rows of 64 elements) is the
// K-major A operand of the first product and the MN-major A operand of the second. The cache is
// converted to fp16 while it is staged: bf16 and e2m1 x e4m3 values are exact in fp16 (|x| <
// 65504), FP8 window codes are exact and their per-token scale is applied to the logits and to
// P in fp32. Q~ (rotated query) is rounded to fp16 once. S^T (64 columns) and O^T (4 blocks of 64
// columns) live in tensor memory. The CTA has 32 warps, so that the gather of a tile's key rows
// has many loads in flight; for the softmax warp w owns the keys of TMEM lane quarter w%4 (one
// key per thread) and 8 heads; per-head maxima and sums are reduced across the keys with warp
// reduce-scatters. The running maximum is only raised when a tile's maximum exceeds it by more
// than 8 (then O^T is rescaled in tensor memory), so P <= e^8 stays well inside fp16.
//
// Each CTA handles `tiles_per_split` consecutive tiles of one request's key list and writes the
// same un-normalised partials (max, sum, output) as the CUDA-core path; the shared combine kernel
// merges the splits and applies the inverse rotation.

#include "ckv_internal.h"
#include "ckv_ptx.cuh"

namespace ckv {
namespace {

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kTile = 128;
constexpr int kThreads = 1024;  // 32 warps: many loads in flight per SM while staging
constexpr int kChunks = kD / 64;
constexpr uint32_t kXChunk = kTile * 128;        // bytes of one 64-element chunk of the tile
constexpr uint32_t kXBytes = kXChunk * kChunks;  // 128 KB
constexpr uint32_t kQChunk = kH * 128;
constexpr uint32_t kQBytes = kQChunk * kChunks;  // 64 KB
constexpr uint32_t kPBytes = kTile * kH * 2;     // 16 KB
constexpr uint32_t kSCol = 0;
constexpr uint32_t kOCol = 256;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescale = 8.0f;

// shared memory carve-up (byte offsets from a 1024-aligned base)
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffQ = kOffX + kXBytes;
constexpr uint32_t kOffP = kOffQ + kQBytes;          // also the rotary table in the prologue
constexpr uint32_t kOffRow = kOffP + kPBytes;        // int64[128] pool row (-1: absent key)
constexpr uint32_t kOffLs = kOffRow + 8 * kTile;     // float[128] logit factor per key
constexpr uint32_t kOffVs = kOffLs + 4 * kTile;      // float[128] value factor per key
constexpr uint32_t kOffWin = kOffVs + 4 * kTile;     // int[128]   1: window token
constexpr uint32_t kOffRed = kOffWin + 4 * kTile;    // float[4][64]
constexpr uint32_t kOffM = kOffRed + 4 * 4 * kH;     // float[64] running max
constexpr uint32_t kOffA = kOffM + 4 * kH;           // float[64] rescale factor of this tile
constexpr uint32_t kOffL = kOffA + 4 * kH;           // float[64] running sum
constexpr uint32_t kOffFlag = kOffL + 4 * kH;        // int[4]
constexpr uint32_t kOffBar = kOffFlag + 16;          // uint64 mbarrier: MMA completion
constexpr uint32_t kOffBarQ = kOffBar + 8;           // uint64 mbarrier: query bytes landed
constexpr uint32_t kOffTmem = kOffBarQ + 8;          // uint32 TMEM base
constexpr uint32_t kSmemUsed = kOffTmem + 8;
constexpr int kSmemBytes = static_cast<int>(kSmemUsed) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// ------------------------------------------------------------------------------------ PTX

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T, both described by shared-memory matrix descriptors
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on the mbarrier once every MMA issued so far by this thread has completed
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// shared-memory matrix descriptor: 128-byte swizzle, sm_100 descriptor version 1
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B, M = 128, N = 64
constexpr uint32_t kIdescS = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 15) | (1u << 16);  // A and B MN-major

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t half2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

__device__ __forceinline__ uint32_t pack_f32x2(float a, float b) {
  return half2_bits(__floats2half2_rn(a, b));
}

__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu), __NV_E4M3);
  return half2_bits(__half2(r));
}

// Reduction of N (64 or 32) per-thread values across a warp; afterwards t[0 .. N/32) hold the
// reduction of entries (N/32)*lane .. (N/32)*lane + N/32 - 1.
template <int N, bool kMax>
__device__ __forceinline__ void reduce_scatter(float (&t)[N], int lane) {
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int o = 16 >> s;
    const int half = N >> (s + 1);
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? t[i] : t[i + half];
      const float keep = upper ? t[i + half] : t[i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, o);
      t[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

// Reduction of one value per (head of 8, lane) over the warp's 32 lanes: three reduce-scatter
// stages, then two butterfly stages; lane l returns the reduction of entry l >> 2.
template <bool kMax>
__device__ __forceinline__ float warp_reduce8(float (&t)[8], int lane) {
  reduce_scatter<8, kMax>(t, lane);
  float v = t[0];
#pragma unroll
  for (int o = 2; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, v, o);
    v = kMax ? fmaxf(v, x) : v + x;
  }
  return v;
}

// raw bytes of one 8-element granule of a key, loaded before conversion
struct Raw {
  uint4 a, b;
  uint32_t s;
};

template <int CT, int WT>
__device__ __forceinline__ Raw load_granule(const LayerParams& p, int64_t row, bool win, int g) {
  Raw r;
  r.a = make_uint4(0, 0, 0, 0);
  r.b = make_uint4(0, 0, 0, 0);
  r.s = 0;
  if (row < 0) return r;
  if (win) {
    const uint8_t* base = p.win_codes + row * p.win_row_bytes;
    if constexpr (WT == CKV_FP8_E4M3) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(base) + g);
      r.a.x = v.x;
      r.a.y = v.y;
    } else {
      r.a = __ldg(reinterpret_cast<const uint4*>(base) + 2 * g);
      r.b = __ldg(reinterpret_cast<const uint4*>(base) + 2 * g + 1);
    }
    return r;
  }
  const uint8_t* base = p.comp_codes + row * p.comp_row_bytes;
  if constexpr (CT == CKV_BF16) {
    r.a = __ldg(reinterpret_cast<const uint4*>(base) + g);
  } else if constexpr (CT == CKV_NVFP4) {
    r.a.x = __ldg(reinterpret_cast<const uint32_t*>(base) + g);
    r.s = __ldg(p.comp_scales + row * (kD / 16) + (g >> 1));
  } else {
    r.a = __ldg(reinterpret_cast<const uint4*>(base) + 2 * g);
    r.b = __ldg(reinterpret_cast<const uint4*>(base) + 2 * g + 1);
  }
  return r;
}

template <int CT, int WT>
__device__ __forceinline__ uint4 convert_granule(const Raw& r, bool win) {
  if (win) {
    if constexpr (WT == CKV_FP8_E4M3) {
      return make_uint4(e4m3x2_to_h2(r.a.x), e4m3x2_to_h2(r.a.x >> 16), e4m3x2_to_h2(r.a.y),
                        e4m3x2_to_h2(r.a.y >> 16));
    } else {
      return make_uint4(pack_f32x2(__uint_as_float(r.a.x), __uint_as_float(r.a.y)),
                        pack_f32x2(__uint_as_float(r.a.z), __uint_as_float(r.a.w)),
                        pack_f32x2(__uint_as_float(r.b.x), __uint_as_float(r.b.y)),
                        pack_f32x2(__uint_as_float(r.b.z), __uint_as_float(r.b.w)));
    }
  }
  if constexpr (CT == CKV_BF16) {
    const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = pack_f32x2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    return make_uint4(o[0], o[1], o[2], o[3]);
  } else if constexpr (CT == CKV_NVFP4) {
    const __half s = __half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(r.s), __NV_E4M3));
    const __half2 s2 = __half2(s, s);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = half2_bits(__hmul2(e2m1x2_to_half2(static_cast<uint8_t>(r.a.x >> (8 * i))), s2));
    return make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    return make_uint4(pack_f32x2(__uint_as_float(r.a.x), __uint_as_float(r.a.y)),
                      pack_f32x2(__uint_as_float(r.a.z), __uint_as_float(r.a.w)),
                      pack_f32x2(__uint_as_float(r.b.x), __uint_as_float(r.b.y)),
                      pack_f32x2(__uint_as_float(r.b.z), __uint_as_float(r.b.w)));
  }
}

// byte offset of 16-byte granule g of row `row` in a 128-byte-swizzled operand made of chunks
// of `chunk_bytes` (64 elements per row and chunk)
__device__ __forceinline__ uint32_t swz(uint32_t chunk_bytes, int row, int g) {
  return static_cast<uint32_t>(g >> 3) * chunk_bytes + static_cast<uint32_t>(row) * 128u +
         (static_cast<uint32_t>((g & 7) ^ (row & 7)) << 4);
}

// Pool row, window flag and factors of the keys of one tile (threads 0..127, one key each):
// the logit factor is sm_scale times the window token's FP8 scale, the value factor that scale.
template <int WT>
__device__ __forceinline__ void key_meta(const LayerParams& p, int b, int L, const int32_t* idx,
                                         int idx_stride, int64_t n_c, int64_t n_sel, int64_t n_win,
                                         int64_t k_first, int64_t k_end, int64_t* key_row,
                                         int* key_win, float* key_vs, float* key_ls,
                                         uint32_t* status) {
  const int tid = threadIdx.x;
  if (tid >= kTile) return;
  const int64_t kk = k_first + tid;
  int64_t row = -1;
  int win = 0;
  float vs = 1.f;
  if (kk < k_end) {
    if (kk < n_sel) {
      const int64_t ent = idx ? idx[static_cast<int64_t>(b) * idx_stride + kk] : kk;
      if (ent < 0 || ent >= n_c) atomicOr(status, CKV_DEV_BAD_INDEX);
      else row = comp_row(p, b, ent, status);
    } else {
      win = 1;
      row = win_row(p, b, L - n_win + (kk - n_sel), status);
      if (row >= 0 && WT == CKV_FP8_E4M3) vs = p.win_scales[row];
    }
  }
  key_row[tid] = row;
  key_win[tid] = win;
  key_vs[tid] = vs;
  key_ls[tid] = p.sm_scale * vs;
}

// ------------------------------------------------------------------------------------ kernel

template <int CT, int WT>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const float* q, const int32_t* idx,
    const int32_t* cnt, int idx_stride, AttnWs ws, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  int64_t* key_row = reinterpret_cast<int64_t*>(base + kOffRow);
  float* key_ls = reinterpret_cast<float*>(base + kOffLs);
  float* key_vs = reinterpret_cast<float*>(base + kOffVs);
  int* key_win = reinterpret_cast<int*>(base + kOffWin);
  float* red = reinterpret_cast<float*>(base + kOffRed);
  float* m_run = reinterpret_cast<float*>(base + kOffM);
  float* alpha = reinterpret_cast<float*>(base + kOffA);
  float* l_run = reinterpret_cast<float*>(base + kOffL);
  int* flags = reinterpret_cast<int*>(base + kOffFlag);
  const uint32_t bar = sb + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffTmem);

  const int b = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bar_q = sb + kOffBarQ;

  // ---- set-up that reads no global memory, before waiting for the previous kernel: barriers,
  //      running max and sum, tensor memory
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar_q, 1);
    fence_proxy_async();
    flags[0] = flags[1] = 0;
  }
  if (tid < kH) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  if (warp == 0) tmem_alloc(sb + kOffTmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto release = [&]() {   // every exit after the allocation (block-uniform)
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  };
  griddep_wait();
  griddep_launch();

  const int L = seq_len[b];
  if (L < 1 || L > max_seq_len) {  // flagged by the combine
    release();
    return;
  }
  const int64_t n_c = L / p.r;
  const int64_t n_sel = idx ? min(static_cast<int64_t>(max(cnt[b], 0)), static_cast<int64_t>(idx_stride)) : n_c;
  const int64_t n_win = min(p.W, L);
  const int64_t n_keys = n_sel + n_win;
  const int64_t k_begin = static_cast<int64_t>(split) * ws.keys_per_split;
  if (k_begin >= n_keys) {
    release();
    return;
  }
  const int64_t k_end = min(n_keys, k_begin + ws.keys_per_split);
  const int n_tiles = static_cast<int>((k_end - k_begin + kTile - 1) / kTile);

  // ---- the prepared query image (64 KB, written per request by the prep kernel) is bulk-copied
  //      into the Q region while the keys of tile 0 are resolved and staged
  if (tid == 0) {
    const uint8_t* img = ws.qimage + static_cast<int64_t>(b) * kQBytes;
    constexpr uint32_t kPiece = 16384;
    mbar_expect_tx(bar_q, kQBytes);
#pragma unroll 1
    for (uint32_t off = 0; off < kQBytes; off += kPiece) bulk_g2s(sb + kOffQ + off, img + off, kPiece, bar_q);
  }
  key_meta<WT>(p, b, L, idx, idx_stride, n_c, n_sel, n_win, k_begin, k_end, key_row, key_win, key_vs,
               key_ls, status);
  __syncthreads();
  uint32_t phase = 0;
  bool ok = true;
  bool q_ready = false;

  for (int tile = 0; tile < n_tiles && ok; ++tile) {
    const int64_t k_first = k_begin + static_cast<int64_t>(tile) * kTile;
    const int n_valid = static_cast<int>(min(static_cast<int64_t>(kTile), k_end - k_first));
    if (tile > 0) {
      key_meta<WT>(p, b, L, idx, idx_stride, n_c, n_sel, n_win, k_begin + static_cast<int64_t>(tile) * kTile,
                   k_end, key_row, key_win, key_vs, key_ls, status);
      __syncthreads();
    }

    // ---- stage the tile as fp16 (absent keys are zero rows): warp w converts kpw consecutive
    //      keys (4 of a full tile, 2 when it holds at most 64 keys), lane l the granules l and l+32
    //      of each (the key's row and kind read once per key), all of them in flight at once. Rows
    //      that are not staged hold stale or uninitialised values: their logits are masked and no
    //      PV step reads them.
    {
      constexpr int kB = (CT == CKV_F32 || WT == CKV_F32) ? 2 : 4;  // fp32 granules are 32 bytes
      const int kpw = n_valid > kTile / 2 ? 4 : 2;
#pragma unroll
      for (int u0 = 0; u0 < 4; u0 += kB) {
        if (u0 >= kpw) break;
        Raw r[kB][2];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (u0 + u < kpw) {
            const int j = kpw * warp + u0 + u;
            const int64_t row = key_row[j];
            const bool win = key_win[j] != 0;
            r[u][0] = load_granule<CT, WT>(p, row, win, lane);
            r[u][1] = load_granule<CT, WT>(p, row, win, lane + 32);
          }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (u0 + u < kpw) {
            const int j = kpw * warp + u0 + u;
            const bool win = key_win[j] != 0;
            st_shared_v4(sb + kOffX + swz(kXChunk, j, lane), convert_granule<CT, WT>(r[u][0], win));
            st_shared_v4(sb + kOffX + swz(kXChunk, j, lane + 32), convert_granule<CT, WT>(r[u][1], win));
          }
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    if (!q_ready) {   // the query image must have landed before the first MMA reads it
      ok = __syncthreads_and(mbar_wait(bar_q, 0)) != 0;
      q_ready = true;
      if (!ok) break;
    }
    __syncthreads();

    // ---- S^T = X . Q~^T
    if (tid == 128) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a = sdesc(sb + kOffX + c * kXChunk + ks * 32, 16, 1024);
          const uint64_t bq = sdesc(sb + kOffQ + c * kQChunk + ks * 32, 16, 1024);
          mma_f16(tmem + kSCol, a, bq, kIdescS, (c | ks) != 0);
        }
      }
      mma_commit(bar);
    }
    ok = __syncthreads_and(mbar_wait(bar, phase)) != 0;  // uniform across the CTA
    phase ^= 1;
    tc_fence_after();
    if (!ok) break;

    // ---- softmax over the tile's keys: key j = TMEM lane; warp w reads the lanes of quarter w%4
    //      and the 8 heads of group w/4
    {
      const int q4 = warp & 3, hg = warp >> 2;
      const int j = q4 * 32 + lane;
      const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
      uint32_t raw[8];
      tmem_ld8(tmem + lane_base + kSCol + 8 * hg, raw);
      const float f = key_ls[j];
      const bool valid = key_row[j] >= 0;
      float sv[8], t[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        sv[h] = valid ? __uint_as_float(raw[h]) * f : -INFINITY;
        t[h] = sv[h];
      }
      const float mx = warp_reduce8<true>(t, lane);
      if ((lane & 3) == 0) red[q4 * kH + 8 * hg + (lane >> 2)] = mx;
      __syncthreads();
      if (tid < kH) {
        const float mt = fmaxf(fmaxf(red[tid], red[kH + tid]), fmaxf(red[2 * kH + tid], red[3 * kH + tid]));
        const float mo = m_run[tid];
        float mn = mo, al = 1.f;
        if (mt > mo + kRescale || (mo == -INFINITY && mt > -INFINITY)) {
          mn = mt;
          al = mo == -INFINITY ? 0.f : __expf(mo - mn);
          if (mo != -INFINITY) flags[0] = 1;
        }
        m_run[tid] = mn;
        alpha[tid] = al;
      }
      __syncthreads();
      const float vs = key_vs[j];
      uint32_t packed[4];
#pragma unroll
      for (int h = 0; h < 8; h += 2) {
        const float m0 = m_run[8 * hg + h], m1 = m_run[8 * hg + h + 1];
        const float p0 = m0 == -INFINITY ? 0.f : __expf(sv[h] - m0);
        const float p1 = m1 == -INFINITY ? 0.f : __expf(sv[h + 1] - m1);
        t[h] = p0;
        t[h + 1] = p1;
        packed[h >> 1] = pack_f32x2(p0 * vs, p1 * vs);
      }
      st_shared_v4(sb + kOffP + static_cast<uint32_t>(j) * 128u + (static_cast<uint32_t>(hg ^ (j & 7)) << 4),
                   make_uint4(packed[0], packed[1], packed[2], packed[3]));
      const float sm = warp_reduce8<false>(t, lane);
      if ((lane & 3) == 0) red[q4 * kH + 8 * hg + (lane >> 2)] = sm;
      __syncthreads();
      if (tid < kH)
        l_run[tid] = l_run[tid] * alpha[tid] + ((red[tid] + red[kH + tid]) + (red[2 * kH + tid] + red[3 * kH + tid]));
      // rescale the output accumulated so far where the running max was raised
      if (tile > 0 && flags[0]) {
#pragma unroll 1
        for (int m = 0; m < 4; ++m) {
          const uint32_t ta = tmem + lane_base + kOCol + 64 * m + 8 * hg;
          uint32_t o[8];
          tmem_ld8(ta, o);
#pragma unroll
          for (int h = 0; h < 8; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[8 * hg + h]);
          tmem_st8(ta, o);
        }
      }
      fence_proxy_async();
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) flags[0] = 0;

    // ---- O^T += X^T . P^T
    if (tid == 128) {
      tc_fence_after();
#pragma unroll 1
      for (int kk = 0; kk < (n_valid + 15) / 16; ++kk) {   // consecutive MMAs go to different accumulators
        const uint64_t bp = sdesc(sb + kOffP + kk * 2048, 8192, 1024);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint64_t a = sdesc(sb + kOffX + 2 * m * kXChunk + kk * 2048, kXChunk, 1024);
          mma_f16(tmem + kOCol + 64 * m, a, bp, kIdescPV, (tile > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(bar);
    }
    ok = __syncthreads_and(mbar_wait(bar, phase)) != 0;
    phase ^= 1;
    tc_fence_after();
  }

  // ---- partial outputs: O^T lane = dim, column = head (warp w: lane quarter w%4, heads of
  //      group w/4). Each head's row is stored as fp16 after division by a power of two 2^e,
  //      e = (exponent of the row's max |o|) - 15 (at least -126), so that every value lies below
  //      2^15 in magnitude with a relative step of 2^-11 of the row's max; e goes to part_sc.
  if (ok) {
    const int q4 = warp & 3, hg = warp >> 2;
    const int64_t slot = (static_cast<int64_t>(b) * ws.splits + split) * kH;
    uint32_t o[4][8];
#pragma unroll
    for (int m = 0; m < 4; ++m)
      tmem_ld8(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + kOCol + 64 * m + 8 * hg, o[m]);
    float t[8];
#pragma unroll
    for (int h = 0; h < 8; ++h)
      t[h] = fmaxf(fmaxf(fabsf(__uint_as_float(o[0][h])), fabsf(__uint_as_float(o[1][h]))),
                   fmaxf(fabsf(__uint_as_float(o[2][h])), fabsf(__uint_as_float(o[3][h]))));
    const float amax_w = warp_reduce8<true>(t, lane);
    if ((lane & 3) == 0) red[q4 * kH + 8 * hg + (lane >> 2)] = amax_w;
    __syncthreads();
    if (tid < kH) {
      const float amax = fmaxf(fmaxf(red[tid], red[kH + tid]), fmaxf(red[2 * kH + tid], red[3 * kH + tid]));
      int ex = 0;
      float sc = 1.f;
      if (amax > 0.f && amax <= 3.4e38f) {   // finite, non-zero
        frexpf(amax, &ex);                    // amax = f * 2^ex, f in [0.5, 1)
        sc = ldexpf(1.f, ex - 15 > -126 ? ex - 15 : -126);
      }
      alpha[tid] = sc;
      ws.part_sc[slot + tid] = sc;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float inv = 1.f / alpha[8 * hg + h];   // exact: a power of two
      __half* dst = reinterpret_cast<__half*>(ws.part_h) + (slot + 8 * hg + h) * kD + 32 * q4 + lane;
#pragma unroll
      for (int m = 0; m < 4; ++m) dst[128 * m] = __float2half_rn(__uint_as_float(o[m][h]) * inv);
    }
    if (tid < kH) reinterpret_cast<float2*>(ws.part_ml)[slot + tid] = make_float2(m_run[tid], l_run[tid]);
  }
  if (!ok) {
    if (tid == 0) atomicOr(status, CKV_DEV_TIMEOUT);
    const int64_t slot = (static_cast<int64_t>(b) * ws.splits + split) * kH;
    if (tid < kH) reinterpret_cast<float2*>(ws.part_ml)[slot + tid] = make_float2(-INFINITY, 0.f);
  }
  release();
}

template <int CT, int WT>
cudaError_t launch_tc(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                      const float* q, const int32_t* idx, const int32_t* cnt, int idx_stride,
                      const AttnWs& ws, uint32_t* status, cudaStream_t stream) {
  auto kern = attn_tc_kernel<CT, WT>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(ws.splits, batch);
  return launch_kernel(kern, grid, dim3(kThreads), kSmemBytes, stream, p, seq_len, max_seq_len, q, idx,
                       cnt, idx_stride, ws, status);
}

}  // namespace

// fp32 caches stay on the CUDA-core path: their values are neither exact in fp16 nor inside its
// range, and fp32 arithmetic attends them as stored
bool attention_tc_supported(const LayerParams& p) {
  return p.H == kH && p.D == kD && (p.comp_dtype == CKV_BF16 || p.comp_dtype == CKV_NVFP4) &&
         p.win_dtype == CKV_FP8_E4M3;
}

int attention_tc_tiles_per_split(int batch, int64_t max_keys) {
  const int64_t tiles = static_cast<int64_t>(batch) * ((max_keys + kTile - 1) / kTile);
  const int64_t cap = 4 * static_cast<int64_t>(sm_count());
  int64_t t = tiles > cap ? (tiles + cap - 1) / cap : 1;
  return static_cast<int>(t < 8 ? t : 8);
}

int attention_tc_keys_per_split(int batch, int64_t max_keys) {
  // half tiles (64 keys; the MMAs still run at M = 128 over the staged half) while they fit one
  // wave: twice the CTAs, each staging half the rows
  const int64_t halves = static_cast<int64_t>(batch) * ((max_keys + kTile / 2 - 1) / (kTile / 2));
  if (halves <= sm_count()) return kTile / 2;
  return kTile * attention_tc_tiles_per_split(batch, max_keys);
}

cudaError_t launch_attention_tc(const LayerParams& p, int batch, const int32_t* seq_len,
                                int max_seq_len, const float* q, const int32_t* idx,
                                const int32_t* cnt, int idx_stride, const AttnWs& ws,
                                uint32_t* status, cudaStream_t stream) {
#define CKV_TC(CT, WT) \
  if (p.comp_dtype == CT && p.win_dtype == WT) \
    return launch_tc<CT, WT>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream);
  CKV_TC(CKV_BF16, CKV_FP8_E4M3)
  CKV_TC(CKV_NVFP4, CKV_FP8_E4M3)
#undef CKV_TC
  return cudaErrorInvalidValue;
}

}  // namespace ckv

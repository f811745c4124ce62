// Scoring of an NVFP4 compressed cache on the tensor cores (the head-averaged indexer, D = 512).
//
// aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section "Vykon neprinesl jeden kernel": the
// "Sparse MQA logits" kernel scores only the candidate positions, and attention reads an NVFP4
// compressed cache. The score of entry j is s_j = q_bar . k_j (q_bar: the head-averaged, rotated
// and scaled query), with k_j = e2m1 code x e4m3 scale of its 16-element block.
//
// On CUDA cores every element costs a conversion chain (e2m1 -> f16 -> f32) and an fp32 FMA, which
// bounds that kernel by its ALU pipe. Here each element is decoded once into an fp16 operand
// image (e2m1 x e4m3 is exact in fp16) and the dot products run as one contraction per tile:
//     D[entries, 16] = K'[entries, D] . B[16, D]^T      (tcgen05 kind::f16, fp32 accumulation)
// with B's row 0 the fp16 rounding of q_bar * 2^sh, row 1 the fp16 rounding of the remainder and
// rows 2..15 zero (sh puts |q_bar|'s largest element in [2^8, 2^9)), so s_j = (D[j,0] + D[j,1])
// 2^-sh carries q_bar to about 2^-22 relative.
//
// Warp roles (512 threads, one CTA per SM, persistent over a contiguous range of the flattened
// (request, 128-entry tile) list):
//   warp 0 lane 0   producer: per tile, for each 64-entry run (one pool block holds >= 64 entries
//                   at ratio <= 4) TMA loads of the run's codes (two boxes of 64 rows x 128 bytes,
//                   128-byte swizzle) and a bulk copy of its scales into one of 3 raw stages
//   warp 1 lane 0   MMA issuer: per 64-dim chunk, 4 MMAs (M = 128, N = 16, K = 16) into one of two
//                   accumulators (16 columns of tensor memory each)
//   warp 2          owns the tensor memory
//   warps 4..7      epilogue: one entry per thread (TMEM lane), score = (D0 + D1) 2^-sh, stored
//                   with the count of its first radix digit, as the CUDA-core score kernel does
//   warps 8..15     decoders: thread t takes entry t/2 and half t%2 of every 64-dim chunk (16 bytes
//                   of codes, two block scales) and writes 32 fp16 values into one of 4 chunk
//                   slots; at every request switch they build that request's B image
// Every wait is bounded; the first role to give up raises an abort flag, the producer waits for its
// copies in flight, the MMA issuer for its last commit, and only then is the tensor memory freed
// and CKV_DEV_TIMEOUT set.

#include <cuda.h>

#include "ckv_internal.h"
#include "ckv_ptx.cuh"

namespace ckv {
namespace {

constexpr int kD = 512;
constexpr int kTile = 128;       // entries per tile (MMA M)
constexpr int kRun = 64;         // entries per TMA box (rows)
constexpr int kChunks = kD / 64; // 64-dim chunks
constexpr int kRawStages = 3;
constexpr int kASlots = 4;
constexpr int kThreads = 512;
constexpr int kFirstDecWarp = 8;
constexpr int kDecThreads = 256;
constexpr uint32_t kRawCodes = 2 * 2 * kRun * 128;      // 32 KB: [run][half][64 rows][128 B]
constexpr uint32_t kRawScales = kTile * 32;             // 4 KB: [128 entries][32 B]
constexpr uint32_t kRawStage = kRawCodes + kRawScales;  // 36 KB
constexpr uint32_t kASlot = kTile * 128;                // 16 KB: 128 rows x 64 dims fp16
constexpr uint32_t kBChunk = 16 * 128;                  // 2 KB: 16 rows x 64 dims fp16
constexpr uint32_t kBSlot = kBChunk * kChunks;          // 16 KB

constexpr uint32_t kOffRaw = 0;
constexpr uint32_t kOffA = kOffRaw + kRawStages * kRawStage;
constexpr uint32_t kOffB = kOffA + kASlots * kASlot;
constexpr uint32_t kOffRed = kOffB + 2 * kBSlot;        // float[8]: max reductions
constexpr uint32_t kOffBar = kOffRed + 64;
// raw_full[3], raw_empty[3], a_full[4], a_empty[4], b_full[2], b_empty[2], d_full[2], d_empty[2], drain
constexpr int kNumBars = 23;
constexpr uint32_t kOffTmem = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffFlag = kOffTmem + 8;
constexpr uint32_t kOffPrefix = kOffFlag + 8;           // int32[batch + 1], then n_c [batch]
static_assert(kOffRaw % 1024 == 0 && kRawStage % 1024 == 0 && kOffA % 1024 == 0 && kOffB % 1024 == 0,
              "swizzled operands start on 1024-byte boundaries");

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

// D[tmem] (+)= A[smem] . B[smem]^T, fp16 operands, fp32 accumulation
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// K-major operand with 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;          // leading byte offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;  // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;          // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;          // 128-byte swizzle
  return d;
}

// fp32 accumulator, fp16 A and B (both K-major), M = 128, N = 16
constexpr uint32_t kIdesc = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t half2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// bounded wait (polls that suspend the thread, ckv_ptx.cuh) that also gives up once another role
// has raised the abort flag
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t phase, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait_sleep(bar, phase, kWaitSuspendNs)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

// 2^e as a float for -126 <= e <= 127
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// the shift that puts a largest magnitude with float bits `mb` into [2^8, 2^9) (0 for zero)
__device__ __forceinline__ int norm_shift(uint32_t mb) {
  if (mb == 0u) return 0;
  return max(-126, min(126, 8 - (static_cast<int>(mb >> 23) - 127)));
}

// Tile t of the flattened (request, tile) list: request b, first entry e0, valid entries n_valid.
struct TileInfo {
  int b;
  int64_t e0;
  int n_valid;
};

// Walks a CTA's consecutive tiles (binary search for the first, then forward only).
struct TileWalk {
  const int32_t* prefix;
  const int32_t* n_c;
  int b;
  __device__ TileWalk(const int32_t* pf, const int32_t* nc, int batch, int64_t t0) : prefix(pf), n_c(nc) {
    int lo = 0, hi = batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= t0) lo = mid; else hi = mid;
    }
    b = lo;
  }
  __device__ __forceinline__ TileInfo at(int64_t t) {
    while (prefix[b + 1] <= t) ++b;
    TileInfo ti;
    ti.b = b;
    ti.e0 = (t - prefix[b]) * kTile;
    ti.n_valid = static_cast<int>(min(static_cast<int64_t>(kTile), static_cast<int64_t>(n_c[b]) - ti.e0));
    return ti;
  }
};

// the pool block holding entry e of request b, or -1 (flagged) when unmapped
__device__ __forceinline__ int32_t entry_block(const LayerParams& p, int b, int64_t e, uint32_t* status, bool flag) {
  const int32_t phys = p.comp_table[static_cast<int64_t>(b) * p.table_stride + ((e * p.r) >> 8)];
  if (phys < 0 || phys >= p.comp_blocks) {
    if (flag) atomicOr(status, CKV_DEV_BAD_BLOCK);
    return -1;
  }
  return phys;
}

// the power-of-two shift of a request's q_bar, computed by one whole warp over all D dims (every
// warp that asks gets the same value, with no barrier between warps)
__device__ __forceinline__ int qbar_shift(const float* qb, int lane) {
  uint32_t mb = 0;
#pragma unroll
  for (int d = lane; d < kD; d += 32) mb = max(mb, __float_as_uint(qb[d]) & 0x7fffffffu);
  return norm_shift(__reduce_max_sync(0xffffffffu, mb));
}

__global__ void __launch_bounds__(kThreads, 1) score_nvfp4_tc_kernel(const __grid_constant__ CUtensorMap codes_map,
                                                                      LayerParams p, int batch, IndexerWs ws,
                                                                      float* scores, int64_t stride, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffFlag);
  int32_t* prefix = reinterpret_cast<int32_t*>(base + kOffPrefix);
  int32_t* n_c = prefix + batch + 1;
  const uint32_t bar0 = sb + kOffBar;
  auto raw_full = [&](int s) { return bar0 + 8u * s; };
  auto raw_empty = [&](int s) { return bar0 + 8u * (3 + s); };
  auto a_full = [&](int s) { return bar0 + 8u * (6 + s); };
  auto a_empty = [&](int s) { return bar0 + 8u * (10 + s); };
  auto b_full = [&](int s) { return bar0 + 8u * (14 + s); };
  auto b_empty = [&](int s) { return bar0 + 8u * (16 + s); };
  auto d_full = [&](int s) { return bar0 + 8u * (18 + s); };
  auto d_empty = [&](int s) { return bar0 + 8u * (20 + s); };
  const uint32_t drain = bar0 + 8u * 22;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- set-up before waiting for the previous kernel: barriers, zero rows of the B images, TMEM
  if (tid == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(raw_full(s), 1);
      mbar_init(raw_empty(s), kDecThreads / 32);
    }
    for (int s = 0; s < kASlots; ++s) {
      mbar_init(a_full(s), kDecThreads / 32);
      mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_full(s), kDecThreads / 32);
      mbar_init(b_empty(s), 1);
      mbar_init(d_full(s), 1);
      mbar_init(d_empty(s), 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
  }
  for (uint32_t i = tid; i < 2 * kBSlot / 16; i += kThreads)  // rows 2..15 of both B images stay zero
    st_shared_v4(sb + kOffB + 16 * i, make_uint4(0, 0, 0, 0));
  fence_proxy_async();
  if (warp == 2) tmem_alloc(sb + kOffTmem, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<uint32_t*>(base + kOffTmem);
  griddep_wait();
  griddep_launch();

  // tiles per request and their exclusive prefix
  {
    const int per = (batch + kThreads - 1) / kThreads;
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
    int32_t* scan = reinterpret_cast<int32_t*>(base + kOffRed);
    if (lane == 31) scan[warp] = v;
    __syncthreads();
    int32_t before = 0, total = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      if (w < warp) before += scan[w];
      total += scan[w];
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

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: codes (TMA, swizzled) and scales (bulk) of the tile's runs
      int64_t it = 0;
      TileWalk walk(prefix, n_c, batch, t_lo);
      for (int64_t t = t_lo; t < t_hi && !*abort_flag; ++t, ++it) {
        const TileInfo ti = walk.at(t);
        const int st = static_cast<int>(it % kRawStages);
        if (!wait_or_abort(raw_empty(st), (static_cast<uint32_t>(it / kRawStages) & 1u) ^ 1u, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        int32_t phys[2];
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int64_t e = ti.e0 + kRun * j;
          phys[j] = e < n_c[ti.b] ? entry_block(p, ti.b, e, status, true) : -1;
          if (phys[j] >= 0) bytes += 2 * kRun * 128 + kRun * 32;
        }
        mbar_expect_tx(raw_full(st), bytes);  // also the stage's one arrival (0 bytes: nothing loaded)
        const uint32_t stage = sb + kOffRaw + st * kRawStage;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (phys[j] < 0) continue;
          const int64_t row = static_cast<int64_t>(phys[j]) * p.epb + ((ti.e0 + kRun * j) & (p.epb - 1));
#pragma unroll
          for (int hb = 0; hb < 2; ++hb)
            tma_load_2d(stage + (2 * j + hb) * (kRun * 128), &codes_map, 128 * hb, static_cast<int>(row), raw_full(st));
          bulk_g2s(stage + kRawCodes + j * (kRun * 32), p.comp_scales + row * 32, kRun * 32, raw_full(st));
        }
      }
      // nothing may land in shared memory after the CTA exits: wait for the stages still in flight
      for (int64_t j = it > kRawStages ? it - kRawStages : 0; j < it; ++j)
        if (!mbar_wait(raw_full(static_cast<int>(j % kRawStages)), static_cast<uint32_t>(j / kRawStages) & 1u))
          *abort_flag = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMAs: per chunk, D[acc] (+)= A(slot) . B(chunk)^T
      int64_t it = 0, g = 0;
      int prev_b = -1, ns = 0, bs = 0;
      bool issued = false, ok = true;
      TileWalk walk(prefix, n_c, batch, t_lo);
      for (int64_t t = t_lo; t < t_hi && ok; ++t, ++it) {
        const TileInfo ti = walk.at(t);
        if (ti.b != prev_b) {
          bs = ns & 1;
          ok = wait_or_abort(b_full(bs), static_cast<uint32_t>(ns >> 1) & 1u, abort_flag);
          prev_b = ti.b;
          ++ns;
        }
        const int acc = static_cast<int>(it & 1);
        ok = ok && wait_or_abort(d_empty(acc), (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u, abort_flag);
        for (int c = 0; c < kChunks && ok; ++c, ++g) {
          const int s = static_cast<int>(g % kASlots);
          ok = wait_or_abort(a_full(s), static_cast<uint32_t>(g / kASlots) & 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = sb + kOffA + s * kASlot;
          const uint32_t b0 = sb + kOffB + bs * kBSlot + c * kBChunk;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tmem + 16u * acc, sdesc_sw128(a0 + ks * 32), sdesc_sw128(b0 + ks * 32), kIdesc, (c | ks) != 0);
          mma_commit(a_empty(s));
          issued = true;
        }
        if (!ok) break;
        mma_commit(d_full(acc));
        const bool last_of_request = t + 1 == t_hi || prefix[ti.b + 1] <= t + 1;
        if (last_of_request) mma_commit(b_empty(bs));
      }
      if (!ok) *abort_flag = 1;
      if (issued) {  // every MMA issued has completed before the tensor memory is released
        mma_commit(drain);
        if (!mbar_wait(drain, 0)) *abort_flag = 1;
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- epilogue: entry j = 32 (warp - 4) + lane = TMEM lane
    const int q4 = warp - 4;
    const int j = 32 * q4 + lane;
    int64_t it = 0;
    int prev_b = -1;
    float unscale = 1.f;
    TileWalk walk(prefix, n_c, batch, t_lo);
    for (int64_t t = t_lo; t < t_hi; ++t, ++it) {
      const TileInfo ti = walk.at(t);
      if (ti.b != prev_b) {  // this request's q_bar scale, as the decoders compute it
        unscale = exp2i(-qbar_shift(ws.qbar + static_cast<int64_t>(ti.b) * kD, lane));
        prev_b = ti.b;
      }
      const int acc = static_cast<int>(it & 1);
      const bool ok = __all_sync(0xffffffffu, wait_or_abort(d_full(acc), static_cast<uint32_t>(it >> 1) & 1u, abort_flag));
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t d[2];
      tmem_ld2(tmem + (static_cast<uint32_t>(32 * q4) << 16) + 16u * acc, d);
      tc_fence_before();
      mbar_arrive(d_empty(acc));
      const int64_t e = ti.e0 + j;
      const bool writer = j < ti.n_valid;
      uint32_t bin = 0xffffffffu - lane;
      if (writer) {
        // entries of an unmapped block score 0 (the block was flagged by the producer)
        const bool mapped = entry_block(p, ti.b, e, status, false) >= 0;
        const float s = mapped ? (__uint_as_float(d[0]) + __uint_as_float(d[1])) * unscale : 0.f;
        scores[static_cast<int64_t>(ti.b) * stride + e] = s;
        bin = f32_order_key(s) >> 21;
      }
      const uint32_t same = __match_any_sync(0xffffffffu, bin);
      if (writer && lane == __ffs(same) - 1)
        atomicAdd(ws.hist + static_cast<int64_t>(ti.b) * kHistBins + bin, static_cast<uint32_t>(__popc(same)));
    }
  } else if (warp >= kFirstDecWarp) {
    // ---------------- decoders: entry je = dt / 2, half h = dt % 2 of every 64-dim chunk
    const int dt = tid - 32 * kFirstDecWarp;
    const int je = dt >> 1, h = dt & 1;
    const int run = je / kRun, r = je % kRun;
    int64_t it = 0, g = 0;
    int prev_b = -1, ns = 0;
    bool ok = true;
    TileWalk walk(prefix, n_c, batch, t_lo);
    for (int64_t t = t_lo; t < t_hi && ok; ++t, ++it) {
      const TileInfo ti = walk.at(t);
      if (ti.b != prev_b) {
        // B image of the request in slot ns & 1: row 0 = fp16(q_bar 2^sh), row 1 = fp16 of the
        // remainder; thread dt holds dims 2 dt, 2 dt + 1 (chunk dt / 32, granule (dt % 32) / 4)
        const int bs = ns & 1;
        ok = __all_sync(0xffffffffu, wait_or_abort(b_empty(bs), (static_cast<uint32_t>(ns >> 1) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        const float* qb = ws.qbar + static_cast<int64_t>(ti.b) * kD;
        const float up = exp2i(qbar_shift(qb, lane));
        const float2 v = reinterpret_cast<const float2*>(qb)[dt];
        const float a = v.x * up, c = v.y * up;
        const __half2 hi = __floats2half2_rn(a, c);
        const float2 back = __half22float2(hi);
        const __half2 lo = __floats2half2_rn(a - back.x, c - back.y);
        const int ch = dt >> 5, gr = (dt & 31) >> 2;
        const uint32_t bslot = sb + kOffB + bs * kBSlot + ch * kBChunk + 4u * (dt & 3);
        st_shared_u32(bslot + 0 * 128 + ((gr ^ 0) << 4), half2_bits(hi));
        st_shared_u32(bslot + 1 * 128 + ((gr ^ 1) << 4), half2_bits(lo));
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_full(bs));
        prev_b = ti.b;
        ++ns;
      }
      const int st = static_cast<int>(it % kRawStages);
      ok = __all_sync(0xffffffffu, wait_or_abort(raw_full(st), static_cast<uint32_t>(it / kRawStages) & 1u, abort_flag));
      if (!ok) break;
      const uint32_t stage = sb + kOffRaw + st * kRawStage;
      for (int c = 0; c < kChunks; ++c, ++g) {
        const int s = static_cast<int>(g % kASlots);
        ok = __all_sync(0xffffffffu, wait_or_abort(a_empty(s), (static_cast<uint32_t>(g / kASlots) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        // 16 bytes of codes: box half c / 4, granule 2 (c % 4) + h of row r (128-byte swizzle)
        const int gi = 2 * (c & 3) + h;
        const uint4 codes = ld_shared_v4(stage + (2 * run + (c >> 2)) * (kRun * 128) + r * 128 + ((gi ^ (r & 7)) << 4));
        const uint32_t sc2 = ld_shared_u16(stage + kRawCodes + je * 32 + 4 * c + 2 * h);
        const __half s0 = __half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(sc2 & 0xffu), __NV_E4M3));
        const __half s1 = __half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(sc2 >> 8), __NV_E4M3));
        const __half2 sa = __half2(s0, s0), sbv = __half2(s1, s1);
        const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
        uint32_t o[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          o[k] = half2_bits(__hmul2(e2m1x2_to_half2(static_cast<uint8_t>(w[k >> 2] >> (8 * (k & 3)))), k < 8 ? sa : sbv));
        const uint32_t a0 = sb + kOffA + s * kASlot + je * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(a0 + (((4 * h + i) ^ (je & 7)) << 4), make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full(s));
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(raw_empty(st));
    }
    if (!ok) *abort_flag = 1;
  }
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicOr(status, CKV_DEV_TIMEOUT);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
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

}  // namespace

bool score_nvfp4_tc_supported(const LayerParams& p) {
  return p.comp_dtype == CKV_NVFP4 && p.D == kD && p.epb >= kRun;
}

cudaError_t launch_score_nvfp4_tc(const LayerParams& p, int batch, int max_seq_len, const IndexerWs& ws,
                                  float* scores, int64_t stride, uint32_t* status, cudaStream_t stream) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  // the codes as a 2-D tensor [pool rows][256 bytes], loaded in boxes of 64 rows x 128 bytes with
  // the 128-byte swizzle
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD / 2), static_cast<cuuint64_t>(p.comp_blocks) * p.epb};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD / 2)};
  const cuuint32_t box[2] = {128, kRun};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p.comp_codes, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int smem = static_cast<int>(kOffPrefix + sizeof(int32_t) * (2 * batch + 1)) + 1024;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(score_nvfp4_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>(batch) * ((static_cast<int64_t>(max_seq_len) / p.r + kTile - 1) / kTile);
  int64_t grid = sm_count();
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  prof_begin(kProfScore, stream);
  e = launch_kernel(score_nvfp4_tc_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), static_cast<size_t>(smem),
                    stream, map, p, batch, ws, scores, stride, status);
  prof_end(kProfScore, stream);
  return e;
}

}  // namespace ckv

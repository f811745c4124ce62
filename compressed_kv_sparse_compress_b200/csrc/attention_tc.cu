// Tensor-core attention path (tcgen05, kind::f16, fp32 accumulation in tensor memory) for
// H = 64 query heads sharing one K=V vector of D = 512 (multi-query attention), over a bf16 or
// NVFP4 compressed cache and an FP8 window.
//
// 24-ai.news "vLLM uveo DeepSeek V4 s 8,7x manjim KV cacheom", section "Kako funkcionira
// optimizacija KV cachea?": every head reads the same shared K=V vector, so the heads x keys
// contractions are dense matrix products; aidevelopers.cz "DeepSeek-V4.1-Flash ve vLLM", section
// "Vykon neprinesl jeden kernel": attention over an NVFP4 compressed cache.
//
// Products (keys in tiles of 32; all operands fp16 in shared memory, 128-byte swizzled rows):
//     S[hi|lo, keys]  = [Q'hi; Q'lo] . X'^T     M = 128 (the 64 hi rows of the query, then its 64
//                                               lo rows), N = 32 keys, K = D; A = Q', B = X'
//                                               (both K-major)
//     O^T[D, heads]  += X'^T . P^T               M = 128 dims (4 blocks), N = 64 heads, K = keys;
//                                               A = X'^T (MN-major: the same tile), B = P (K-major)
// Exactness: the rotated query of head h is scaled by a power of two g_h^-1 (its largest element
// lands in [2^8, 2^9)) and split into fp16 hi + lo parts, which carry its fp32 value to about
// 2^-22; each key is scaled by a power of two of its own (largest element in [2^8, 2^9)) before
// it is converted to fp16, which is exact for bf16 values, e4m3 codes and e2m1 x e4m3 products
// whatever their magnitude. The logit of (head h, key j) is (S_hi + S_lo) g_h f_j sm_scale
// log2(e), where the value factor f_j is the key's power of two times its FP8 token scale (1 for
// the compressed entries). The softmax runs in base 2 with a running maximum that is raised only
// when a tile exceeds it by more than 8 nats; the weights enter P as p_j f_j / F, F being a
// power-of-two running bound of the value factors raised only past 16 F, so P stays below 2^16
// and O^T = F^-1 sum_j p_j x_j. Raising either bound rescales O^T in tensor memory.
//
// Warp roles (672 threads):
//   warps 0..3   softmax: warp w reads TMEM lane quarter w (w < 2: the hi rows of heads
//                32w .. 32w+31; w >= 2: their lo rows); a hi warp and its lo partner swap half of
//                their keys through shared memory, so that each thread owns 16 keys of one head
//   warp 4       owns the tensor memory; lane 0 issues every MMA (the logits of tile t+1 before
//                the output product of tile t, so the tensor pipe works while the softmax runs)
//   warps 5..20  loaders: each resolves the pool rows of its 2 keys of every tile, keeps the raw
//                bytes of the next two tiles in flight in registers and converts a tile into the
//                fp16 operand image once its shared-memory stage (one of 2) is free; they also
//                build the query image at the start and write the partial outputs at the end
// Every wait on an mbarrier is bounded; a role that gives up raises an abort flag that the others
// poll, every issued MMA is drained before the epilogue and before the tensor memory is freed, and
// the split is then marked empty with CKV_DEV_TIMEOUT set.
//
// Each CTA takes keys_per_split consecutive keys of one request's key list (the window tokens
// [max(0, L-W), L) first, then the selected entries, or every entry of a dense layer) and writes
// an un-normalised partial (maximum in base 2, sum, output rows as fp16 with a power-of-two
// scale); the combine kernel merges the splits and applies the inverse rotation.

#include "ckv_internal.h"
#include "ckv_ptx.cuh"

namespace ckv {

// Failure-path hook for tests (ckv_debug_force_timeout): the request whose MMA issuers wait on a
// barrier that nothing completes, -1 for none.
__device__ int g_attn_forced_timeout = -1;

namespace {

constexpr int kH = 64;
constexpr int kD = 512;
constexpr int kTile = 32;                              // keys per tile (N of the logits product)
constexpr int kMaxTiles = 16;                          // tiles per split at most
constexpr int kChunks = kD / 64;                       // 64-dim chunks (128-byte rows)
constexpr int kSoftWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kFirstLoadWarp = 5;
constexpr int kLoadWarps = 16;
constexpr int kThreads = 32 * (kFirstLoadWarp + kLoadWarps);  // 672
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kSoftThreads = 32 * kSoftWarps;
static_assert(kTile == 2 * kLoadWarps, "each loader warp stages two keys of a tile");
static_assert(kMaxTiles * 2 <= 32, "one lane of a loader warp per (tile, key) of the split");
static_assert(kH == 4 * kLoadWarps, "each loader warp builds the query image of four heads");

constexpr uint32_t kQChunk = 2 * kH * 128;             // 16 KB: 64 hi rows, then 64 lo rows
constexpr uint32_t kQBytes = kQChunk * kChunks;        // 128 KB
constexpr uint32_t kXChunk = kTile * 128;              // 4 KB
constexpr uint32_t kXStage = kXChunk * kChunks;        // 32 KB
constexpr uint32_t kPBytes = kH * 128;                 // 8 KB: row = head; stage s in bytes 64s..64s+63
constexpr uint32_t kXchStride = 20;                    // floats per lane in an exchange slot
constexpr uint32_t kXchSlot = 32 * kXchStride * 4;     // 2560 B
constexpr uint32_t kSCol = 0;                          // S stage s: columns 32 s
constexpr uint32_t kOCol = 256;                        // O^T dims block m: columns 256 + 64 m
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRaiseLog2 = 8.0f * kLog2e;            // the running max moves past +8 nats
constexpr float kRaiseF = 16.0f;                       // the value bound moves past 16x

// shared memory carve-up (byte offsets from a 1024-aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffX = kOffQ + kQBytes;
constexpr uint32_t kOffP = kOffX + 2 * kXStage;
constexpr uint32_t kOffXch = kOffP + kPBytes;            // float[4 slots][32 lanes][20]
constexpr uint32_t kOffKf = kOffXch + 4 * kXchSlot;      // float[2 stages][32]: key value factors
constexpr uint32_t kOffRed = kOffKf + 2 * kTile * 4;     // float[2][4][32]: max and bound per lane
constexpr uint32_t kOffAlpha = kOffRed + 2 * 4 * 32 * 4; // float[64]: O^T rescale per head
constexpr uint32_t kOffQs = kOffAlpha + kH * 4;          // float[64]: query scale g_h per head
constexpr uint32_t kOffEpi = kOffQs + kH * 4;            // float[4][64]: output amax per lane quarter
constexpr uint32_t kOffRope = kOffEpi + 4 * kH * 4;      // double[256][2]: cos, sin per rotary pair
constexpr uint32_t kOffMisc = kOffRope + 256 * 16;       // int abort; float F
constexpr uint32_t kOffBar = kOffMisc + 16;              // 11 mbarriers
constexpr uint32_t kOffTmem = kOffBar + 11 * 8;
constexpr uint32_t kSmemUsed = kOffTmem + 8;
constexpr int kSmemBytes = static_cast<int>(kSmemUsed) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

// mbarriers: xfull[2] (loaders -> MMA, softmax), xfree[2] (output product of the stage's tile
// done -> loaders, softmax), sfull[2] (logits done -> softmax), sfree[2] (softmax read the logits
// -> MMA), pfull[2] (softmax wrote P -> MMA), drain (every MMA done)
constexpr int kBarXfull = 0, kBarXfree = 2, kBarSfull = 4, kBarSfree = 6, kBarPfull = 8, kBarDrain = 10;

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

// instruction descriptors, kind::f16 with fp32 accumulation and fp16 A and B:
//   logits: M = 128, N = 32, A and B K-major;  output: M = 128, N = 64, A MN-major, B K-major
constexpr uint32_t kIdescS = (1u << 4) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24) | (1u << 15);

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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// barrier `id` over `n` threads that also ANDs (kAnd) or ORs a predicate across them
template <bool kAnd>
__device__ __forceinline__ bool bar_red(int id, int n, bool v) {
  uint32_t out;
  if constexpr (kAnd) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %1, 0;\n bar.red.and.pred p, %2, %3, p;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %1, 0;\n bar.red.or.pred p, %2, %3, p;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
        : "memory");
  }
  return out != 0;
}

// bounded wait for the completion of the barrier phase with parity `phase` (polls that suspend the
// thread, ckv_ptx.cuh); also gives up once another role has raised the abort flag
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t phase, volatile int* abort_flag,
                                              uint32_t limit = kWaitLimit) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait_sleep(bar, phase, kWaitSuspendNs)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

// ------------------------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t half2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

__device__ __forceinline__ uint32_t pack_f32x2(float a, float b) {
  return half2_bits(__floats2half2_rn(a, b));
}

// 2^e as a float for -126 <= e <= 127
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// the power-of-two shift that puts a largest magnitude with float bits `mb` into [2^8, 2^9)
// (0 for an all-zero vector), within the range where both 2^shift and 2^-shift are normal
__device__ __forceinline__ int norm_shift(uint32_t mb) {
  if (mb == 0u) return 0;
  const int e = static_cast<int>(mb >> 23) - 127;
  return max(-126, min(126, 8 - e));
}

// the smallest power of two >= x (x finite and > 0)
__device__ __forceinline__ float pow2_ceil(float x) {
  const uint32_t u = __float_as_uint(x);
  const uint32_t e = (u >> 23) + ((u & 0x7fffffu) != 0u ? 1u : 0u);
  return e >= 255u ? INFINITY : __uint_as_float(e << 23);
}

// Raw bytes of one 8-element granule of a key: bf16 16 B, FP8 window 8 B, NVFP4 4 B of codes and
// the e4m3 scale of its 16-element block.
struct Raw {
  uint4 a;
  uint32_t s;
};

template <int CT>
__device__ __forceinline__ Raw load_granule(const LayerParams& p, int64_t row, bool win, int g) {
  Raw r;
  r.a = make_uint4(0, 0, 0, 0);
  r.s = 0;
  if (row < 0) return r;
  if (win) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.win_codes + row * p.win_row_bytes) + g);
    r.a.x = v.x;
    r.a.y = v.y;
    return r;
  }
  const uint8_t* base = p.comp_codes + row * p.comp_row_bytes;
  if constexpr (CT == CKV_BF16) {
    r.a = __ldg(reinterpret_cast<const uint4*>(base) + g);
  } else {
    r.a.x = __ldg(reinterpret_cast<const uint32_t*>(base) + g);
    r.s = __ldg(p.comp_scales + row * (kD / 16) + (g >> 1));
  }
  return r;
}

// the granule's 8 values as fp32 (exact): e4m3 codes of a window token (its scale is applied
// through the key factor), bf16 values, or e2m1 codes times their block's e4m3 scale
template <int CT>
__device__ __forceinline__ void decode_granule(const Raw& r, bool win, float (&v)[8]) {
  if (win) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w = i < 2 ? r.a.x : r.a.y;
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w >> (16 * (i & 1))) & 0xffffu), __NV_E4M3);
      const float2 f = __half22float2(__half2(h));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
    return;
  }
  if constexpr (CT == CKV_BF16) {
    const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    const __half s = __half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(r.s), __NV_E4M3));
    const __half2 s2 = __half2(s, s);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(__hmul2(e2m1x2_to_half2(static_cast<uint8_t>(r.a.x >> (8 * i))), s2));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
}

// byte offset of 16-byte granule g (8 dims) of row `row` in an operand made of 64-dim chunks of
// `chunk_bytes`, rows of 128 bytes with the 128-byte swizzle
__device__ __forceinline__ uint32_t swz(uint32_t chunk_bytes, int row, int g) {
  return static_cast<uint32_t>(g >> 3) * chunk_bytes + static_cast<uint32_t>(row) * 128u +
         (static_cast<uint32_t>((g & 7) ^ (row & 7)) << 4);
}

// The key list of request b: window tokens first, then the selected (or all) entries.
struct Keys {
  int L;
  int64_t n_c, n_sel, n_win, n_keys;
};

// Pool row (-1: absent, with the status bit set) of key k of request b; window keys set *win.
__device__ __forceinline__ int64_t key_row(const LayerParams& p, const Keys& kl, int b, const int32_t* idx,
                                           int idx_stride, int64_t k, bool* win, uint32_t* status) {
  *win = k < kl.n_win;
  if (*win) return win_row(p, b, kl.L - kl.n_win + k, status);
  const int64_t e = k - kl.n_win;
  const int64_t ent = idx ? idx[static_cast<int64_t>(b) * idx_stride + e] : e;
  if (ent < 0 || ent >= kl.n_c) {
    atomicOr(status, CKV_DEV_BAD_INDEX);
    return -1;
  }
  return comp_row(p, b, ent, status);
}

// ------------------------------------------------------------------------------------ kernel

// rope_ready: the step's query pass already wrote the cos/sin table into ws.rope
template <int CT>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const float* q, const int32_t* idx,
    const int32_t* cnt, int idx_stride, AttnWs ws, uint32_t* status, bool rope_ready) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  float* kf = reinterpret_cast<float*>(base + kOffKf);
  float* red = reinterpret_cast<float*>(base + kOffRed);
  float* alpha_sm = reinterpret_cast<float*>(base + kOffAlpha);
  float* qs = reinterpret_cast<float*>(base + kOffQs);
  float* epi = reinterpret_cast<float*>(base + kOffEpi);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc);
  float* f_final = reinterpret_cast<float*>(base + kOffMisc + 4);
  auto bar = [&](int i) { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffTmem);

  // requests on x so that the first split of every request is launched first and the splits that
  // find no keys (short requests of a mixed batch) come last
  const int b = blockIdx.x, split = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- set-up that reads no global memory, before waiting for the previous kernel
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarXfull + s), kLoadWarps);
      mbar_init(bar(kBarXfree + s), 1);
      mbar_init(bar(kBarSfull + s), 1);
      mbar_init(bar(kBarSfree + s), kSoftThreads);
      mbar_init(bar(kBarPfull + s), kSoftThreads);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    *f_final = 0.f;
    fence_proxy_async();
  }
  griddep_wait();
  griddep_launch();

  Keys kl;
  kl.L = seq_len[b];
  const bool live = kl.L >= 1 && kl.L <= max_seq_len;  // a bad length is flagged by the combine
  kl.n_c = live ? kl.L / p.r : 0;
  kl.n_sel = !live ? 0 : idx ? min(static_cast<int64_t>(max(cnt[b], 0)), static_cast<int64_t>(idx_stride)) : kl.n_c;
  kl.n_win = live ? min(p.W, kl.L) : 0;
  kl.n_keys = kl.n_win + kl.n_sel;
  const int64_t k_begin = static_cast<int64_t>(split) * ws.keys_per_split;
  if (k_begin >= kl.n_keys) return;  // nothing to attend (uniform across the CTA; nothing held)
  if (warp == kMmaWarp) tmem_alloc(sb + kOffTmem, kTmemCols);
  tc_fence_before();
  __syncthreads();  // barrier initialisation and the tensor memory address
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  double* rope_sm = reinterpret_cast<double*>(base + kOffRope);
  const int nk = static_cast<int>(min(kl.n_keys - k_begin, static_cast<int64_t>(ws.keys_per_split)));
  const int n_tiles = (nk + kTile - 1) / kTile;
  const int64_t slot = (static_cast<int64_t>(b) * ws.splits + split) * kH;

  // ---- prologue (loaders): resolve the rows of their keys, put the first two tiles' loads in
  //      flight, build the query image (4 heads per warp)
  const int li = warp - kFirstLoadWarp;  // loader index (warps >= kFirstLoadWarp)
  // lane j of a loader warp holds the row of key 2 li + (j & 1) of tile j >> 1
  long long my_row = -1;
  int my_win = 0;
  float my_tscale = 1.f;
  Raw ring[2][2][2];  // [tile parity][key u][granule lane, lane + 32]
  auto row_of = [&](int t, int u, bool* win, float* tsc) -> int64_t {
    const int src = 2 * t + u;
    *win = __shfl_sync(0xffffffffu, my_win, src) != 0;
    *tsc = __shfl_sync(0xffffffffu, my_tscale, src);
    return static_cast<int64_t>(__shfl_sync(0xffffffffu, my_row, src));
  };
  auto issue = [&](int t, Raw (&r)[2][2]) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      bool win;
      float tsc;
      const int64_t row = row_of(t, u, &win, &tsc);
      r[u][0] = load_granule<CT>(p, row, win, lane);
      r[u][1] = load_granule<CT>(p, row, win, lane + 32);
    }
  };
  if (warp < kSoftWarps) {
    // the cos/sin of every rotary pair at the query position L-1 (fp64 angles), one pair per
    // thread: taken from the step's table when its query pass wrote it, else computed here (and
    // stored by split 0 for the combine's inverse rotation)
    double* rope_g = ws.rope + static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2;
    for (int i = tid; i < p.d_r / 2; i += kSoftThreads) {
      double sn, cs;
      if (rope_ready) {
        cs = rope_g[2 * i];
        sn = rope_g[2 * i + 1];
      } else {
        sincos(static_cast<double>(kl.L - 1) * rope_inv_freq(p, i), &sn, &cs);
        if (split == 0) {
          rope_g[2 * i] = cs;
          rope_g[2 * i + 1] = sn;
        }
      }
      rope_sm[2 * i] = cs;
      rope_sm[2 * i + 1] = sn;
    }
  }
  if (warp >= kFirstLoadWarp) {
    const int t = lane >> 1, u = lane & 1;
    const int kloc = t * kTile + 2 * li + u;
    if (t < n_tiles && kloc < nk) {
      bool win;
      my_row = key_row(p, kl, b, idx, idx_stride, k_begin + kloc, &win, status);
      my_win = win ? 1 : 0;
      if (win && my_row >= 0) my_tscale = p.win_scales[my_row];
    }
    issue(0, ring[0]);
    if (n_tiles > 1) issue(1, ring[1]);
  }
  __syncthreads();  // the rotary table
  if (warp >= kFirstLoadWarp) {
    // query image, heads 4 li .. 4 li + 3: lane l holds dims 16 l .. 16 l + 15 (granules 2l,
    // 2l + 1 of chunk l/4); the rotary pairs 8 l .. 8 l + 7 are rotated at the query position L-1
    // (fp64 angles); hi rows are h, lo rows 64 + h
    const int first_rope = (kD - p.d_r) / 2;
    const float* qb = q + static_cast<int64_t>(b) * kH * kD;
#pragma unroll 1
    for (int hh = 0; hh < 4; ++hh) {
      const int h = 4 * li + hh;
      float x[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(qb + static_cast<int64_t>(h) * kD + 16 * lane) + k);
        x[4 * k] = v.x;
        x[4 * k + 1] = v.y;
        x[4 * k + 2] = v.z;
        x[4 * k + 3] = v.w;
      }
      if (8 * lane + 7 >= first_rope) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int pr = 8 * lane + k;
          if (pr >= first_rope) {
            const double rc = rope_sm[2 * (pr - first_rope)], rs = rope_sm[2 * (pr - first_rope) + 1];
            const double a0 = x[2 * k], a1 = x[2 * k + 1];
            x[2 * k] = static_cast<float>(a0 * rc - a1 * rs);
            x[2 * k + 1] = static_cast<float>(a0 * rs + a1 * rc);
          }
        }
      }
      uint32_t mb = 0;
#pragma unroll
      for (int k = 0; k < 16; ++k) mb = max(mb, __float_as_uint(x[k]) & 0x7fffffffu);
      const int sh = norm_shift(__reduce_max_sync(0xffffffffu, mb));
      const float up = exp2i(sh);
      if (lane == 0) qs[h] = exp2i(-sh);
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float a = x[2 * k] * up, c = x[2 * k + 1] * up;
        const __half2 h16 = __floats2half2_rn(a, c);
        const float2 back = __half22float2(h16);
        hi[k] = half2_bits(h16);
        lo[k] = pack_f32x2(a - back.x, c - back.y);
      }
      const uint32_t qa = sb + kOffQ;
      st_shared_v4(qa + swz(kQChunk, h, 2 * lane), make_uint4(hi[0], hi[1], hi[2], hi[3]));
      st_shared_v4(qa + swz(kQChunk, h, 2 * lane + 1), make_uint4(hi[4], hi[5], hi[6], hi[7]));
      st_shared_v4(qa + swz(kQChunk, kH + h, 2 * lane), make_uint4(lo[0], lo[1], lo[2], lo[3]));
      st_shared_v4(qa + swz(kQChunk, kH + h, 2 * lane + 1), make_uint4(lo[4], lo[5], lo[6], lo[7]));
    }
    fence_proxy_async();
  }
  __syncthreads();  // the query image and its scales

  if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------- MMAs: the logits of tile t, then the output product of tile t-1
      bool issued = false;
      auto pv = [&](int u) -> bool {
        const int s = u & 1;
        if (!wait_or_abort(bar(kBarPfull + s), static_cast<uint32_t>(u >> 1) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t xs = sb + kOffX + s * kXStage;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint64_t bp = sdesc(sb + kOffP + 64 * s + 32 * kk, 16, 1024);
#pragma unroll
          for (int m = 0; m < 4; ++m)
            mma_f16(tmem + kOCol + 64 * m, sdesc(xs + 2 * m * kXChunk + kk * 2048, kXChunk, 1024), bp, kIdescPV,
                    (u > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(kBarXfree + s));
        return true;
      };
      // the failure-path hook: a wait on the drain barrier, which nothing completes before the
      // first MMA, runs out and the CTA takes its failure path
      bool ok = g_attn_forced_timeout != b || wait_or_abort(bar(kBarDrain), 0, abort_flag, 16);
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int s = t & 1;
        ok = wait_or_abort(bar(kBarXfull + s), static_cast<uint32_t>(t >> 1) & 1u, abort_flag) &&
             (t < 2 || wait_or_abort(bar(kBarSfree + s), static_cast<uint32_t>((t >> 1) - 1) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs = sb + kOffX + s * kXStage;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tmem + kSCol + 32 * s, sdesc(sb + kOffQ + c * kQChunk + ks * 32, 16, 1024),
                    sdesc(xs + c * kXChunk + ks * 32, 16, 1024), kIdescS, (c | ks) != 0);
        }
        mma_commit(bar(kBarSfull + s));
        issued = true;
        if (t > 0) ok = pv(t - 1);
      }
      if (ok) ok = pv(n_tiles - 1);
      if (!ok) *abort_flag = 1;
      if (issued) {  // every MMA issued has completed before O^T is read or the memory freed
        mma_commit(bar(kBarDrain));
        if (!mbar_wait(bar(kBarDrain), 0)) *abort_flag = 1;
      }
    }
    __syncwarp();
  } else if (warp < kSoftWarps) {
    // ---------------- softmax: thread (quarter q4, lane) = TMEM lane 32 q4 + lane: head h, hi
    //                  (q4 < 2) or lo rows; after the swap it owns keys kb .. kb + 15 of head h
    const int q4 = warp;
    const bool hi_row = q4 < 2;
    const int h = 32 * (q4 & 1) + lane;
    const int kb = hi_row ? 0 : 16;
    const float ch = qs[h] * p.sm_scale * kLog2e;
    float* xch_mine = reinterpret_cast<float*>(base + kOffXch + q4 * kXchSlot) + lane * kXchStride;
    const float* xch_peer = reinterpret_cast<const float*>(base + kOffXch + (q4 ^ 2) * kXchSlot) + lane * kXchStride;
    float* red_m = red;            // [4][32]
    float* red_f = red + 4 * 32;   // [4][32]
    float m_run = -INFINITY, F_run = 0.f, l_part = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1;
      const uint32_t ph = static_cast<uint32_t>(t >> 1) & 1u;
      bool got = __all_sync(0xffffffffu, wait_or_abort(bar(kBarSfull + s), ph, abort_flag) &&
                                             wait_or_abort(bar(kBarXfull + s), ph, abort_flag));
      ok = bar_red<true>(1, kSoftThreads, got);  // one decision for the four warps
      if (!ok) break;
      tc_fence_after();
      uint32_t raw[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * q4) << 16) + kSCol + 32 * s, raw);
      tc_fence_before();
      mbar_arrive(bar(kBarSfree + s));
      // swap: a hi row hands its keys 16..31 to its lo partner, a lo row its keys 0..15
      float own[16], give[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        own[i] = __uint_as_float(hi_row ? raw[i] : raw[16 + i]);
        give[i] = __uint_as_float(hi_row ? raw[16 + i] : raw[i]);
      }
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4*>(xch_mine + i) = make_float4(give[i], give[i + 1], give[i + 2], give[i + 3]);
      named_sync(1, kSoftThreads);
      float lg[16];
      float mx = -INFINITY, fmx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        const float4 o = *reinterpret_cast<const float4*>(xch_peer + i);
        const float pv4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float f = kf[s * kTile + kb + i + k];
          const float sv = own[i + k] + pv4[k];
          lg[i + k] = f > 0.f ? sv * f * ch : -INFINITY;
          mx = fmaxf(mx, lg[i + k]);
          fmx = fmaxf(fmx, f > 0.f ? f : 0.f);
        }
      }
      red_m[q4 * 32 + lane] = mx;
      red_f[q4 * 32 + lane] = fmx;
      named_sync(1, kSoftThreads);
      const float mt = fmaxf(mx, red_m[(q4 ^ 2) * 32 + lane]);
      const float ft = fmaxf(fmx, red_f[(q4 ^ 2) * 32 + lane]);
      float m_new = m_run, F_new = F_run;
      if (mt > -INFINITY && (m_run == -INFINITY || mt > m_run + kRaiseLog2)) m_new = mt;
      if (ft > 0.f && ft > kRaiseF * F_run) F_new = pow2_ceil(ft);
      const float a_l = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
      const bool moved = m_new != m_run || F_new != F_run;
      if (hi_row) alpha_sm[h] = F_run > 0.f ? a_l * (F_run / F_new) : 0.f;
      const bool rescale = bar_red<false>(1, kSoftThreads, t > 0 && moved);  // alpha visible too
      float psum = 0.f;
      uint32_t packed[8];
      const float inv_F = F_new > 0.f ? 1.f / F_new : 0.f;  // a power of two: exact
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float p0 = lg[i] > -INFINITY ? exp2f(lg[i] - m_new) : 0.f;
        const float p1 = lg[i + 1] > -INFINITY ? exp2f(lg[i + 1] - m_new) : 0.f;
        psum += p0 + p1;
        const float f0 = kf[s * kTile + kb + i], f1 = kf[s * kTile + kb + i + 1];
        packed[i >> 1] = pack_f32x2(p0 * (f0 > 0.f ? f0 : 0.f) * inv_F, p1 * (f1 > 0.f ? f1 : 0.f) * inv_F);
      }
      l_part = l_part * a_l + psum;
      m_run = m_new;
      F_run = F_new;
      const uint32_t prow = sb + kOffP + static_cast<uint32_t>(h) * 128u;
      const int g0 = 4 * s + kb / 8;
      st_shared_v4(prow + (static_cast<uint32_t>(g0 ^ (h & 7)) << 4),
                   make_uint4(packed[0], packed[1], packed[2], packed[3]));
      st_shared_v4(prow + (static_cast<uint32_t>((g0 + 1) ^ (h & 7)) << 4),
                   make_uint4(packed[4], packed[5], packed[6], packed[7]));
      if (rescale) {
        // O^T holds the output products of tiles 0 .. t-1: wait for the last of them, then scale
        // column (head) c of every dims block of this warp's lane quarter by alpha[c]
        const int u = t - 1;
        got = __all_sync(0xffffffffu,
                         wait_or_abort(bar(kBarXfree + (u & 1)), static_cast<uint32_t>(u >> 1) & 1u, abort_flag));
        if (got) {
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
            for (int c0 = 0; c0 < kH; c0 += 8) {
              const uint32_t ta = tmem + (static_cast<uint32_t>(32 * q4) << 16) + kOCol + 64 * m + c0;
              uint32_t o[8];
              tmem_ld8(ta, o);
#pragma unroll
              for (int c = 0; c < 8; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha_sm[c0 + c]);
              tmem_st8(ta, o);
            }
          }
        }
        ok = bar_red<true>(1, kSoftThreads, got);
        if (!ok) break;
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(kBarPfull + s));
    }
    if (!ok) {
      *abort_flag = 1;
    } else {
      // the head's sum: hi row plus its lo partner (they share the maximum)
      if (!hi_row) red_f[q4 * 32 + lane] = l_part;
      named_sync(1, kSoftThreads);
      if (hi_row) {
        const float l = l_part + red_f[(q4 ^ 2) * 32 + lane];
        reinterpret_cast<float2*>(ws.part_ml)[slot + h] = make_float2(m_run, l);
        if (h == 0) *f_final = F_run;
      }
    }
  } else {
    // ---------------- loaders: stage tile t into stage t & 1 once the output product of tile t-2
    //                  has released it
    auto stage = [&](int t, Raw (&r)[2][2]) -> bool {
      const int s = t & 1;
      if (t >= 2 && !__all_sync(0xffffffffu, wait_or_abort(bar(kBarXfree + s),
                                                             static_cast<uint32_t>((t >> 1) - 1) & 1u, abort_flag)))
        return false;
      const uint32_t xs = sb + kOffX + s * kXStage;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int key = 2 * li + u;
        bool win;
        float tsc;
        const int64_t row = row_of(t, u, &win, &tsc);
        float v[2][8];
        decode_granule<CT>(r[u][0], win, v[0]);
        decode_granule<CT>(r[u][1], win, v[1]);
        uint32_t mb = 0;
#pragma unroll
        for (int g = 0; g < 2; ++g)
#pragma unroll
          for (int k = 0; k < 8; ++k) mb = max(mb, __float_as_uint(v[g][k]) & 0x7fffffffu);
        // a power of two that puts the key's largest magnitude in [2^8, 2^9); the key factor is
        // its inverse times the token scale (0 marks an absent key, whose row is zeros)
        const int sh = norm_shift(__reduce_max_sync(0xffffffffu, mb));
        const float up = exp2i(sh);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint4 o;
          o.x = pack_f32x2(v[g][0] * up, v[g][1] * up);
          o.y = pack_f32x2(v[g][2] * up, v[g][3] * up);
          o.z = pack_f32x2(v[g][4] * up, v[g][5] * up);
          o.w = pack_f32x2(v[g][6] * up, v[g][7] * up);
          st_shared_v4(xs + swz(kXChunk, key, lane + 32 * g), o);
        }
        if (lane == 0) kf[s * kTile + key] = row >= 0 ? tsc * exp2i(-sh) : 0.f;
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarXfull + s));
      return true;
    };
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; t += 2) {
      ok = stage(t, ring[0]);
      if (ok && t + 2 < n_tiles) issue(t + 2, ring[0]);
      if (ok && t + 1 < n_tiles) {
        ok = stage(t + 1, ring[1]);
        if (ok && t + 3 < n_tiles) issue(t + 3, ring[1]);
      }
    }
    if (!ok) *abort_flag = 1;
  }

  __syncthreads();  // every role done; the MMA thread has drained the tensor pipe
  const bool aborted = *abort_flag != 0;
  if (!aborted && warp >= kFirstLoadWarp) {
    // ---------------- partial outputs: O^T lane = dim, column = head. Loader warp li reads its
    //                  TMEM lane quarter and head groups li/4 and li/4 + 4. Each head's row is
    //                  stored as fp16 after division by 2^e, e = (exponent of the row's max
    //                  |O^T|) - 15 (at least -126): values below 2^15 with a step of 2^-11 of the
    //                  row's max; part_sc = 2^e F.
    tc_fence_after();
    const int q4 = warp & 3;
    const float F = *f_final;
    auto load_group = [&](int hg, uint32_t (&o)[4][8]) {
#pragma unroll
      for (int m = 0; m < 4; ++m)
        tmem_ld8(tmem + (static_cast<uint32_t>(32 * q4) << 16) + kOCol + 64 * m + 8 * hg, o[m]);
    };
#pragma unroll 1
    for (int gi = 0; gi < 2; ++gi) {
      const int hg = li / 4 + 4 * gi;
      uint32_t o[4][8];
      load_group(hg, o);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float a = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) a = fmaxf(a, fabsf(__uint_as_float(o[m][c])));
        a = warp_max(a);
        if (lane == 0) epi[q4 * kH + 8 * hg + c] = a;
      }
    }
    named_sync(2, kLoadThreads);
#pragma unroll 1
    for (int gi = 0; gi < 2; ++gi) {
      const int hg = li / 4 + 4 * gi;
      uint32_t o[4][8];
      load_group(hg, o);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int hh = 8 * hg + c;
        const float amax = fmaxf(fmaxf(epi[hh], epi[kH + hh]), fmaxf(epi[2 * kH + hh], epi[3 * kH + hh]));
        int ex = 0;
        float sc = 1.f;
        if (amax > 0.f && amax <= 3.4e38f) {
          frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
          sc = exp2i(ex - 15 > -126 ? ex - 15 : -126);
        }
        const float inv = 1.f / sc;  // exact: a power of two
        __half* dst = reinterpret_cast<__half*>(ws.part_h) + (slot + hh) * kD + 32 * q4 + lane;
#pragma unroll
        for (int m = 0; m < 4; ++m) dst[128 * m] = __float2half_rn(__uint_as_float(o[m][c]) * inv);
        if (q4 == 0 && lane == 0) ws.part_sc[slot + hh] = sc * F;
      }
    }
  }
  if (aborted) {
    if (tid == 0) atomicOr(status, CKV_DEV_TIMEOUT);
    if (tid < kH) reinterpret_cast<float2*>(ws.part_ml)[slot + tid] = make_float2(-INFINITY, 0.f);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int CT>
cudaError_t launch_tc(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                      const float* q, const int32_t* idx, const int32_t* cnt, int idx_stride,
                      const AttnWs& ws, uint32_t* status, cudaStream_t stream, bool rope_ready) {
  auto kern = attn_tc_kernel<CT>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(batch, ws.splits);
  return launch_kernel(kern, grid, dim3(kThreads), kSmemBytes, stream, p, seq_len, max_seq_len, q, idx,
                       cnt, idx_stride, ws, status, rope_ready);
}

}  // namespace

// bf16 and NVFP4 compressed caches with an FP8 window at H = 64, D = 512. fp32 caches stay on the
// CUDA-core path: fp32 arithmetic attends them as stored.
bool attention_tc_supported(const LayerParams& p) {
  return p.H == kH && p.D == kD && (p.comp_dtype == CKV_BF16 || p.comp_dtype == CKV_NVFP4) &&
         p.win_dtype == CKV_FP8_E4M3;
}

// Keys per split: t tiles of 32 keys, t in 1 .. 16, minimising (waves of one CTA per SM) x
// (t + 2), the 2 standing for a split's fixed cost (query image, rows, partial write).
int attention_tc_keys_per_split(int batch, int64_t max_keys) {
  const int64_t tiles = max_keys > 0 ? (max_keys + kTile - 1) / kTile : 1;
  const int64_t sms = sm_count();
  int best_t = 1;
  int64_t best = -1;
  for (int t = 1; t <= kMaxTiles; ++t) {
    const int64_t ctas = static_cast<int64_t>(batch) * ((tiles + t - 1) / t);
    const int64_t cost = ((ctas + sms - 1) / sms) * (t + 2);
    if (best < 0 || cost < best) {
      best = cost;
      best_t = t;
    }
    if (t >= tiles) break;
  }
  return kTile * best_t;
}

cudaError_t attention_force_timeout(int request) {
  return cudaMemcpyToSymbol(g_attn_forced_timeout, &request, sizeof(int));
}

cudaError_t launch_attention_tc(const LayerParams& p, int batch, const int32_t* seq_len,
                                int max_seq_len, const float* q, const int32_t* idx,
                                const int32_t* cnt, int idx_stride, const AttnWs& ws,
                                uint32_t* status, cudaStream_t stream, bool rope_ready) {
  if (p.win_dtype != CKV_FP8_E4M3) return cudaErrorInvalidValue;
  if (p.comp_dtype == CKV_BF16)
    return launch_tc<CKV_BF16>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream,
                               rope_ready);
  if (p.comp_dtype == CKV_NVFP4)
    return launch_tc<CKV_NVFP4>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream,
                                rope_ready);
  return cudaErrorInvalidValue;
}

}  // namespace ckv

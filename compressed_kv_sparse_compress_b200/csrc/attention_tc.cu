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
//     S[rows, keys]  = Q' . X'^T      M = 128 query rows, N = 32 keys, K = D; A = Q', B = X'
//                                    (both K-major). Row 32 g + i (g = 0..3, i = 0..31) holds the
//                                    hi part (i < 16) or the lo part (i >= 16) of head 16 g + i % 16,
//                                    so both parts of a head sit in one warp's lane quarter.
//     O^T[D, heads] += X'^T . P^T     M = 128 dims (4 blocks), N = 64 heads, K = keys;
//                                    A = X'^T (MN-major: the same tile), B = P (K-major)
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
//   warps 0..3   softmax: thread (warp g, lane i) reads TMEM lane 32 g + i, the hi (i < 16) or
//                lo row of head 16 g + i % 16; the two partners swap half of their keys by
//                shuffles, so that each owns 16 keys of its head
//   warp 4       owns the tensor memory; lane 0 issues every MMA (the output product of tile t-1
//                as soon as its weights are written, else right after the logits of tile t)
//   warps 5..20  loaders: each resolves the pool rows of its 2 keys of every tile, keeps the raw
//                bytes of the next two tiles in flight in registers and converts a tile into the
//                fp16 operand in registers before its shared-memory stage (one of 2) is free; they
//                also build the query image at the start and write the partial outputs at the end
// Every wait on an mbarrier is bounded; a role that gives up raises an abort flag that the others
// poll, every issued MMA is drained before the epilogue and before the tensor memory is freed, and
// the split is then marked empty with CKV_DEV_TIMEOUT set.
//
// Start-up: with `early` set (a fused decode step, whose first kernel has already waited for the
// producers of the query and the lengths), the query image, the rotary table, the barriers and the
// tensor memory are set up before the kernel waits for its predecessor (the top-k selection or the
// append), so that work overlaps the predecessor's tail; everything that the predecessor writes
// (selected indices, counts, cache rows) is read after the wait.
//
// Each CTA takes keys_per_split consecutive keys of one request's key list (the window tokens
// [max(0, L-W), L) first, then the selected entries, or every entry of a dense layer) and writes
// an un-normalised partial: the maximum (base 2) and sum of every head, and O^T as fp16 rows of
// 64 heads per dim, each head's column divided by a power of two taken from its sum; the combine
// kernel merges the splits and applies the inverse rotation.

#include "ckv_internal.h"
#include "ckv_ptx.cuh"
#include "qimage.cuh"

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
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kMaxRopePairs = 256;
static_assert(kTile == 2 * kLoadWarps, "each loader warp stages two keys of a tile");
static_assert(kMaxTiles * 2 <= 32, "one lane of a loader warp per (tile, key) of the split");
static_assert(kH == 4 * kLoadWarps, "each loader warp builds the query image of four heads");

constexpr uint32_t kQChunk = 2 * kH * 128;             // 16 KB: 128 query rows of 64 dims
constexpr uint32_t kQBytes = kQChunk * kChunks;        // 128 KB
constexpr int kQTmemChunks = 6;                        // query chunks 0..5 live in tensor memory
constexpr uint32_t kXChunk = kTile * 128;              // 4 KB: one tile's keys of one 64-dim chunk
constexpr uint32_t kXStage = kXChunk * kChunks;        // 32 KB
constexpr int kXStages = 4;                            // operand stages (tile t in stage t % 4)
// Stages 2 j and 2 j + 1 form a pair of 64 KB: chunk c of stage 2 j + i at 8 KB c + 4 KB i, so that
// the 64 keys of both are one K-major operand of 64 rows (the logits of two tiles in one product).
constexpr uint32_t kXPairChunk = 2 * kXChunk;          // 8 KB: chunk stride inside a pair
constexpr uint32_t kPRegion = kH * 128;                // 8 KB: P of two tiles, row = head (64 B each)
constexpr int kPStages = 4;                            // P of tile t in stage t % 4
constexpr uint32_t kSCol = 0;                          // S stage s: columns 32 s
constexpr uint32_t kQCol = 64;                         // query chunk c < 6: columns 64 + 32 c (2 fp16 each)
constexpr uint32_t kOCol = 256;                        // O^T dims block m: columns 256 + 64 m
constexpr uint32_t kTmemCols = 512;
static_assert(kQCol + 32 * kQTmemChunks <= kOCol, "tensor memory columns");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRaiseLog2 = 8.0f * kLog2e;            // the running max moves past +8 nats
constexpr float kRaiseF = 16.0f;                       // the value bound moves past 16x

// shared memory carve-up (byte offsets from a 1024-aligned base). At the start, the operand stages
// hold query chunks 0..5 until they are moved into tensor memory; chunks 6, 7 stay in kOffQ.
constexpr uint32_t kOffX = 0;
constexpr uint32_t kOffQ = kOffX + kXStages * kXStage;
constexpr uint32_t kOffP = kOffQ + (kChunks - kQTmemChunks) * kQChunk;
constexpr uint32_t kOffKf = kOffP + (kPStages / 2) * kPRegion;  // float[4 stages][32]: key value factors
constexpr uint32_t kOffAlpha = kOffKf + kXStages * kTile * 4;  // float[2][64]: O^T rescale per head (by tile parity)
constexpr uint32_t kOffQs = kOffAlpha + 2 * kH * 4;      // float[64]: query scale g_h per head
constexpr uint32_t kOffInvSc = kOffQs + kH * 4;          // float[64]: 1 / (partial scale) per head
constexpr uint32_t kOffRope = kOffInvSc + kH * 4;        // double[256][2]: cos, sin per rotary pair
constexpr uint32_t kOffDummy = kOffRope + kMaxRopePairs * 16;  // 512 B: target of the epilogue's warm-up pass
constexpr uint32_t kOffMisc = kOffDummy + 512;            // int abort
constexpr uint32_t kOffBar = kOffMisc + 16;              // kNumBars mbarriers
constexpr uint32_t kOffTmem = kOffBar + 19 * 8;
constexpr uint32_t kSmemUsed = kOffTmem + 8;
constexpr int kSmemBytes = static_cast<int>(kSmemUsed) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kSmemUsed <= (1u << 18), "descriptor start addresses are 14 bits of 16-byte units");
static_assert(kOffQs % 16 == 0, "bulk-copy destination");

// mbarriers: xfull[4] (loaders -> MMA, softmax), xfree[4] (output product of the stage's tile
// done -> loaders, softmax), sfull[2] (logits done -> softmax), sfree[2] (softmax read the logits
// -> MMA), pfull[4] (softmax wrote P -> MMA), drain (every MMA done), qfull (the bulk copy of a
// query image built by the step's query pass has landed), qtmem (query chunks 0..5 are in tensor
// memory and the operand stages free)
constexpr int kBarXfull = 0, kBarXfree = 4, kBarSfull = 8, kBarSfree = 10, kBarPfull = 12, kBarDrain = 16,
              kBarQfull = 17, kBarQtmem = 18, kNumBars = 19;

// shared-memory address (from the base) of operand stage x (chunk 0)
static_assert(kOffX == 0, "stage addresses are offsets from the base");
__host__ __device__ constexpr uint32_t xstage_smem(int x) {
  return static_cast<uint32_t>(x >> 1) * (2 * kXStage) + static_cast<uint32_t>(x & 1) * kXChunk;
}

// shared-memory address (from the base) of query image chunk c
__host__ __device__ constexpr uint32_t qchunk_smem(int c) {
  return c < kQTmemChunks ? kOffX + static_cast<uint32_t>(c) * kQChunk
                          : kOffQ + static_cast<uint32_t>(c - kQTmemChunks) * kQChunk;
}

static_assert(kQTmemChunks * kQChunk <= kXStages * kXStage, "the stages hold the moved chunks at the start");
static_assert(kQBytes == kQImageBytes && kQChunk == kQiChunk && kH == kQiHeads && kD == kQiDim,
              "the query operand is laid out as qimage.cuh describes");

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

// D[tmem] (+)= A[smem] . B[smem]^T, both described by shared-memory matrix descriptors. The whole
// warp executes the call with the same operands (so that they stay warp-uniform); the thread that
// elect.sync picks (the same one on every call of a fully active warp) issues the MMA.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, q;\n .reg .b32 e;\n setp.ne.b32 p, %4, 0;\n elect.sync e|q, 0xffffffff;\n"
      " @q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem]^T: A is 128 lanes (rows) x 8 columns per K = 16 step, two fp16
// elements of the row's K per 32-bit column
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, q;\n .reg .b32 e;\n setp.ne.b32 p, %4, 0;\n elect.sync e|q, 0xffffffff;\n"
      " @q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// the elected thread's arrival on the mbarrier once every MMA it has issued so far has completed
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred q;\n .reg .b32 e;\n elect.sync e|q, 0xffffffff;\n"
      " @q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(bar)
      : "memory");
}

// shared-memory matrix descriptor: 128-byte swizzle, sm_100 descriptor version 1. The start
// address is bits 0..13 (16-byte units), so a descriptor of an address a few KB further on is this
// one plus the offset / 16 (no carry leaves the field below 256 KB).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// instruction descriptors, kind::f16 with fp32 accumulation and fp16 A and B:
//   logits: M = 128, N = 32 (one tile) or 64 (two), A and B K-major;
//   output: M = 128, N = 64, A MN-major, B K-major
constexpr uint32_t kIdescS = (1u << 4) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescS2 = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);  // two tiles
constexpr uint32_t kIdescPV = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24) | (1u << 15);

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  tmem_wait_ld();
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 consecutive columns of this warp's lane quarter; the caller waits (tmem_wait_ld)
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
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

// loads of key bytes, each read once: not kept in L1 (which then holds the registers that the
// kernel spills)
__device__ __forceinline__ uint2 ldg_stream2(const void* ptr) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream1(const void* ptr) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream_u8(const void* ptr) {
  uint16_t v;
  asm("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(ptr));
  return v;
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
    const uint2 v = ldg_stream2(reinterpret_cast<const uint2*>(p.win_codes + row * p.win_row_bytes) + g);
    r.a.x = v.x;
    r.a.y = v.y;
    return r;
  }
  const uint8_t* base = p.comp_codes + row * p.comp_row_bytes;
  if constexpr (CT == CKV_BF16) {
    r.a = ldg_stream(reinterpret_cast<const uint4*>(base) + g);
  } else {
    r.a.x = ldg_stream1(reinterpret_cast<const uint32_t*>(base) + g);
    r.s = ldg_stream_u8(p.comp_scales + row * (kD / 16) + (g >> 1));
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
  int L, n_c, n_sel, n_win, n_keys;  // key counts fit in int: at most max_seq_len + W
};

// One key's two granules (dims 8 lane .. 8 lane + 7 and 256 + 8 lane ..) as fp16 after the key's
// power-of-two normalisation, and the key's value factor (0 marks an absent key, whose row is
// zeros).
template <int CT>
__device__ __forceinline__ float convert_key(const Raw (&r)[2], bool win, bool present, float tsc,
                                             uint4 (&o)[2]) {
  float v[2][8];
  decode_granule<CT>(r[0], win, v[0]);
  decode_granule<CT>(r[1], win, v[1]);
  uint32_t mb = 0;
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int k = 0; k < 8; ++k) mb = max(mb, __float_as_uint(v[g][k]) & 0x7fffffffu);
  const int sh = norm_shift(__reduce_max_sync(0xffffffffu, mb));
  const float up = exp2i(sh);
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    o[g].x = pack_f32x2(v[g][0] * up, v[g][1] * up);
    o[g].y = pack_f32x2(v[g][2] * up, v[g][3] * up);
    o[g].z = pack_f32x2(v[g][4] * up, v[g][5] * up);
    o[g].w = pack_f32x2(v[g][6] * up, v[g][7] * up);
  }
  return present ? tsc * exp2i(-sh) : 0.f;
}

// ------------------------------------------------------------------------------------ kernel

// early: the query and the lengths may be read before waiting for the previous kernel (see the
// file comment); prepared: the step's query pass already wrote the cos/sin table into ws.rope and
// the query image into ws.qimage / ws.qscale, which are then bulk-copied instead of built here;
// warm: run the warm-up pass described below (an early launch whose CTAs all run in one wave and
// whose previous kernel runs a while)
template <int CT>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(
    LayerParams p, const int32_t* seq_len, int max_seq_len, const float* q, const int32_t* idx,
    const int32_t* cnt, int idx_stride, AttnWs ws, uint32_t* status, bool early, bool prepared, bool warm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(base);
  float* kf = reinterpret_cast<float*>(base + kOffKf);
  float* alpha_sm = reinterpret_cast<float*>(base + kOffAlpha);
  float* qs = reinterpret_cast<float*>(base + kOffQs);
  float* inv_sc = reinterpret_cast<float*>(base + kOffInvSc);
  double* rope_sm = reinterpret_cast<double*>(base + kOffRope);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc);
  auto bar = [&](int i) { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffTmem);

  // requests on x so that the first split of every request is launched first and the splits that
  // find no keys (short requests of a mixed batch) come last
  const int b = blockIdx.x, split = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int li = warp - kFirstLoadWarp;  // loader index (warps >= kFirstLoadWarp)
  const int k_begin = split * ws.keys_per_split;

  auto init_barriers = [&]() {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(bar(kBarXfull + s), kLoadWarps);
      mbar_init(bar(kBarXfree + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSfull + s), 1);
      mbar_init(bar(kBarSfree + s), kSoftThreads);
    }
    for (int s = 0; s < kPStages; ++s) mbar_init(bar(kBarPfull + s), kSoftThreads);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarQfull), 1);
    mbar_init(bar(kBarQtmem), kSoftThreads);
  };
  if (tid == 0) {
    init_barriers();
    *abort_flag = 0;
  }

  // ---- start-up that reads only the query and the length: the tensor memory, the rotary table
  //      and the query image. Returns false (uniformly) when the split holds no key whatever the
  //      selection, before anything is allocated.
  Keys kl{};
  // a loader lane's key: tile kt = lane >> 1, key 2 li + (lane & 1) of the tile
  const int kt = lane >> 1;
  const int my_k = k_begin + kt * kTile + 2 * li + (lane & 1);
  const bool my_slot = warp >= kFirstLoadWarp && kt < kMaxTiles && my_k - k_begin < ws.keys_per_split;
  long long my_row = -1;
  int my_win = 0;
  // rows that depend only on the length and the block tables: window tokens, and every entry of a
  // dense layer (a selected entry's row waits for the selection)
  auto resolve_static = [&]() {
    if (!my_slot) return;
    if (my_k < kl.n_win) {
      my_row = win_row(p, b, kl.L - kl.n_win + my_k, status);
      my_win = 1;
    } else if (!idx && my_k - kl.n_win < kl.n_c) {
      my_row = comp_row(p, b, my_k - kl.n_win, status);
    }
  };
  auto startup = [&]() -> bool {
    kl.L = seq_len[b];
    const bool live = kl.L >= 1 && kl.L <= max_seq_len;  // a bad length is flagged by the combine
    kl.n_c = live ? kl.L / p.r : 0;
    kl.n_win = live ? min(p.W, kl.L) : 0;
    const int most = kl.n_win + (idx ? min(kl.n_c, idx_stride) : kl.n_c);
    if (k_begin >= most) return false;
    if (warp == kMmaWarp) tmem_alloc(sb + kOffTmem, kTmemCols);
    if (prepared) {
      if (warp >= kFirstLoadWarp) resolve_static();
    } else {
      // query rows of heads 4 li .. 4 li + 3, two at a time: lane l holds dims 16 l .. 16 l + 15
      // of each; the first two heads' loads are in flight while the rotary table is computed
      float4 qv[2][4];
      const float* qb = q + static_cast<int64_t>(b) * kH * kD;
      auto load_q = [&](int h0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            qv[hh][k] = __ldg(reinterpret_cast<const float4*>(qb + static_cast<int64_t>(h0 + hh) * kD + 16 * lane) + k);
      };
      if (warp >= kFirstLoadWarp) {
        load_q(4 * li);
        resolve_static();
      } else if (warp < kSoftWarps) {
        // cos, sin of every rotary pair at the query position L-1 (fp64 angles), one pair per thread
        for (int i = tid; i < p.d_r / 2; i += kSoftThreads) {
          double sn, cs;
          rope_sincos(static_cast<double>(kl.L - 1) * rope_inv_freq(p, i), &sn, &cs);
          rope_sm[2 * i] = cs;
          rope_sm[2 * i + 1] = sn;
        }
      }
      __syncthreads();  // the rotary table
      if (warp >= kFirstLoadWarp) {
        const int first_rope = (kD - p.d_r) / 2;
#pragma unroll
        for (int hq = 0; hq < 4; ++hq) {
          const int hh = hq & 1, h = 4 * li + hq;
          if (hq == 2) load_q(4 * li + 2);
          float x[16];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[4 * k] = qv[hh][k].x;
            x[4 * k + 1] = qv[hh][k].y;
            x[4 * k + 2] = qv[hh][k].z;
            x[4 * k + 3] = qv[hh][k].w;
          }
          uint4 hi[2], lo[2];
          const float sc = qimage_head(x, lane, first_rope, rope_sm, hi, lo);
          if (lane == 0) qs[h] = sc;
          // granules 2 lane, 2 lane + 1 lie in image chunk lane / 4
          const uint32_t qa = sb + qchunk_smem(lane >> 2) - static_cast<uint32_t>(lane >> 2) * kQChunk;
          const int rh = qimage_row(h, 0), rl = qimage_row(h, 1);
          st_shared_v4(qa + qimage_offset(rh, 2 * lane), hi[0]);
          st_shared_v4(qa + qimage_offset(rh, 2 * lane + 1), hi[1]);
          st_shared_v4(qa + qimage_offset(rl, 2 * lane), lo[0]);
          st_shared_v4(qa + qimage_offset(rl, 2 * lane + 1), lo[1]);
        }
      }
    }
    fence_proxy_async();  // the barriers' initialisation and the query image, for the async proxy
    tc_fence_before();
    __syncthreads();      // the query image, its scales and the tensor memory address
    tc_fence_after();
    return true;
  };

  if (!early) {  // the query and the lengths are read after the previous kernel is done
    griddep_wait();
    griddep_launch();
  }
  if (!startup()) return;

  // Pass 0 (with `warm`) is a warm-up, run while the previous kernel is still running: the loaders (on absent keys), the MMA issuer, the softmax warps and the partial-output
  // code run once on whatever the memories hold, all at the same time, with the loaders' operand
  // stores and the partial-output traffic aimed at a 512-byte scratch area, no global store and no
  // wait for or arrival on any barrier; only the issuer waits for its MMAs. Each SM runs one CTA of this kernel, so without it the real pass (pass 1)
  // would fetch that code cold on its critical path (CTAs of later waves find it warm). The
  // barriers are initialised afresh between the passes.
  int64_t slot = 0;
  bool aborted = false;
#pragma unroll 1
  for (int pass = warm ? 0 : 1; pass < 2; ++pass) {
  const bool dry = pass == 0;
  int n_tiles;
  int32_t my_ent = -1;
  if (dry) {
    // as many tiles as the split can hold at most (from the length alone), up to 2
    const int most = kl.n_win + (idx ? min(kl.n_c, idx_stride) : kl.n_c);
    const int nk_max = min(most - k_begin, ws.keys_per_split);
    n_tiles = min(2, (nk_max + kTile - 1) / kTile);
  } else {
    if (early) {
      griddep_wait();
      griddep_launch();
    }
    if (prepared && warp == kMmaWarp && lane == 0) {  // the query image and its scales, from L2
      const uint8_t* img = ws.qimage + static_cast<int64_t>(b) * kQImageBytes;
      mbar_expect_tx(bar(kBarQfull), kQBytes + kH * 4);
      for (int c = 0; c < kChunks; ++c) bulk_g2s(sb + qchunk_smem(c), img + c * kQChunk, kQChunk, bar(kBarQfull));
      bulk_g2s(sb + kOffQs, ws.qscale + static_cast<int64_t>(b) * kH, kH * 4, bar(kBarQfull));
    }
    // the selected entry of a loader lane's key, loaded before the count is known (any position
    // below the index stride is readable)
    if (idx && my_slot && my_k >= kl.n_win && my_k - kl.n_win < idx_stride)
      my_ent = idx[static_cast<int64_t>(b) * idx_stride + (my_k - kl.n_win)];
    kl.n_sel = kl.n_c == 0 ? 0 : idx ? min(max(cnt[b], 0), idx_stride) : kl.n_c;
    kl.n_keys = kl.n_win + kl.n_sel;
    if (k_begin >= kl.n_keys) {  // the selection left this split empty (uniform; no MMA issued)
      if (warp == kMmaWarp) {
        if (prepared) mbar_wait(bar(kBarQfull), 0);  // no copy in flight at the exit
        tmem_dealloc(*tmem_slot, kTmemCols);
      }
      return;
    }
    const int nk = min(kl.n_keys - k_begin, ws.keys_per_split);
    n_tiles = (nk + kTile - 1) / kTile;
    slot = (static_cast<int64_t>(b) * ws.splits + split) * kH;
    if (split == 0 && !prepared && tid < p.d_r) {  // the table for the combine's inverse rotation
      ws.rope[static_cast<int64_t>(b) * (p.d_r / 2 + 1) * 2 + tid] = rope_sm[tid];
    }
  }
  const uint32_t tmem = *tmem_slot;

  if (warp == kMmaWarp) {
    // ---------------- MMAs (the whole warp runs this; one elected lane issues): the logits of tile t, and the
    //                  output product of tile t-1 (before the logits of tile t when its weights are
    //                  already written)
    const uint64_t dq = sdesc(sb + kOffQ, 16, 1024);
    const uint64_t dx = sdesc(sb + kOffX, 16, 1024);
    const uint64_t da = sdesc(sb + kOffX, kXPairChunk, 1024);
    const uint64_t dp = sdesc(sb + kOffP, 16, 1024);
    // One issue site for each product keeps the code that runs once per CTA (cold in the
    // instruction cache) short: S(t) then the output product of tile t-1, or the other way round
    // when the weights of tile t-1 are already written.
    bool issued = false;
    // the failure-path hook: a wait on the drain barrier, which nothing completes before the first
    // MMA, runs out and the CTA takes its failure path
    bool ok = dry || g_attn_forced_timeout != b || wait_or_abort(bar(kBarDrain), 0, abort_flag, 16);
    if (prepared && !dry) ok = __all_sync(0xffffffffu, wait_or_abort(bar(kBarQfull), 0, abort_flag)) && ok;
    ok = ok && (dry || __all_sync(0xffffffffu, wait_or_abort(bar(kBarQtmem), 0, abort_flag)));  // query chunks 0..5 moved
    int g = 0, u = 0;  // the next logits group (tiles 2 g, 2 g + 1) and the next output product
#pragma unroll 1
    while (ok && u < n_tiles) {
      const int t0 = 2 * g;
      bool pv;
      if (t0 >= n_tiles) {
        pv = true;
      } else if (u >= t0) {
        pv = false;  // the logits of tile u come first
      } else if (u < t0 - 2) {
        pv = true;   // tiles t0, t0 + 1 write the P stages of tiles t0 - 4, t0 - 3
      } else {       // either: the output product when its weights are already written
        pv = !dry && __all_sync(0xffffffffu, mbar_test_wait(bar(kBarPfull + (u & (kPStages - 1))), static_cast<uint32_t>(u >> 2) & 1u));
      }
      if (pv) {
        const int x = u & (kXStages - 1);
        ok = dry || __all_sync(0xffffffffu, wait_or_abort(bar(kBarPfull + (u & (kPStages - 1))),
                                                           static_cast<uint32_t>(u >> 2) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint64_t ax = da + (xstage_smem(x) >> 4);
        const uint64_t bp = dp + (((u >> 1) & 1) * kPRegion >> 4) + 4 * (u & 1);
#pragma unroll 1
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
          for (int m = 0; m < 4; ++m)
            mma_f16(tmem + kOCol + 64 * m, ax + m * (2 * kXPairChunk >> 4) + kk * (2048 >> 4), bp + 2 * kk, kIdescPV,
                    (u > 0 || kk > 0) ? 1u : 0u);
        }
        if (!dry) mma_commit(bar(kBarXfree + x));
        ++u;
      } else {
        // the logits of tiles t0 and t0 + 1 (stages of one pair) in one N = 64 product, or of the
        // last tile alone; S stage i gets tile t0 + i
        const bool two = t0 + 1 < n_tiles;
        const int x0 = t0 & (kXStages - 1);
        ok = dry || wait_or_abort(bar(kBarXfull + x0), static_cast<uint32_t>(t0 >> 2) & 1u, abort_flag) &&
             (!two || wait_or_abort(bar(kBarXfull + x0 + 1), static_cast<uint32_t>((t0 + 1) >> 2) & 1u, abort_flag)) &&
             (g == 0 || wait_or_abort(bar(kBarSfree + 0), static_cast<uint32_t>(g - 1) & 1u, abort_flag)) &&
             (g == 0 || !two || wait_or_abort(bar(kBarSfree + 1), static_cast<uint32_t>(g - 1) & 1u, abort_flag));
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint64_t bx = dx + (xstage_smem(x0) >> 4);
        const uint32_t idesc = two ? kIdescS2 : kIdescS;
        // K = 0 .. 383 with the query rows in tensor memory, K = 384 .. 511 from shared memory
#pragma unroll 1
        for (int c = 0; c < kQTmemChunks; ++c) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16_ts(tmem + kSCol, tmem + kQCol + 32 * c + 8 * ks, bx + c * (kXPairChunk >> 4) + 2 * ks, idesc,
                       (c | ks) != 0);
        }
#pragma unroll
        for (int c = kQTmemChunks; c < kChunks; ++c) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tmem + kSCol, dq + (c - kQTmemChunks) * (kQChunk >> 4) + 2 * ks,
                    bx + c * (kXPairChunk >> 4) + 2 * ks, idesc, 1u);
        }
        if (!dry) {
          mma_commit(bar(kBarSfull + 0));
          if (two) mma_commit(bar(kBarSfull + 1));
        }
        issued = true;
        ++g;
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    if (issued) {  // every MMA issued has completed before O^T is read or the memory freed
      mma_commit(bar(kBarDrain));
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarDrain), 0)) && lane == 0) *abort_flag = 1;
    }
  } else if (warp < kSoftWarps) {
    // ---------------- softmax: thread (warp g, lane i) = TMEM lane 32 g + i: head h = 16 g + i % 16,
    //                  hi (i < 16) or lo row; after the swap it owns keys kb .. kb + 15 of head h
    const bool hi_row = lane < 16;
    const int h = 16 * warp + (lane & 15);
    const int kb = hi_row ? 0 : 16;
    bool ok = true;
    if (prepared && !dry)  // one decision for the four warps, which share a named barrier below
      ok = bar_red<true>(1, kSoftThreads, __all_sync(0xffffffffu, wait_or_abort(bar(kBarQfull), 0, abort_flag)));
    if (ok) {
      // query chunks 0..5 into tensor memory: thread (warp w, lane l) moves row 32 w + l, granule g
      // of chunk c (dims 64 c + 8 g ..) to columns kQCol + 32 c + 4 g .. + 3
      const int r = 32 * warp + lane;
#pragma unroll 1
      for (int c = 0; c < kQTmemChunks; ++c) {
        uint32_t v[32];
        const uint32_t row = sb + qchunk_smem(c) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v[4 * g]), "=r"(v[4 * g + 1]), "=r"(v[4 * g + 2]), "=r"(v[4 * g + 3])
                       : "r"(row + (static_cast<uint32_t>(g ^ (r & 7)) << 4)));
        tmem_st32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + kQCol + 32 * c, v);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      if (!dry) mbar_arrive(bar(kBarQtmem));  // also releases the operand stages to the loaders
    }
    const float ch = qs[h] * p.sm_scale * kLog2e;
    float m_run = -INFINITY, F_run = 0.f, l_part = 0.f;
#pragma unroll 1
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int s = t & 1, x = t & (kXStages - 1);
      const bool got = dry || __all_sync(0xffffffffu, wait_or_abort(bar(kBarSfull + s), static_cast<uint32_t>(t >> 1) & 1u, abort_flag) &&
                                                          wait_or_abort(bar(kBarXfull + x), static_cast<uint32_t>(t >> 2) & 1u, abort_flag));
      bool rescale_me = false;
      if (got) {
        tc_fence_after();
        uint32_t raw[32];
        tmem_ld32_async(tmem + (static_cast<uint32_t>(32 * warp) << 16) + kSCol + 32 * s, raw);
        tmem_wait_ld();
        tc_fence_before();
        if (!dry) mbar_arrive(bar(kBarSfree + s));
        // swap with the partner row (lane ^ 16): a hi row hands over keys 16..31, a lo row keys 0..15
        float lg[16];
        float mx = -INFINITY, fmx = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float own = __uint_as_float(hi_row ? raw[i] : raw[16 + i]);
          const float give = __uint_as_float(hi_row ? raw[16 + i] : raw[i]);
          const float sv = own + __shfl_xor_sync(0xffffffffu, give, 16);
          const float f = kf[x * kTile + kb + i];
          lg[i] = f > 0.f ? sv * f * ch : -INFINITY;
          mx = fmaxf(mx, lg[i]);
          fmx = fmaxf(fmx, f);
        }
        const float mt = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float ft = fmaxf(fmx, __shfl_xor_sync(0xffffffffu, fmx, 16));
        float m_new = m_run, F_new = F_run;
        if (mt > -INFINITY && (m_run == -INFINITY || mt > m_run + kRaiseLog2)) m_new = mt;
        if (ft > 0.f && ft > kRaiseF * F_run) F_new = pow2_ceil(ft);
        const float a_l = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
        rescale_me = t > 0 && (m_new != m_run || F_new != F_run);
        if (hi_row) alpha_sm[s * kH + h] = F_run > 0.f ? a_l * (F_run / F_new) : 0.f;
        float psum = 0.f;
        uint32_t packed[8];
        const float inv_F = F_new > 0.f ? 1.f / F_new : 0.f;  // a power of two: exact
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float p0 = lg[i] > -INFINITY ? exp2f(lg[i] - m_new) : 0.f;
          const float p1 = lg[i + 1] > -INFINITY ? exp2f(lg[i + 1] - m_new) : 0.f;
          psum += p0 + p1;
          const float f0 = kf[x * kTile + kb + i], f1 = kf[x * kTile + kb + i + 1];
          packed[i >> 1] = pack_f32x2(p0 * f0 * inv_F, p1 * f1 * inv_F);
        }
        l_part = l_part * a_l + psum;
        m_run = m_new;
        F_run = F_new;
        const uint32_t prow = sb + kOffP + static_cast<uint32_t>((t >> 1) & 1) * kPRegion + static_cast<uint32_t>(h) * 128u;
        const int g0 = 4 * s + kb / 8;
        st_shared_v4(prow + (static_cast<uint32_t>(g0 ^ (h & 7)) << 4),
                     make_uint4(packed[0], packed[1], packed[2], packed[3]));
        st_shared_v4(prow + (static_cast<uint32_t>((g0 + 1) ^ (h & 7)) << 4),
                     make_uint4(packed[4], packed[5], packed[6], packed[7]));
      }
      // one barrier per tile in the common case: a raised bound or a failed wait anywhere takes
      // the slow path (the rescale factors are visible after it)
      if (bar_red<false>(1, kSoftThreads, rescale_me || !got)) {
        ok = bar_red<true>(1, kSoftThreads, got);
        if (!ok) break;
        // O^T holds the output products of tiles 0 .. t-1: wait for the last of them, then scale
        // column (head) c of every dims block of this warp's lane quarter by alpha[c]
        const int u = t - 1;
        const bool done = u < 0 || dry || __all_sync(0xffffffffu, wait_or_abort(bar(kBarXfree + (u & (kXStages - 1))),
                                                                          static_cast<uint32_t>(u >> 2) & 1u, abort_flag));
        if (done && u >= 0) {
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
            for (int c0 = 0; c0 < kH; c0 += 8) {
              const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + kOCol + 64 * m + c0;
              uint32_t o[8];
              tmem_ld8(ta, o);
#pragma unroll
              for (int c = 0; c < 8; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha_sm[s * kH + c0 + c]);
              tmem_st8(ta, o);
            }
          }
        }
        ok = bar_red<true>(1, kSoftThreads, done);
        if (!ok) break;
      }
      if (!dry) {
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(kBarPfull + (t & (kPStages - 1))));
      }
    }
    if (!ok) {
      *abort_flag = 1;
    } else {
      // the head's sum: hi row plus its lo partner (they share the maximum). O^T's column of the
      // head is below 2^13 l (|x'| < 2^9, P_j <= 16 p_j), so dividing it by a power of two
      // sc >= l / 4 keeps it below 2^15 in fp16.
      const float l = l_part + __shfl_xor_sync(0xffffffffu, l_part, 16);
      if (hi_row) {
        const float sc = l > 0.f ? pow2_ceil(l * 1.001f) * 0.25f : 1.f;
        inv_sc[h] = 1.f / sc;  // exact: a power of two
        if (!dry) {
          reinterpret_cast<float2*>(ws.part_ml)[slot + h] = make_float2(m_run, l);
          ws.part_sc[slot + h] = sc * F_run;
        }
      }
    }
  } else {
    // ---------------- loaders: lane j holds the row of key 2 li + (j & 1) of tile j >> 1
    if (!dry && idx && my_slot && my_k >= kl.n_win && my_k < kl.n_keys) {
      if (my_ent < 0 || my_ent >= kl.n_c) {
        atomicOr(status, CKV_DEV_BAD_INDEX);
      } else {
        my_row = comp_row(p, b, my_ent, status);
      }
    }
    // the warm-up's keys are all absent (their operand rows are zeros and nothing is loaded)
    const long long row_use = dry ? -1ll : my_row;
    const int win_use = dry ? 0 : my_win;
    float my_tscale = 1.f;
    if (win_use && row_use >= 0) my_tscale = p.win_scales[row_use];  // consumed at the conversion
    auto row_of = [&](int t, int u, bool* win) -> int64_t {
      const int src = 2 * t + u;
      *win = __shfl_sync(0xffffffffu, win_use, src) != 0;
      return static_cast<int64_t>(__shfl_sync(0xffffffffu, row_use, src));
    };
    auto issue = [&](int t, Raw (&r)[2][2]) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        bool win;
        const int64_t row = row_of(t, u, &win);
        r[u][0] = load_granule<CT>(p, row, win, lane);
        r[u][1] = load_granule<CT>(p, row, win, lane + 32);
      }
    };
    Raw ring[2][2][2];  // [tile parity][key u][granule lane, lane + 32]
    issue(0, ring[0]);
    if (n_tiles > 1) issue(1, ring[1]);
    // tile t: convert its bytes in registers, put the loads of tile t+2 in flight in the freed
    // slot, then wait until the output product of tile t-2 has released the stage and store
    auto stage = [&](int t, Raw (&r)[2][2]) -> bool {
      const int x = t & (kXStages - 1);
      uint4 cv[2][2];
      float kfv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        bool win;
        const int64_t row = row_of(t, u, &win);
        const float tsc = __shfl_sync(0xffffffffu, my_tscale, 2 * t + u);
        kfv[u] = convert_key<CT>(r[u], win, row >= 0, tsc, cv[u]);
      }
      if (t + 2 < n_tiles) issue(t + 2, r);
      // the stage is free once the output product of tile t - 4 is done (tiles 0..2 go where the
      // query chunks were: wait until they are in tensor memory)
      const bool free_ = dry || (t >= kXStages ? wait_or_abort(bar(kBarXfree + x), static_cast<uint32_t>((t >> 2) - 1) & 1u, abort_flag)
                                               : t > 0 || wait_or_abort(bar(kBarQtmem), 0, abort_flag));
      if (!__all_sync(0xffffffffu, free_)) return false;
      const uint32_t xs = sb + (dry ? kOffDummy : xstage_smem(x));
      const uint32_t omask = dry ? 511u : 0xffffffffu;  // the warm-up writes to the scratch area
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int key = 2 * li + u;
        st_shared_v4(xs + (swz(kXPairChunk, key, lane) & omask), cv[u][0]);
        st_shared_v4(xs + (swz(kXPairChunk, key, lane + 32) & omask), cv[u][1]);
        if (lane == 0) kf[x * kTile + key] = kfv[u];
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0 && !dry) mbar_arrive(bar(kBarXfull + x));
      return true;
    };
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; t += 2) {
      ok = stage(t, ring[0]);
      if (ok && t + 1 < n_tiles) ok = stage(t + 1, ring[1]);
    }
    if (!ok) *abort_flag = 1;
  }

  // ---------------- partial outputs: loader warp li reads TMEM lane quarter g = warp % 4 of dims
  //                  block m = li / 4, i.e. dims d0 .. d0 + 31 with d0 = 128 m + 32 g (lane = dim),
  //                  all 64 heads, and writes the rows of 64 fp16 values (head h divided by its
  //                  scale) to part_h[slot][d][h]: first into the free operand stage (16-byte
  //                  chunks swizzled by the row so that the lanes hit distinct banks), then from
  //                  there with stores of 512 contiguous bytes per instruction (in the warm-up pass
  //                  the loaders run this at once, with the shared-memory traffic aimed at a
  //                  512-byte scratch area and no store).
  if (!dry) {
    __syncthreads();  // every role done; the MMA thread has drained the tensor pipe
    aborted = *abort_flag != 0;
  }
  if (!aborted && warp >= kFirstLoadWarp) {
    tc_fence_after();
    const int g = warp & 3, m = li >> 2;
    const int d0 = 128 * m + 32 * g;
    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * g) << 16) + kOCol + 64 * m;
    const uint32_t rmask = dry ? 3u : 31u;
    const uint32_t stage = sb + (dry ? kOffDummy : kOffX + static_cast<uint32_t>(d0) * 128u);
    const uint32_t my_row = stage + (static_cast<uint32_t>(lane) & rmask) * 128u;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      uint32_t o[32];
      tmem_ld32_async(ta + 32 * half, o);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * half + j;  // 16-byte chunk: heads 8 c .. 8 c + 7
        const float4 s0 = *reinterpret_cast<const float4*>(inv_sc + 8 * c);
        const float4 s1 = *reinterpret_cast<const float4*>(inv_sc + 8 * c + 4);
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          w[k] = pack_f32x2(__uint_as_float(o[8 * j + 2 * k]) * sv[2 * k], __uint_as_float(o[8 * j + 2 * k + 1]) * sv[2 * k + 1]);
        st_shared_v4(my_row + ((static_cast<uint32_t>(c) ^ (static_cast<uint32_t>(lane) & 7u)) << 4),
                     make_uint4(w[0], w[1], w[2], w[3]));
      }
    }
    __syncwarp();
    // copy-out: instruction k moves rows 4 k .. 4 k + 3 (lane l: row 4 k + l / 8, chunk l % 8)
    uint4* dst = reinterpret_cast<uint4*>(ws.part_h + (slot * kD + static_cast<int64_t>(d0) * kH));
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
      const uint32_t r = static_cast<uint32_t>(4 * k + (lane >> 3)), c = static_cast<uint32_t>(lane & 7);
      uint4 v;
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(stage + (r & rmask) * 128u + ((c ^ (r & 7u)) << 4))
                   : "memory");
      if (!dry) dst[r * 8 + c] = v;
    }
  }
  if (dry) {
    // every role is done and the tensor pipe drained: fresh barriers for the real pass (an abort
    // raised by the warm-up stays raised)
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      for (int i = 0; i < kNumBars; ++i) mbar_inval(bar(i));
      init_barriers();
    }
    __syncthreads();
    tc_fence_after();
  }
  }  // pass
  if (aborted) {
    if (tid == 0) atomicOr(status, CKV_DEV_TIMEOUT);
    if (tid < kH) reinterpret_cast<float2*>(ws.part_ml)[slot + tid] = make_float2(-INFINITY, 0.f);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    if (prepared) mbar_wait(bar(kBarQfull), 0);  // no copy in flight at the exit (also after an abort)
    tc_fence_after();
    tmem_dealloc(*tmem_slot, kTmemCols);
  }
}

template <int CT>
cudaError_t launch_tc(const LayerParams& p, int batch, const int32_t* seq_len, int max_seq_len,
                      const float* q, const int32_t* idx, const int32_t* cnt, int idx_stride,
                      const AttnWs& ws, uint32_t* status, cudaStream_t stream, bool early, bool prepared) {
  auto kern = attn_tc_kernel<CT>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(batch, ws.splits);
  // the warm-up pays when it overlaps a previous kernel that runs a while (the top-k selection of a
  // sparse layer) and every CTA is in the first wave
  const bool warm = early && idx != nullptr && static_cast<int64_t>(batch) * ws.splits <= sm_count();
  return launch_kernel(kern, grid, dim3(kThreads), kSmemBytes, stream, p, seq_len, max_seq_len, q, idx,
                       cnt, idx_stride, ws, status, early, prepared && ws.qimage && ws.qscale, warm);
}

}  // namespace

// bf16 and NVFP4 compressed caches with an FP8 window at H = 64, D = 512. fp32 caches stay on the
// CUDA-core path: fp32 arithmetic attends them as stored.
bool attention_tc_supported(const LayerParams& p) {
  return p.H == kH && p.D == kD && p.d_r <= 2 * kMaxRopePairs &&
         (p.comp_dtype == CKV_BF16 || p.comp_dtype == CKV_NVFP4) && p.win_dtype == CKV_FP8_E4M3;
}

// Keys per split: t tiles of 32 keys, t in 1 .. 16, minimising (waves of one CTA per SM) x
// (t + 8), the 8 standing for a split's fixed cost in tiles (start-up from a cold instruction
// cache, key resolution, the partial write; measured on the 64-request mixed step: a cost of 2
// gave 260.5 us per step, 8 to 16 gave 252.7; single-wave launches choose the same t either way).
int attention_tc_keys_per_split(int batch, int64_t max_keys) {
  const int64_t tiles = max_keys > 0 ? (max_keys + kTile - 1) / kTile : 1;
  const int64_t sms = sm_count();
  int best_t = 1;
  int64_t best = -1;
  for (int t = 1; t <= kMaxTiles; ++t) {
    const int64_t ctas = static_cast<int64_t>(batch) * ((tiles + t - 1) / t);
    const int64_t cost = ((ctas + sms - 1) / sms) * (t + 8);
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
                                uint32_t* status, cudaStream_t stream, bool early, bool prepared) {
  if (p.win_dtype != CKV_FP8_E4M3) return cudaErrorInvalidValue;
  if (p.comp_dtype == CKV_BF16)
    return launch_tc<CKV_BF16>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream,
                               early, prepared);
  if (p.comp_dtype == CKV_NVFP4)
    return launch_tc<CKV_NVFP4>(p, batch, seq_len, max_seq_len, q, idx, cnt, idx_stride, ws, status, stream,
                                early, prepared);
  return cudaErrorInvalidValue;
}

}  // namespace ckv

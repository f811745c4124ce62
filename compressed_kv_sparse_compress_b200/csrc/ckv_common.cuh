// Device helpers shared by the kernels of libckv: number formats, rotary embedding, paged
// addressing and the layer parameter block. sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ckv.h"

namespace ckv {

constexpr int kBlockTokens = 256;  // fixed logical block of 256 positions

// Everything a kernel needs about one layer, passed by value.
struct LayerParams {
  int H, D, d_r, r, W;
  int comp_dtype, win_dtype;
  int epb;               // entries per pool block = 256 / r
  int comp_row_bytes;    // code bytes per compressed entry
  int win_row_bytes;     // code bytes per window token
  float sm_scale;
  double rope_base;
  uint8_t* comp_codes;
  uint8_t* comp_scales;  // NVFP4: D/16 bytes per entry
  uint8_t* win_codes;
  float* win_scales;     // FP8: one per token
  float* res_kv;         // [B][r][D]
  float* res_logit;      // [B][r]
  const int32_t* comp_table;
  const int32_t* win_table;
  int table_stride;
  int comp_blocks, win_blocks;
  // base^(-2i/d_r) for rotary pair i, computed on the host in fp64 (d_r <= 2 * kRopeTable;
  // larger rotary widths compute it on the device)
  static constexpr int kRopeTable = 64;
  double inv_freq[kRopeTable];
};

// ------------------------------------------------------------------------------- formats

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ uint8_t f32_to_e4m3_satfinite(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint8_t f32_to_e2m1_satfinite(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest)) & 0xF;
}

// two e2m1 codes (low nibble = first element) -> half2 (exact)
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint8_t byte) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(byte), __NV_E2M1);
  return __half2(r);
}

// ------------------------------------------------------------------------------- rotary

// inverse frequency of rotary pair i: base^(-2i/d_r), fp64
__device__ __forceinline__ double rope_inv_freq(int i, int d_r, double base) {
  return pow(base, -(2.0 * i) / static_cast<double>(d_r));
}

// the same, from the layer's host-computed table when it holds pair i
__device__ __forceinline__ double rope_inv_freq(const LayerParams& p, int i) {
  return i < LayerParams::kRopeTable ? p.inv_freq[i] : rope_inv_freq(i, p.d_r, p.rope_base);
}

// sin and cos of a rotary angle (fp64, |angle| up to ~2^40): the angle is first reduced by the
// nearest multiple k of 2 pi with 2 pi split into a head and a tail double (Cody and Waite's
// additive reduction), so that the library's sincos sees |r| <= pi, its short path. The reduction
// error is about k * 2^-106, far below the fp64 rounding of the angle itself.
__device__ __forceinline__ void rope_sincos(double angle, double* sn, double* cs) {
  constexpr double kTwoPiHi = 6.283185307179586;        // the double nearest 2 pi
  constexpr double kTwoPiLo = 2.4492935982947064e-16;   // 2 pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  const double k = rint(angle * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, angle);
  r = fma(-k, kTwoPiLo, r);
  sincos(r, sn, cs);
}

// rotate the pair (a, b) by angle pos * inv_freq (inverse: by the negative angle), in fp64
__device__ __forceinline__ void rope_rotate_pair(double a, double b, double pos, double inv_freq,
                                                 bool inverse, double* oa, double* ob) {
  double s, c;
  sincos(pos * inv_freq, &s, &c);
  if (inverse) s = -s;
  *oa = a * c - b * s;
  *ob = a * s + b * c;
}

// ------------------------------------------------------------------------------- paging

// Pool row of compressed entry i of request b, or -1 (status bit set) when unmapped.
__device__ __forceinline__ int64_t comp_row(const LayerParams& p, int b, int64_t entry,
                                            uint32_t* status) {
  const int64_t lblk = (entry * p.r) >> 8;  // r and 256/r are powers of two
  const int32_t phys = p.comp_table[static_cast<int64_t>(b) * p.table_stride + lblk];
  if (phys < 0 || phys >= p.comp_blocks) {
    atomicOr(status, CKV_DEV_BAD_BLOCK);
    return -1;
  }
  return static_cast<int64_t>(phys) * p.epb + (entry & (p.epb - 1));
}

// Pool row of window token t of request b, or -1 (status bit set) when unmapped.
__device__ __forceinline__ int64_t win_row(const LayerParams& p, int b, int64_t t,
                                           uint32_t* status) {
  const int32_t phys = p.win_table[static_cast<int64_t>(b) * p.table_stride + (t >> 8)];
  if (phys < 0 || phys >= p.win_blocks) {
    atomicOr(status, CKV_DEV_BAD_BLOCK);
    return -1;
  }
  return static_cast<int64_t>(phys) * kBlockTokens + (t & (kBlockTokens - 1));
}

// ------------------------------------------------------------------------------- misc

// Order-preserving map of an fp32 value to uint32 (larger key <=> larger value; -0 < +0).
__device__ __forceinline__ uint32_t f32_order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Programmatic dependent launch: every kernel of the library starts with
//   griddep_wait();      // the previous kernel in the stream has completed, its writes visible
//   griddep_launch();    // the next kernel may be scheduled now (it waits the same way)
// so a launch overlaps the previous kernel's tail while all memory accesses stay ordered.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// hint: bring the 128-byte line holding p into L2 (writes no register, orders nothing)
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace ckv

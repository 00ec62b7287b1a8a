// Device helpers shared by the kernels: error word, number formats, partial
// RoPE.  Format rules (the pages name the formats but not their scaling):
//   KV row   first D-R dims FP8 E4M3 with one fp32 scale s = amax/448 per row
//            (s = 1 for an all-zero row), code = E4M3_rn_satfinite(x / s);
//            last R dims BF16 (round to nearest even).  Page "V4终于终于终于终于
//            是来了", section "HCA——重度压缩注意力": RoPE dims BF16, others FP8.
//   MXFP4    per 32 values one E8M0 scale 2^e, e = floor(log2 amax) - 2
//            clamped to [-127, 127] (e = 0 for an all-zero block), element
//            code = E2M1_rn_satfinite(x * 2^-e).  Podcast summary page,
//            section "2.1 推理与计算效率": FP4 on the indexer path.
//   RoPE     pairs (2i, 2i+1) of the last R dims, angle pos * base^(-2i/R),
//            computed in fp64 so that positions up to 2^20 keep full accuracy.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <atomic>

#include "layout.cuh"

namespace csa {

__device__ __forceinline__ void set_err(const Layout& L, int32_t code, int32_t detail) {
  int32_t* e = L.err();
  if (atomicCAS(e, 0, code) == 0) e[1] = detail;
}

// Tokens visible to query i of a launch (causal visibility).  A decode
// launch (q_per_req == 0): query i is its request's latest token and sees
// the request's whole length.  A chunk of queries (q_per_req = C > 0): the
// queries come in runs of C per request, in position order, for the
// request's C latest tokens, so query i sits at position len - C + i % C and
// sees the tokens up to and including its own.
__device__ __forceinline__ int64_t visible_tokens(int64_t len, int q_per_req, int i) {
  return q_per_req > 0 ? len - q_per_req + (i % q_per_req) + 1 : len;
}

__device__ __forceinline__ uint8_t e4m3_rn(float y) {
  return (uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_val(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}

__device__ __forceinline__ uint16_t bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float bf16_val(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// Two E2M1 codes in one byte: `lo` in bits 0-3, `hi` in bits 4-7.
__device__ __forceinline__ uint8_t e2m1x2_rn(float lo, float hi) {
  return (uint8_t)__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest);
}

// E2M1 value of a 4-bit code, exact.
__device__ __forceinline__ float e2m1_val(uint32_t c) {
  const uint32_t mag = c & 7u;
  // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 as (mag < 2 ? mag*0.5 : (2 + (mag&1)) * 2^((mag>>1) - 2))
  float v = (mag < 2u) ? 0.5f * (float)mag : (float)(2u + (mag & 1u)) * __int_as_float((127 + (int)(mag >> 1) - 2) << 23);
  return (c & 8u) ? -v : v;
}

// Shared exponent of one MX block from its amax (see the rule above).
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int e = ilogbf(amax) - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ float exp2i(int e) {  // 2^e for -126 <= e <= 127, exact
  return __int_as_float((e + 127) << 23);
}

// Multiply by 2^-e exactly (two steps keep every factor a normal fp32).
__device__ __forceinline__ float scale_pow2(float x, int e) {
  const int a = -e / 2, b = -e - a;
  return (x * exp2i(a)) * exp2i(b);
}

// Rotate the pair (x0, x1) by angle pos * theta, in fp64 (positions reach
// 2^20, so an fp32 angle would be off by up to 0.06 rad).  The angle is
// first reduced to [-pi, pi] by subtracting the nearest multiple of 2*pi,
// given as a two-double constant, which keeps sin/cos on their short path.
__device__ __forceinline__ void rope_pair(float& x0, float& x1, double theta, int64_t pos) {
  constexpr double kTwoPiHi = 6.283185307179586;           // 2*pi rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;      // 2*pi - kTwoPiHi
  const double ang = (double)pos * theta;
  const double kq = rint(ang * (1.0 / kTwoPiHi));
  const double r = fma(-kq, kTwoPiHi, ang) - kq * kTwoPiLo;
  double s, c;
  sincos(r, &s, &c);
  const double a = x0, b = x1;
  x0 = (float)(a * c - b * s);
  x1 = (float)(a * s + b * c);
}

// Block-wide max of non-negative values; `red` holds >= 32 floats.
__device__ __forceinline__ float block_max_nonneg(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  v = (l < nw) ? red[l] : 0.f;
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;  // every thread holds the result
}

// Quantise a row held in shared memory (fp32, already rotated) into the KV
// format and store it.  All threads of the block take part.
__device__ __forceinline__ void store_kv_row(const float* row, int D, int R, uint8_t* fp8,
                                             uint16_t* bf16, float* scale, float* red) {
  float amax = 0.f;
  for (int d = threadIdx.x; d < D - R; d += blockDim.x) amax = fmaxf(amax, fabsf(row[d]));
  amax = block_max_nonneg(amax, red);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  for (int d = threadIdx.x; d < D - R; d += blockDim.x) fp8[d] = e4m3_rn(__fdiv_rn(row[d], s));
  for (int d = threadIdx.x; d < R; d += blockDim.x) bf16[d] = bf16_rn(row[D - R + d]);
  if (threadIdx.x == 0) *scale = s;
}

// fp32 storage format: copy a row held in shared memory (already rotated) to
// its stored place as it is.  All threads of the block take part.
__device__ __forceinline__ void store_f32_row(const float* row, int n, float* dst) {
  for (int d = threadIdx.x; d < n; d += blockDim.x) dst[d] = row[d];
}

// Quantise an index key held in shared memory (fp32, d_I values) to MXFP4 and
// store it as key `s` of a page's index tile (code and scale layout in
// layout.cuh).  One warp per 32-value chunk; padding chunks and scales are
// written by the warps that own them.
__device__ __forceinline__ void store_index_key(const Layout& L, const float* key, int s, uint8_t* tile,
                                                uint8_t* sfchunk) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int CH = L.dI / 32;
  for (int c = w; c < 4; c += blockDim.x >> 5) {
    if (c < CH) {
      const float x = key[c * 32 + l];
      float a = fabsf(x);
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      const int e = mx_exponent(a);
      const float y = scale_pow2(x, e);
      const float y_hi = __shfl_down_sync(0xffffffffu, y, 1);
      if ((l & 1) == 0) tile[L.idx_code_off(s, c) + (l >> 1)] = e2m1x2_rn(y, y_hi);
      if (l == 0) sfchunk[Layout::idx_sf_off(s, c)] = (uint8_t)(e + 127);
    } else {
      if (c < L.CHs && l < 16) tile[L.idx_code_off(s, c) + l] = 0;
      if (l == 0) sfchunk[Layout::idx_sf_off(s, c)] = 127;
    }
  }
}

// Host side: whether the kernel set-up marked by `done` (one bit per device)
// still has to run on device `dev`; devices beyond 63 always run it.  Set-up
// calls (function attributes, occupancy queries) are per device, and two
// host threads may both run one (they are idempotent).
inline bool setup_needed(const std::atomic<uint64_t>& done, int dev) {
  return dev < 0 || dev >= 64 || !((done.load(std::memory_order_acquire) >> dev) & 1u);
}
inline void setup_done(std::atomic<uint64_t>& done, int dev) {
  if (dev >= 0 && dev < 64) done.fetch_or(uint64_t(1) << dev, std::memory_order_release);
}

}  // namespace csa

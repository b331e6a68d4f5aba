// Per-token 1x128 FP8 quantisation of activations: x[batch][M][K] (BF16 or
// FP32) -> E4M3 codes q[batch][M][K] and UE8M0 scale words in the packed,
// MN-major layout the GEMMs read ([batch][ceil(K/512)][align4(M)]).
//
// (DeepGEMM pages: the ssnai.com analysis, "库不做预处理": FP8 casting is left
// to the caller, who must produce the scale layout the kernels expect; this
// kernel is that step, fused into one pass.)
//
// For every row and 128-wide K group: amax = max|x|; the scale is the
// smallest power of two s with amax / s <= 448 (s = 1 for an all-zero
// group, clamped to UE8M0's [2^-127, 2^127]); q = E4M3(x / s) rounded to
// nearest even with saturation.  x / s is an exact multiply by a power of two.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace dg {

__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p, int i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_as_float(const float* p, int i) { return p[i]; }

// Loads 16 consecutive elements (32 B of BF16 or 64 B of FP32) as floats.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 w = __ldg(q + h);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * h + 2 * i] = __uint_as_float(u[i] << 16);
      v[8 * h + 2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void load16(const float* p, float (&v)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const float4 w = __ldg(q + h);
    v[4 * h] = w.x;
    v[4 * h + 1] = w.y;
    v[4 * h + 2] = w.z;
    v[4 * h + 3] = w.w;
  }
}

// UE8M0 byte of the smallest power of two s with amax / s <= 448.  With
// amax = m * 2^E (1 <= m < 2): 448 * 2^e >= amax  <=>  1.75 * 2^(e+8) >= m * 2^E,
// so e = E - 8 when m <= 1.75 and E - 7 otherwise.
__device__ __forceinline__ uint32_t ue8m0_scale_byte(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int expf = static_cast<int>((bits >> 23) & 0xFF);
  const uint32_t mant = bits & 0x7FFFFFu;
  if (amax == 0.0f) return 127u;  // all-zero group: scale 1
  if (expf == 0) return 0u;       // subnormal amax: the smallest UE8M0 scale already fits
  int byte = expf - 8 + (mant > 0x600000u ? 1 : 0);
  return static_cast<uint32_t>(byte < 0 ? 0 : byte);
}

// 2^(127 - byte) as a float (the reciprocal of the scale), exact.
__device__ __forceinline__ float inv_scale(uint32_t byte) {
  const int k = 127 - static_cast<int>(byte);  // in [-127, 127]
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// Two floats -> two E4M3 codes (round to nearest even, saturating), lo in bits 0-7.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// One warp per (batch, row, group of four 128-wide K blocks); lane l handles
// elements [16l, 16l+16) of that 512-wide span, so lanes 8j..8j+7 form K block j.
template <typename T>
__global__ void __launch_bounds__(256) quantize_1x128_kernel(const T* __restrict__ x, uint8_t* __restrict__ q,
                                                            uint32_t* __restrict__ sf, int batch, int M, int K,
                                                            int kp, int mn4) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long units = static_cast<long long>(batch) * mn4 * kp;
  const int kb_total = K >> 7;
  for (long long u = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units;
       u += warps) {
    // units run span-fastest along a row, so consecutive warps read and write consecutive bytes
    const int p = static_cast<int>(u % kp);
    const long long rest = u / kp;
    const int m = static_cast<int>(rest % mn4);
    const int b = static_cast<int>(rest / mn4);
    uint32_t word = 0;
    if (m < M) {
      const int j = lane >> 3;               // K block within the span
      const int kblock = 4 * p + j;
      const bool valid = kblock < kb_total;  // K is a multiple of 128: a block is all in or all out
      const size_t row = (static_cast<size_t>(b) * M + m) * static_cast<size_t>(K);
      const size_t off = row + static_cast<size_t>(512) * p + 16 * lane;
      float v[16];
      float amax = 0.0f;
      if (valid) {
        load16(x + off, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const uint32_t byte = valid ? ue8m0_scale_byte(amax) : 0u;
      if (valid) {
        const float inv = inv_scale(byte);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) | (cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
        *reinterpret_cast<uint4*>(q + off) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      // byte of K block j sits in lane 8j: gather the four into one little-endian word
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) word |= __shfl_sync(0xffffffffu, byte, 8 * jj) << (8 * jj);
    }
    if (lane == 0) sf[(static_cast<size_t>(b) * kp + p) * mn4 + m] = word;
  }
}

}  // namespace dg

// Step a1: per-vector e4m3 quantisation of bf16 vectors of 128 elements.
// scale = amax / 448 (1 when amax == 0); code = RNE-saturate(x / scale), all in fp32.
#pragma once
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace dsa {

// One warp per 128-element vector; each lane converts 4 consecutive elements.
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const uint16_t* __restrict__ x, int64_t n_vec,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scale) {
  const int64_t vec = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (vec >= n_vec) return;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + vec * 128 + lane * 4));
  float v[4];
  v[0] = __uint_as_float(raw.x << 16);
  v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  v[2] = __uint_as_float(raw.y << 16);
  v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const __nv_fp8x2_storage_t c01 =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t c23 =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[2], s), __fdiv_rn(v[3], s)), __NV_SATFINITE, __NV_E4M3);
  const uint32_t packed = static_cast<uint32_t>(c01) | (static_cast<uint32_t>(c23) << 16);
  *reinterpret_cast<uint32_t*>(codes + vec * 128 + lane * 4) = packed;
  if (lane == 0) scale[vec] = s;
}

}  // namespace dsa

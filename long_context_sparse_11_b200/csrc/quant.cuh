// Step a1: per-vector e4m3 quantisation of bf16 vectors of 128 elements.
// scale = amax / 448 (1 when amax == 0); code = RNE-saturate(x / scale), all in fp32.
#pragma once
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace dsa {

// One warp per 128-element vector; each lane converts 4 consecutive elements.
__global__ void __launch_bounds__(256) quant_e4m3_kernel(const uint16_t* __restrict__ x, int64_t n_vec,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scale) {
  grid_dependency_sync();
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

namespace dsa {

// Decode-side a1: the new tokens' rows (indexer keys, dim 128, or latent rows, dim 576) are
// quantised per token with the rule above and stored at their slots of a paged e4m3 pool.
// One warp per row; lane l converts the 4-element chunks l, l + 32, ... (dim / 4 chunks).
// Row r belongs to sequence seq[r] (r itself when seq is null) at position pos[r]; its slot is
// page block_table[seq][pos / 64], entry pos % 64.  A row whose sequence, position or page is
// out of range is skipped and flagged in the status word.
constexpr int CACHE_WRITE_MAX_CHUNKS = 5;  // ceil(576 / 4 / 32)

__device__ __forceinline__ void cache_write_row(const uint16_t* __restrict__ x, int64_t r, int lane, int32_t dim,
                                                const int32_t* __restrict__ seq, const int32_t* __restrict__ pos,
                                                const int32_t* __restrict__ block_table, int32_t batch,
                                                int32_t max_pages, int32_t n_pages, uint8_t* __restrict__ pool,
                                                float* __restrict__ pool_scale, int* status) {
  const int32_t b = seq ? seq[r] : static_cast<int32_t>(r);
  const int32_t t = pos[r];
  int32_t page = -1;
  if (b >= 0 && b < batch && t >= 0 && (t >> 6) < max_pages)
    page = block_table[static_cast<int64_t>(b) * max_pages + (t >> 6)];
  if (page < 0 || page >= n_pages) {
    if (lane == 0) atomicOr(status, DEVERR_BOUNDS);
    return;
  }
  const int n_chunks = dim >> 2;
  const uint16_t* src = x + r * dim;
  float v[CACHE_WRITE_MAX_CHUNKS][4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < CACHE_WRITE_MAX_CHUNKS; ++i) {
    const int c = lane + 32 * i;
    if (c < n_chunks) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src + c * 4));
      v[i][0] = __uint_as_float(raw.x << 16);
      v[i][1] = __uint_as_float(raw.x & 0xFFFF0000u);
      v[i][2] = __uint_as_float(raw.y << 16);
      v[i][3] = __uint_as_float(raw.y & 0xFFFF0000u);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i][0]), fabsf(v[i][1])), fmaxf(fabsf(v[i][2]), fabsf(v[i][3]))));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const int64_t slot = static_cast<int64_t>(page) * 64 + (t & 63);
  uint8_t* dst = pool + slot * dim;
#pragma unroll
  for (int i = 0; i < CACHE_WRITE_MAX_CHUNKS; ++i) {
    const int c = lane + 32 * i;
    if (c < n_chunks) {
      const __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(v[i][0], s), __fdiv_rn(v[i][1], s)), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(v[i][2], s), __fdiv_rn(v[i][3], s)), __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<uint32_t*>(dst + c * 4) = static_cast<uint32_t>(c01) | (static_cast<uint32_t>(c23) << 16);
    }
  }
  if (lane == 0) pool_scale[slot] = s;
}

__global__ void __launch_bounds__(256) cache_write_e4m3_kernel(
    const uint16_t* __restrict__ x, int32_t n_rows, int32_t dim, const int32_t* __restrict__ seq,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ block_table, int32_t batch, int32_t max_pages,
    int32_t n_pages, uint8_t* __restrict__ pool, float* __restrict__ pool_scale, int* status) {
  grid_dependency_sync();
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= n_rows) return;
  cache_write_row(x, r, threadIdx.x & 31, dim, seq, pos, block_table, batch, max_pages, n_pages, pool, pool_scale,
                  status);
}

// The same write for up to CACHE_WRITE_MAX_POOLS pools in one launch (every layer's latent pool
// and every Full layer's key pool of a decode step: the same sequences, positions and pages).
// blockIdx.y selects the pool.
constexpr int CACHE_WRITE_MAX_POOLS = 128;
struct CacheWritePools {
  const uint16_t* x[CACHE_WRITE_MAX_POOLS];
  uint8_t* pool[CACHE_WRITE_MAX_POOLS];
  float* scale[CACHE_WRITE_MAX_POOLS];
  int32_t dim[CACHE_WRITE_MAX_POOLS];
};

__global__ void __launch_bounds__(256) cache_write_e4m3_pools_kernel(
    const __grid_constant__ CacheWritePools pools, int32_t n_rows, const int32_t* __restrict__ seq,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ block_table, int32_t batch, int32_t max_pages,
    int32_t n_pages, int* status) {
  grid_dependency_sync();
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= n_rows) return;
  const int i = blockIdx.y;
  cache_write_row(pools.x[i], r, threadIdx.x & 31, pools.dim[i], seq, pos, block_table, batch, max_pages, n_pages,
                  pools.pool[i], pools.scale[i], status);
}

}  // namespace dsa

// Split-N decode: one long sequence whose cache is cut into G contiguous slices, one per GPU.
// Every rank scores and selects its own slice; the ranks then exchange only (score, position)
// candidates and partial attention results (O, LSE), never cache rows.  Three small kernels:
//   split_candidates_kernel  a rank's local Top-k -> (score, global position) pairs, ordered by
//                            position (padding last), so that the concatenation over ranks in rank
//                            order is ordered by global position;
//   split_map_kernel         positions of the merged Top-k in the concatenation -> global
//                            positions, and this rank's local positions (-1 elsewhere);
//   combine_parts_kernel     the ranks' partial attention -> the whole: weights exp(LSE_r - LSE).
// The merge itself is the Top-k kernel over the concatenated candidate scores: equal scores go to
// the lower position, which is the lower global position, as in an unsplit selection.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace dsa {
namespace splitn {

constexpr int SORT_N = 2048;  // largest k

// One CTA of 1024 threads per index row: keys (position << 32 | score bits), padding at the end,
// bitonic sort in shared memory.
__global__ void __launch_bounds__(1024) split_candidates_kernel(const float* __restrict__ scores, int64_t ld,
                                                                const int32_t* __restrict__ idx_local, int32_t k,
                                                                int32_t offset, int32_t n_local,
                                                                float* __restrict__ cand_score,
                                                                int32_t* __restrict__ cand_idx, int* status) {
  __shared__ unsigned long long keys[SORT_N];
  const int64_t row = blockIdx.x;
  int n = 1;
  while (n < k) n <<= 1;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    unsigned long long key = ~0ull;
    if (i < k) {
      const int32_t v = idx_local[row * k + i];
      if (v >= 0 && v < n_local) {
        const float s = scores[row * ld + v];
        key = (static_cast<unsigned long long>(static_cast<uint32_t>(v + offset)) << 32) | __float_as_uint(s);
      } else if (v >= n_local) {
        atomicOr(status, DEVERR_BOUNDS);
      }
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const unsigned long long key = keys[i];
    const bool pad = key == ~0ull;
    cand_idx[row * k + i] = pad ? -1 : static_cast<int32_t>(key >> 32);
    cand_score[row * k + i] = pad ? -INFINITY : __uint_as_float(static_cast<uint32_t>(key & 0xFFFFFFFFull));
  }
}

// pos [rows, k] (positions into the rows' candidate arrays, -1 = none) -> idx_global [rows, k]
// (in place over pos) and idx_local [rows, k] (global - lo inside [lo, hi), else -1).
__global__ void split_map_kernel(const int32_t* __restrict__ cand_idx, int32_t n_cand, int32_t k, int32_t rows,
                                 int32_t* idx_global, int32_t* __restrict__ idx_local, int32_t lo, int32_t hi) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(rows) * k) return;
  const int64_t row = i / k;
  const int32_t p = idx_global[i];
  const int32_t g = (p >= 0 && p < n_cand) ? cand_idx[row * n_cand + p] : -1;
  idx_global[i] = g;
  idx_local[i] = (g >= lo && g < hi) ? g - lo : -1;
}

// Partial results of G ranks over disjoint key sets -> the result over their union:
// lse = log sum_r exp(lse_r), out = sum_r exp(lse_r - lse) out_r.  One CTA of 128 threads per
// (row, head); a part with lse_r = -inf (no keys) has weight 0.
__global__ void __launch_bounds__(128) combine_parts_kernel(const uint16_t* __restrict__ o_parts,
                                                            const float* __restrict__ lse_parts, int32_t n_parts,
                                                            int32_t n_q, uint16_t* __restrict__ out,
                                                            float* __restrict__ lse) {
  const int64_t row = blockIdx.x;
  const int h = blockIdx.y, t = threadIdx.x;
  float m = -INFINITY;
  for (int r = 0; r < n_parts; ++r) m = fmaxf(m, lse_parts[(static_cast<int64_t>(r) * n_q + row) * 64 + h]);
  float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (m > -INFINITY) {
    for (int r = 0; r < n_parts; ++r) {
      const float x = lse_parts[(static_cast<int64_t>(r) * n_q + row) * 64 + h];
      if (!(x > -INFINITY)) continue;
      const float wgt = expf(x - m);
      l += wgt;
      const uint2 v = *reinterpret_cast<const uint2*>(o_parts + ((static_cast<int64_t>(r) * n_q + row) * 64 + h) * 512 +
                                                      4 * t);
      acc[0] = fmaf(wgt, __uint_as_float(v.x << 16), acc[0]);
      acc[1] = fmaf(wgt, __uint_as_float(v.x & 0xFFFF0000u), acc[1]);
      acc[2] = fmaf(wgt, __uint_as_float(v.y << 16), acc[2]);
      acc[3] = fmaf(wgt, __uint_as_float(v.y & 0xFFFF0000u), acc[3]);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&a);
  pk.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(out + (row * 64 + h) * 512 + 4 * t) = pk;
  if (lse && t == 0) lse[row * 64 + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace splitn
}  // namespace dsa

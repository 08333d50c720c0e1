// Dense projections that produce the path's inputs (the indexer's q, k and head weights; the
// latent KV rows): C[M, N] = A[M, K] . B[N, K]^T on the 5th-generation tensor cores, bf16 in,
// fp32 accumulate, then small per-row kernels for the norms and the rotary embedding.
//
// GEMM tile: 128 rows of C (TMEM lanes) x BN columns (TMEM columns, BN = 256), K in blocks of
// 64 (one 128-byte swizzled row per operand row), a STAGES-deep TMA ring.  Warp 0 issues the
// TMA loads, warp 1 owns TMEM and issues the MMAs, warps 2..5 read the accumulator back (warp w:
// rows 32*(w%4) .. +31 of the tile) and store fp32 or bf16, masked to M and N.  Rows or columns
// past the operands are zero-filled by TMA.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace dsa {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * 128;          // 16 KB
constexpr int B_STAGE = BN * 128;          // 32 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_BAR = OFF_B + STAGES * B_STAGE;
constexpr int N_BARS = 2 * STAGES + 1;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int THREADS = 6 * 32;
constexpr uint32_t IDESC = make_idesc(1, 1, 0, 0, BM, BN);

struct Params {
  void* c;          // [M, ldc] fp32 or bf16
  int64_t ldc;      // elements
  int32_t m, n, k;
  int32_t out_bf16; // 1: bf16 output, 0: fp32
  int* status;
  uint64_t wait_ns;
};

__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const uint32_t bar0 = base + OFF_BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t done = bar0 + 8u * (2 * STAGES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int kblocks = (p.k + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(empty(s), ((kb / STAGES) & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
        mbar_arrive_expect_tx(full(s), A_STAGE + B_STAGE);
        tma_load_2d(base + OFF_A + s * A_STAGE, &map_a, full(s), kb * BK, m0);
        tma_load_2d(base + OFF_B + s * B_STAGE, &map_b, full(s), kb * BK, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(full(s), (kb / STAGES) & 1, abort_flag, p.status, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t a = make_sdesc(base + OFF_A + s * A_STAGE + kk * 32, 16, 1024);
          const uint64_t b = make_sdesc(base + OFF_B + s * B_STAGE + kk * 32, 16, 1024);
          mma_f16(tmem, a, b, IDESC, (kb | kk) != 0);
        }
        mma_commit(empty(s));
      }
      if (ok) mma_commit(done);
    }
  } else {
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    const bool got = __all_sync(0xffffffffu, mbar_wait(done, 0, abort_flag, p.status, p.wait_ns));
    tc_fence_after();
    if (got) {
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t x[32];
        DSA_TMEM_LD_X32(taddr + c0, x);
        if (row < p.m && n0 + c0 < p.n) {
          const int ncols = min(32, p.n - (n0 + c0));
          if (p.out_bf16) {
            uint16_t* dst = static_cast<uint16_t*>(p.c) + static_cast<int64_t>(row) * p.ldc + n0 + c0;
            if (ncols == 32) {
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __nv_bfloat162 h =
                      __floats2bfloat162_rn(__uint_as_float(x[j + 2 * e]), __uint_as_float(x[j + 2 * e + 1]));
                  w[e] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
              for (int j = 0; j < ncols; ++j) {
                const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(x[j]));
                dst[j] = *reinterpret_cast<const uint16_t*>(&h);
              }
            }
          } else {
            float* dst = static_cast<float*>(p.c) + static_cast<int64_t>(row) * p.ldc + n0 + c0;
            if (ncols == 32) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(x[j]), __uint_as_float(x[j + 1]),
                                                                  __uint_as_float(x[j + 2]), __uint_as_float(x[j + 3]));
            } else {
              for (int j = 0; j < ncols; ++j) dst[j] = __uint_as_float(x[j]);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, BN);
}

// ---------------------------------------------------------------------------- per-row epilogues

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// Indexer keys and head weights from the fused projection [T, 160] fp32 (128 key dims, then 32
// weights): k = LayerNorm(key dims) * gamma + beta -> bf16 [T,128]; w -> fp32 [T,32].
// One warp per token.
__global__ void __launch_bounds__(256) key_norm_kernel(const float* __restrict__ kw, int32_t n, const float* gamma,
                                                       const float* beta, float eps, uint16_t* __restrict__ k_out,
                                                       float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= n) return;
  const float* r = kw + t * 160;
  const float4 v = *reinterpret_cast<const float4*>(r + 4 * lane);
  const float mean = warp_sum(v.x + v.y + v.z + v.w) * (1.f / 128.f);
  const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
  const float var = warp_sum(d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3) * (1.f / 128.f);
  const float inv = rsqrtf(var + eps);
  const float4 g = *reinterpret_cast<const float4*>(gamma + 4 * lane);
  const float4 b = *reinterpret_cast<const float4*>(beta + 4 * lane);
  const uint32_t lo = static_cast<uint32_t>(bf16_bits(d0 * inv * g.x + b.x)) |
                      (static_cast<uint32_t>(bf16_bits(d1 * inv * g.y + b.y)) << 16);
  const uint32_t hi = static_cast<uint32_t>(bf16_bits(d2 * inv * g.z + b.z)) |
                      (static_cast<uint32_t>(bf16_bits(d3 * inv * g.w + b.w)) << 16);
  *reinterpret_cast<uint2*>(k_out + t * 128 + 4 * lane) = make_uint2(lo, hi);
  w_out[t * 32 + lane] = r[128 + lane];
}

// Angle of RoPE pair i at position pos, reduced to [-pi, pi] in double precision (positions reach
// 2^20 radians and more, beyond what an fp32 angle can hold), then cos / sin.
__device__ __forceinline__ void rope_cos_sin(int32_t pos, int i, double theta, float& c, float& s) {
  const double freq = pow(theta, -2.0 * static_cast<double>(i) / 64.0);
  double a = static_cast<double>(pos) * freq;
  a = remainder(a, 6.283185307179586476925286766559);
  double sd, cd;
  sincos(a, &sd, &cd);
  c = static_cast<float>(cd);
  s = static_cast<float>(sd);
}

// Latent rows from the fused projection [T, 576] fp32: RMSNorm of dims 0..511 times gamma, RoPE
// of dims 512..575 at the token's position -> bf16 [T, 576].  One warp per token.
__global__ void __launch_bounds__(256) latent_norm_rope_kernel(const float* __restrict__ y, int32_t n,
                                                               const float* __restrict__ gamma, const int32_t* pos,
                                                               float eps, double theta, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (t >= n) return;
  const float* r = y + t * 576;
  float v[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 a = *reinterpret_cast<const float4*>(r + 128 * j + 4 * lane);
    v[4 * j] = a.x, v[4 * j + 1] = a.y, v[4 * j + 2] = a.z, v[4 * j + 3] = a.w;
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) ss += v[j] * v[j];
  const float inv = rsqrtf(warp_sum(ss) * (1.f / 512.f) + eps);
  uint16_t* o = out + t * 576;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 g = *reinterpret_cast<const float4*>(gamma + 128 * j + 4 * lane);
    const uint32_t lo = static_cast<uint32_t>(bf16_bits(v[4 * j] * inv * g.x)) |
                        (static_cast<uint32_t>(bf16_bits(v[4 * j + 1] * inv * g.y)) << 16);
    const uint32_t hi = static_cast<uint32_t>(bf16_bits(v[4 * j + 2] * inv * g.z)) |
                        (static_cast<uint32_t>(bf16_bits(v[4 * j + 3] * inv * g.w)) << 16);
    *reinterpret_cast<uint2*>(o + 128 * j + 4 * lane) = make_uint2(lo, hi);
  }
  // lane i turns pair i of the 64 RoPE dims
  float c, s;
  rope_cos_sin(pos[t], lane, theta, c, s);
  const float2 x = *reinterpret_cast<const float2*>(r + 512 + 2 * lane);
  const uint32_t pr = static_cast<uint32_t>(bf16_bits(x.x * c - x.y * s)) |
                      (static_cast<uint32_t>(bf16_bits(x.x * s + x.y * c)) << 16);
  *reinterpret_cast<uint32_t*>(o + 512 + 2 * lane) = pr;
}

// Query RoPE in place: q [T, 64, 576] bf16, dims 512..575 of every head turned to pos[t].  One CTA
// of 8 warps per token (warp w: heads w, w + 8, ...; lane = pair).
__global__ void __launch_bounds__(256) rope_query_kernel(uint16_t* __restrict__ q, int32_t n, const int32_t* pos,
                                                         double theta) {
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x;
  if (t >= n) return;
  float c, s;
  rope_cos_sin(pos[t], lane, theta, c, s);
  for (int h = threadIdx.x >> 5; h < 64; h += 8) {
    uint32_t* pp = reinterpret_cast<uint32_t*>(q + (t * 64 + h) * 576 + 512 + 2 * lane);
    const uint32_t u = *pp;
    const float x0 = __uint_as_float(u << 16), x1 = __uint_as_float(u & 0xFFFF0000u);
    *pp = static_cast<uint32_t>(bf16_bits(x0 * c - x1 * s)) | (static_cast<uint32_t>(bf16_bits(x0 * s + x1 * c)) << 16);
  }
}

}  // namespace gemm
}  // namespace dsa

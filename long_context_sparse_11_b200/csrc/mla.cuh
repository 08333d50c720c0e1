// Step a6 (+ a7 paged address translation / FP8 dequant, a8 MTP rows): sparse MLA
// attention of one query row (64 heads) over its selected latent rows.
//
// Both contractions run "transposed" so that every tcgen05.mma is M = 128 and the
// 64 x 512 fp32 output fits in 256 TMEM columns:
//   S^T[key, head]  = KV[key, 0:576] . Q[head, 0:576]        M = 128 keys,  N = 64 heads
//   O^T[dim, head] += V^T[dim, key]  . P^T[key, head]        M = 128 dims (x4), N = 64 heads
// S^T puts one key on each TMEM lane, so the softmax thread of lane t owns key t: masking,
// per-key FP8 dequant scales and the P^T row are all thread-local; only the per-head max
// and sum cross lanes (shuffle transpose-reduce + 4-warp shared-memory step).  The running
// max is updated lazily (only when a head's max grows by more than 2^8), so O^T is
// rescaled in TMEM rarely.
//
// Shared memory: Q as 9 K-major 64-dim sub-tiles [64 heads x 128 B] (72 KB) and one
// 128-key KV tile as 9 sub-tiles [128 keys x 128 B] (144 KB), all 128-byte swizzled.
// The same KV bytes are the K-major A operand of S^T and the MN-major A operand (V^T) of
// O^T.  Once S^T of a tile has completed, its RoPE sub-tile (dims 512..575) is free and
// receives P^T [128 keys x 64 heads], the MN-major B operand of the second MMA.
//
// Rows are gathered with 16-byte cp.async (bf16 cache) or 16-byte loads + e4m3 -> f16
// conversion (paged FP8 cache; the MMAs then run kind::f16 on f16 operands, exact for
// e4m3 values, and the per-token scale is applied to the logits and folded into P^T).
//
// Warps 0-3: softmax / output; warps 4-7: gather; warp 8: TMEM owner + MMA issuer.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace dsa {
namespace mla {

constexpr int TILE = 128;
constexpr int NSUB = 9;
constexpr int SUB_Q = 64 * 128;    // 8 KB
constexpr int SUB_KV = 128 * 128;  // 16 KB
constexpr int OFF_Q = 0;
constexpr int OFF_KV = NSUB * SUB_Q;
constexpr int OFF_P = OFF_KV + 8 * SUB_KV;  // RoPE sub-tile, reused for P^T
constexpr int OFF_MISC = OFF_KV + NSUB * SUB_KV;
// misc layout (bytes from OFF_MISC)
constexpr int M_BAR = 0;          // 6 mbarriers
constexpr int M_TMEM = 64;
constexpr int M_ABORT = 68;
constexpr int M_FLAG = 72;
constexpr int M_MRUN = 128;       // float[64]
constexpr int M_ALPHA = M_MRUN + 256;
constexpr int M_LTOT = M_ALPHA + 256;
constexpr int M_RED = M_LTOT + 256;  // float[4][64]
constexpr int MISC_BYTES = M_RED + 1024;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
constexpr int THREADS = 288;
constexpr int TMEM_COLS = 512;
constexpr uint32_t TM_S = 256;  // S^T buffers at columns 256, 320

struct Params {
  const uint16_t* q;         // [n_q,64,576] bf16
  const uint8_t* kv;         // dense bf16 [n_tokens,row_stride] or paged e4m3 [n_pages,64,576]
  const float* kv_scale;     // paged: [n_pages*64]
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* idx;        // [n_idx_rows, k]
  uint16_t* out;             // [n_q,64,512] bf16
  float* lse;                // [n_q,64] or null
  float* part_o;             // split partials [n_q*n_split,64,512] fp32
  float* part_ml;            // [n_q*n_split,2,64] (m in log2 units, l)
  int64_t row_stride;        // elements (dense)
  int64_t n_tokens;
  int32_t n_q;
  int32_t rows_per_idx;
  int32_t k;
  int32_t n_split;
  int32_t max_pages;
  int32_t n_pages;
  float scale_log2;          // softmax_scale * log2(e)
  int* status;
  uint64_t wait_ns;
};

// Max (or sum) over the 32 lanes of a warp for 64 per-lane values; lane l ends with the
// results for heads 2l and 2l+1.
template <bool MAX>
__device__ __forceinline__ float2 warp_reduce64(const float (&v)[64], int lane) {
  float a[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[32 + i] : v[i];
    const float give = hi ? v[i] : v[32 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 16);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int w = 32, bit = 8; w >= 4; w >>= 1, bit >>= 1) {
#pragma unroll
    for (int i = 0; i < w / 2; ++i) {
      const bool hi = lane & bit;
      const float keep = hi ? a[w / 2 + i] : a[i];
      const float give = hi ? a[i] : a[w / 2 + i];
      const float o = __shfl_xor_sync(0xffffffffu, give, bit);
      a[i] = MAX ? fmaxf(keep, o) : keep + o;
    }
  }
  return make_float2(a[0], a[1]);
}

// Physical cache row of idx value v of sequence seq, or -1 when v is not a valid token.
template <bool PAGED>
__device__ __forceinline__ int64_t kv_row(const Params& p, int32_t seq, int32_t v, int32_t seq_len) {
  if (v < 0) return -1;
  if (!PAGED) {
    if (v >= p.n_tokens) {
      atomicOr(p.status, DEVERR_BOUNDS);
      return -1;
    }
    return v;
  }
  if (v >= seq_len) {
    atomicOr(p.status, DEVERR_BOUNDS);
    return -1;
  }
  const int32_t lp = v >> 6;
  if (lp >= p.max_pages) return -1;
  const int32_t pg = p.block_table[static_cast<int64_t>(seq) * p.max_pages + lp];
  if (pg < 0 || pg >= p.n_pages) {
    atomicOr(p.status, DEVERR_BOUNDS);
    return -1;
  }
  return static_cast<int64_t>(pg) * 64 + (v & 63);
}

template <bool PAGED>
__global__ void __launch_bounds__(THREADS, 1) sparse_mla_kernel(Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  uint8_t* misc = smem + OFF_MISC;
  const uint32_t bar = base + OFF_MISC + M_BAR;
  const uint32_t q_full = bar, kv_full = bar + 8, s_full = bar + 16, p_full = bar + 24, kv_empty = bar + 32;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + M_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + M_ABORT);
  volatile int* rescale_flag = reinterpret_cast<volatile int*>(misc + M_FLAG);
  float* m_run = reinterpret_cast<float*>(misc + M_MRUN);
  float* alpha = reinterpret_cast<float*>(misc + M_ALPHA);
  float* l_tot = reinterpret_cast<float*>(misc + M_LTOT);
  float* red = reinterpret_cast<float*>(misc + M_RED);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t row = blockIdx.x / p.n_split;
  const int32_t split = blockIdx.x % p.n_split;
  const int32_t irow = row / p.rows_per_idx;  // idx row == sequence in paged mode
  const int32_t* idx_row = p.idx + static_cast<int64_t>(irow) * p.k;
  const int32_t n_tiles_all = (p.k + TILE - 1) / TILE;
  const int32_t tps = (n_tiles_all + p.n_split - 1) / p.n_split;
  const int32_t j0 = split * tps;
  const int32_t j1 = min(j0 + tps, n_tiles_all);
  const int32_t n_tiles = max(j1 - j0, 0);
  const int32_t seq_len = PAGED ? p.seq_lens[irow] : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(kv_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(kv_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 64) m_run[threadIdx.x] = -INFINITY;
  if (warp == 8) tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ gather warps
    const int gt = threadIdx.x - 128;
    const int gw = warp - 4;
    // Q row -> 9 K-major sub-tiles (bf16 copy, or bf16 -> f16 for the FP8 cache path)
    const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + static_cast<int64_t>(row) * 64 * 576);
    for (int c = gt; c < 64 * 72; c += 128) {
      const int h = c / 72, ch = c % 72;
      const uint32_t dst = base + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7);
      if (!PAGED) {
        cp_async16(dst, qsrc + h * 1152 + ch * 16, 16);
      } else {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qsrc + h * 1152 + ch * 16));
        uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint4 o;
        uint32_t* ov = &o.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
          const __half2 hh = __floats2half2_rn(lo, hi);
          ov[i] = *reinterpret_cast<const uint32_t*>(&hh);
        }
        *reinterpret_cast<uint4*>(smem + (dst - base)) = o;
      }
    }
    if (!PAGED) cp_async_wait_all();
    fence_async_smem();
    mbar_arrive(q_full);

    for (int i = 0; i < n_tiles; ++i) {
      const int j = j0 + i;
      if (!mbar_wait(kv_empty, (i & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
      const int key0 = gw * 32;
      const int32_t jj = j * TILE + key0 + lane;
      const int32_t v = jj < p.k ? idx_row[jj] : -1;
      const int64_t prow = kv_row<PAGED>(p, irow, v, seq_len);
      for (int kk = 0; kk < 32; ++kk) {
        const int key = key0 + kk;
        const int64_t r = __shfl_sync(0xffffffffu, prow, kk);
        if (!PAGED) {
          const uint8_t* src = p.kv + (r >= 0 ? r : 0) * p.row_stride * 2;
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            const int ch = lane + 32 * t;
            if (ch < 72) {
              const uint32_t dst = base + OFF_KV + (ch >> 3) * SUB_KV + sw128_off(key, ch & 7);
              cp_async16(dst, src + ch * 16, r >= 0 ? 16 : 0);
            }
          }
        } else {
          const uint8_t* src = p.kv + (r >= 0 ? r : 0) * 576;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int ch = lane + 32 * t;  // 16 e4m3 values = dims [16ch, 16ch+16)
            if (ch < 36) {
              uint4 raw = make_uint4(0, 0, 0, 0);
              if (r >= 0) raw = __ldg(reinterpret_cast<const uint4*>(src + ch * 16));
              uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
              uint4 o0, o1;
              uint32_t* ov0 = &o0.x;
              uint32_t* ov1 = &o1.x;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>(w[q4] & 0xFFFFu), __NV_E4M3);
                const __half2_raw bb = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>(w[q4] >> 16), __NV_E4M3);
                const uint32_t pa = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
                const uint32_t pb = static_cast<uint32_t>(bb.x) | (static_cast<uint32_t>(bb.y) << 16);
                if (q4 < 2) {
                  ov0[2 * q4] = pa;
                  ov0[2 * q4 + 1] = pb;
                } else {
                  ov1[2 * (q4 - 2)] = pa;
                  ov1[2 * (q4 - 2) + 1] = pb;
                }
              }
              const int sub = ch >> 2, c8 = 2 * (ch & 3);
              *reinterpret_cast<uint4*>(smem + OFF_KV + sub * SUB_KV + sw128_off(key, c8)) = o0;
              *reinterpret_cast<uint4*>(smem + OFF_KV + sub * SUB_KV + sw128_off(key, c8 + 1)) = o1;
            }
          }
        }
      }
      if (!PAGED) cp_async_wait_all();
      fence_async_smem();
      mbar_arrive(kv_full);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t FMT = PAGED ? 0u : 1u;  // f16 operands for the FP8 cache, else bf16
      constexpr uint32_t ID_S = make_idesc(FMT, FMT, 0, 0, 128, 64);
      constexpr uint32_t ID_PV = make_idesc(FMT, FMT, 1, 1, 128, 64);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status, p.wait_ns);
      tc_fence_after();
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (!mbar_wait(kv_full, i & 1, abort_flag, p.status, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t ds = tmem + TM_S + 64u * (i & 1);
#pragma unroll 1
        for (int d = 0; d < NSUB; ++d) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = make_sdesc(base + OFF_KV + d * SUB_KV + kk * 32, 16, 1024);
            const uint64_t b = make_sdesc(base + OFF_Q + d * SUB_Q + kk * 32, 16, 1024);
            mma_f16(ds, a, b, ID_S, (d | kk) != 0);
          }
        }
        mma_commit(s_full);
        if (!mbar_wait(p_full, i & 1, abort_flag, p.status, p.wait_ns)) break;
        tc_fence_after();
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = make_sdesc(base + OFF_KV + 2 * mb * SUB_KV + kk * 2048, SUB_KV, 1024);
            const uint64_t b = make_sdesc(base + OFF_P + kk * 2048, SUB_KV, 1024);
            mma_f16(tmem + 64u * mb, a, b, ID_PV, (i > 0 || kk > 0));
          }
        }
        mma_commit(kv_empty);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int t = threadIdx.x;  // TMEM lane = key within tile (S^T) = dim within block (O^T)
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float lsum[64];
#pragma unroll
    for (int h = 0; h < 64; ++h) lsum[h] = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int j = j0 + i;
      const int32_t jj = j * TILE + t;
      const int32_t v = jj < p.k ? idx_row[jj] : -1;
      const int64_t prow = kv_row<PAGED>(p, irow, v, seq_len);
      const bool valid = prow >= 0;
      const float kscale = PAGED ? (valid ? p.kv_scale[prow] : 0.f) : 1.f;
      if (!mbar_wait(s_full, i & 1, abort_flag, p.status, p.wait_ns)) break;
      tc_fence_after();
      float z[64];
      {
        uint32_t x[32];
        const uint32_t ta = tmem + TM_S + 64u * (i & 1) + lane_off;
        DSA_TMEM_LD_X32(ta, x);
#pragma unroll
        for (int h = 0; h < 32; ++h) z[h] = __uint_as_float(x[h]);
        DSA_TMEM_LD_X32(ta + 32, x);
#pragma unroll
        for (int h = 0; h < 32; ++h) z[32 + h] = __uint_as_float(x[h]);
      }
      const float zs = p.scale_log2 * kscale;
#pragma unroll
      for (int h = 0; h < 64; ++h) z[h] = valid ? z[h] * zs : -INFINITY;
      const float2 wm = warp_reduce64<true>(z, lane);
      red[warp * 64 + 2 * lane] = wm.x;
      red[warp * 64 + 2 * lane + 1] = wm.y;
      if (t == 0) *rescale_flag = 0;
      named_bar(1, 128);
      if (t < 64) {
        const float tmax = fmaxf(fmaxf(red[t], red[64 + t]), fmaxf(red[128 + t], red[192 + t]));
        const float mo = m_run[t];
        float a = 1.f;
        if (tmax > -INFINITY && (mo == -INFINITY || tmax > mo + 8.f)) {
          a = (mo == -INFINITY) ? 0.f : exp2f(mo - tmax);
          m_run[t] = tmax;
          *rescale_flag = 1;
        }
        alpha[t] = a;
      }
      named_bar(1, 128);
      const bool resc = *rescale_flag != 0;
      // probabilities, partial row sums, P^T row
      uint32_t pk[32];
#pragma unroll
      for (int h2 = 0; h2 < 32; ++h2) {
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * h2 + e;
          const float m = m_run[h];
          const float pr = valid ? exp2f(z[h] - (m == -INFINITY ? 0.f : m)) : 0.f;
          lsum[h] = resc ? fmaf(lsum[h], alpha[h], pr) : lsum[h] + pr;
          pv[e] = pr * kscale;
        }
        if (PAGED) {
          const __half2 hh = __floats2half2_rn(pv[0], pv[1]);
          pk[h2] = *reinterpret_cast<const uint32_t*>(&hh);
        } else {
          const __nv_bfloat162 bb = __floats2bfloat162_rn(pv[0], pv[1]);
          pk[h2] = *reinterpret_cast<const uint32_t*>(&bb);
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(smem + OFF_P + sw128_off(t, c)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      if (resc && i > 0) {
        // O^T (dims on lanes, heads on columns) *= alpha[head]; PV of the previous tile is done
        if (!mbar_wait(kv_empty, (i - 1) & 1, abort_flag, p.status, p.wait_ns)) break;
        tc_fence_after();
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t x[32];
            const uint32_t ta = tmem + 64u * mb + 32u * hh + lane_off;
            DSA_TMEM_LD_X32(ta, x);
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = __float_as_uint(__uint_as_float(x[c]) * alpha[32 * hh + c]);
            DSA_TMEM_ST_X32(ta, x);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ---- final: wait for the last PV, reduce row sums, write the output
    if (n_tiles > 0) ok = mbar_wait(kv_empty, (n_tiles - 1) & 1, abort_flag, p.status, p.wait_ns);
    tc_fence_after();
    const float2 ws = warp_reduce64<false>(lsum, lane);
    named_bar(1, 128);
    red[warp * 64 + 2 * lane] = ws.x;
    red[warp * 64 + 2 * lane + 1] = ws.y;
    named_bar(1, 128);
    if (t < 64) l_tot[t] = red[t] + red[64 + t] + red[128 + t] + red[192 + t];
    named_bar(1, 128);
    if (ok && !*abort_flag) {
      if (p.n_split == 1) {
        uint16_t* orow = p.out + static_cast<int64_t>(row) * 64 * 512;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t x[32];
            if (n_tiles > 0) {
              DSA_TMEM_LD_X32(tmem + 64u * mb + 32u * hh + lane_off, x);
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) x[c] = 0u;
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int h = 32 * hh + c;
              const float l = l_tot[h];
              const float o = l > 0.f ? __uint_as_float(x[c]) / l : 0.f;
              const __nv_bfloat16 ob = __float2bfloat16_rn(o);
              orow[h * 512 + mb * 128 + t] = *reinterpret_cast<const uint16_t*>(&ob);
            }
          }
        }
        if (p.lse && t < 64) {
          const float l = l_tot[t];
          p.lse[static_cast<int64_t>(row) * 64 + t] =
              l > 0.f ? (m_run[t] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      } else {
        const int64_t pr = static_cast<int64_t>(row) * p.n_split + split;
        float* po = p.part_o + pr * 64 * 512;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t x[32];
            if (n_tiles > 0) {
              DSA_TMEM_LD_X32(tmem + 64u * mb + 32u * hh + lane_off, x);
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) x[c] = 0u;
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) po[(32 * hh + c) * 512 + mb * 128 + t] = __uint_as_float(x[c]);
          }
        }
        if (t < 64) {
          p.part_ml[pr * 128 + t] = m_run[t];
          p.part_ml[pr * 128 + 64 + t] = l_tot[t];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, TMEM_COLS);
}

// Combine split-KV partials: one CTA of 128 threads per (row, head), 4 dims per thread.
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int32_t n_split,
                                                      uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int32_t row = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) {
    const int64_t pr = static_cast<int64_t>(row) * n_split + s;
    if (part_ml[pr * 128 + 64 + h] > 0.f) M = fmaxf(M, part_ml[pr * 128 + h]);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n_split; ++s) {
    const int64_t pr = static_cast<int64_t>(row) * n_split + s;
    const float l = part_ml[pr * 128 + 64 + h];
    if (!(l > 0.f)) continue;
    const float wgt = exp2f(part_ml[pr * 128 + h] - M);
    L = fmaf(wgt, l, L);
    const float4 o = *reinterpret_cast<const float4*>(part_o + (pr * 64 + h) * 512 + 4 * t);
    acc.x = fmaf(wgt, o.x, acc.x);
    acc.y = fmaf(wgt, o.y, acc.y);
    acc.z = fmaf(wgt, o.z, acc.z);
    acc.w = fmaf(wgt, o.w, acc.w);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 b = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&a);
  pk.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(row) * 64 + h) * 512 + 4 * t) = pk;
  if (lse && t == 0)
    lse[static_cast<int64_t>(row) * 64 + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace mla
}  // namespace dsa

// Step a6 for the bf16 latent table (prefill and dense rows): sparse MLA with the KV tile
// double-buffered in 64-key halves.
//
// The single-tile kernel (mla.cuh) holds one 128-key tile next to the query row, which fills
// shared memory: the gather of tile j+1 can start only once PV(j) has released the tile, so
// every tile pays gather + S^T + softmax + PV + one L2 latency in sequence.  Here the same
// 144 KB hold two 64-key half tiles.  While the softmax and PV of half h run on one buffer,
// the rows of half h+1 land in the other and S^T(h+1) runs on the tensor core; the chain of a
// buffer (gather, S^T, softmax, PV) is then shared by two halves in flight.
//
//   S^T[key, head]  = KV[key, 0:576] . Q[head, 0:576]      M = 64 keys,  N = 64 heads
//   O^T[dim, head] += V^T[dim, key]  . P^T[key, head]      M = 128 dims (x4), N = 64 heads, K = 64
//
// S^T is an M = 64 product (the tensor core takes as long as for M = 128, so S^T costs twice
// its flops; PV is unchanged): its accumulator rows sit on lanes 0-15 of each 32-lane quadrant
// (key r on lane 32 (r / 16) + r % 16), and each softmax warp reads its 16 keys for 8 heads in
// each half-warp (the 16x32bx2 TMEM load), so all 32 lanes work.
//
// The MMA issuer follows two cursors: S^T of the next half, sub-tile by sub-tile as its rows
// land, and PV of the oldest half whose probabilities are ready, whichever can go; a half's
// S^T is never issued before PV of the half two back (its accumulator and buffer are reused).
//
// Shared memory: Q as 9 K-major 64-dim sub-tiles [64 heads x 128 B] (72 KB); two buffers of
// 9 sub-tiles [64 keys x 128 B] (2 x 72 KB); P^T of a half replaces its RoPE sub-tile once its
// S^T has completed.  Barriers per buffer: a "full" barrier per sub-tile, an "empty" barrier per
// 128-dim block of V (committed when the PV MMAs of that block complete) and one for the whole
// PV (it releases the RoPE sub-tile that held P^T).
#pragma once
#include "mla.cuh"

namespace dsa {
namespace mla {
namespace db {

constexpr int HALF = 64;
constexpr int SUB_H = HALF * 128;  // 8 KB: 64 keys x 64 dims bf16
constexpr int OFF_Q = 0;
constexpr int OFF_KV = NSUB * SUB_Q;                      // 72 KB
constexpr int BUF_BYTES = NSUB * SUB_H;                   // 72 KB per half buffer
constexpr int OFF_MISC = OFF_KV + 2 * BUF_BYTES;          // 216 KB
constexpr int N_BARS = 34;
constexpr int M_TMEM = N_BARS * 8;
constexpr int M_ABORT = M_TMEM + 4;
constexpr int M_NEED = M_TMEM + 8;  // int[2]
constexpr int M_MRUN = 512;         // float[64], log2 units
constexpr int M_ALPHA = M_MRUN + 256;
constexpr int M_LTOT = M_ALPHA + 256;
constexpr int M_RED = M_LTOT + 256;  // float[4 quadrants][64 heads]
constexpr int MISC_BYTES = M_RED + 1024;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(M_NEED + 8 <= M_MRUN, "misc layout");
static_assert(HPW == 16, "the half-warp softmax takes 16 heads per warp (8 per half-warp)");

// barriers
constexpr int B_QFULL = 0, B_QEMPTY = 1;
__host__ __device__ constexpr int b_sfull(int s) { return 2 + s; }
__host__ __device__ constexpr int b_pfull(int b) { return 4 + b; }
__host__ __device__ constexpr int b_pvdone(int b) { return 6 + b; }
__host__ __device__ constexpr int b_full(int b, int d) { return 8 + b * NSUB + d; }
__host__ __device__ constexpr int b_empty(int b, int mb) { return 8 + 2 * NSUB + b * 4 + mb; }
static_assert(b_empty(1, 3) + 1 == N_BARS, "barrier count");

constexpr int GA_CH = HALF * 8;                          // 16-byte chunks per sub-tile of a half
constexpr int MAXC_H = (GA_CH + GA_THREADS - 1) / GA_THREADS;

// Halves of an item: its 128-key tiles, cut at the row's last valid entry.
__device__ __forceinline__ int32_t n_halves(const Params& p, const Item& it) {
  int64_t lim = p.k;
  if (p.valid0 >= 0) lim = min(static_cast<int64_t>(p.k), max(p.valid0 + it.irow, static_cast<int64_t>(0)));
  const int64_t lo = static_cast<int64_t>(it.j0) * TILE;
  const int64_t hi = min(static_cast<int64_t>(it.j0 + it.n_tiles) * TILE, lim);
  return hi > lo ? static_cast<int32_t>((hi - lo + HALF - 1) / HALF) : 0;
}

// Max (or sum) of 8 values over the 16 lanes of each half-warp; lanes 2i and 2i+1 of a half
// end with the result for value index i.
template <bool MAX>
__device__ __forceinline__ float half_reduce8(const float (&v)[8], int lane) {
  float a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    const float keep = hi ? v[4 + i] : v[i];
    const float give = hi ? v[i] : v[4 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 8);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
  float b[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    const float keep = hi ? a[2 + i] : a[i];
    const float give = hi ? a[i] : a[2 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 4);
    b[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
  const bool hi = lane & 2;
  const float keep = hi ? b[1] : b[0];
  const float give = hi ? b[0] : b[1];
  float c = __shfl_xor_sync(0xffffffffu, give, 2);
  c = MAX ? fmaxf(keep, c) : keep + c;
  const float o = __shfl_xor_sync(0xffffffffu, c, 1);
  return MAX ? fmaxf(c, o) : c + o;
}

__global__ void __launch_bounds__(THREADS, 1) sparse_mla_db_kernel(Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  uint8_t* misc = smem + OFF_MISC;
  const uint32_t bar0 = base + OFF_MISC;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + M_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + M_ABORT);
  volatile int* need_flags = reinterpret_cast<volatile int*>(misc + M_NEED);
  float* m_run = reinterpret_cast<float*>(misc + M_MRUN);
  float* alpha = reinterpret_cast<float*>(misc + M_ALPHA);
  float* l_tot = reinterpret_cast<float*>(misc + M_LTOT);
  float* red = reinterpret_cast<float*>(misc + M_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto kv_addr = [&](int b, int d) { return base + OFF_KV + static_cast<uint32_t>(b * BUF_BYTES + d * SUB_H); };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), GA_THREADS);
    mbar_init(bar(B_QEMPTY), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(b_sfull(b)), 1);
      mbar_init(bar(b_pfull(b)), SM_THREADS);
      mbar_init(bar(b_pvdone(b)), 1);
      for (int d = 0; d < NSUB; ++d) mbar_init(bar(b_full(b, d)), GA_THREADS);
      for (int mb = 0; mb < 4; ++mb) mbar_init(bar(b_empty(b, mb)), 1);
    }
    *abort_flag = 0;
    need_flags[0] = 0;
    need_flags[1] = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= SM_WARPS && warp < MMA_WARP) {
    // ================================================================= gather warps
    const int gq = threadIdx.x - SM_THREADS;
    uint32_t gh = 0;  // global half counter (buffer gh & 1, use gh >> 1)
    bool ok = true;
    WorkIter wk = work_begin<false>(p);
    Item it;
    for (int32_t it_n = 0; ok && work_next<false>(p, wk, it); ++it_n) {
      if (!mbar_wait(bar(B_QEMPTY), (it_n & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + static_cast<int64_t>(it.row) * 64 * 576);
      constexpr int QCH = 64 * 72;
      for (int c = gq; c < QCH; c += GA_THREADS) {
        const int h = c / 72, ch = c % 72;
        cp_async16(base + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7), qsrc + h * 1152 + ch * 16, 16);
      }
      cp_async_arrive_noinc(bar(B_QFULL));
      const int32_t nh = n_halves(p, it);
      const int32_t* idx_row = p.idx + static_cast<int64_t>(it.irow) * p.k;
      const int32_t key0 = it.j0 * TILE;
      for (int32_t hh = 0; hh < nh && ok; ++hh, ++gh) {
        const int b = gh & 1;
        const uint32_t par = ((gh >> 1) & 1) ^ 1;
        const uint8_t* src[MAXC_H];
        uint32_t dst[MAXC_H], nb[MAXC_H];
#pragma unroll
        for (int i = 0; i < MAXC_H; ++i) {
          const int c = gq + i * GA_THREADS;
          int64_t r = -1;
          if (c < GA_CH) {
            const int32_t jj = key0 + hh * HALF + (c >> 3);
            const int32_t v = jj < p.k ? idx_row[jj] : -1;
            r = kv_row<false>(p, it.irow, v, 0);
          }
          src[i] = p.kv + (r >= 0 ? r : 0) * p.row_stride * 2 + (c & 7) * 16;
          dst[i] = c < GA_CH ? sw128_off(c >> 3, c & 7) : 0xFFFFFFFFu;
          nb[i] = r >= 0 ? 16u : 0u;
        }
        for (int d = 0; d < NSUB; ++d) {
          if ((d & 1) == 0 &&
              !mbar_wait(bar(d < 8 ? b_empty(b, d / 2) : b_pvdone(b)), par, abort_flag, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int i = 0; i < MAXC_H; ++i)
            if (dst[i] != 0xFFFFFFFFu) cp_async16(kv_addr(b, d) + dst[i], src[i] + d * 128, nb[i]);
          cp_async_arrive_noinc(bar(b_full(b, d)));
        }
      }
    }
  } else if (warp == MMA_WARP) {
    // ================================================================= MMA issuer (two cursors)
    if (lane == 0) {
      constexpr uint32_t ID_S = make_idesc(1, 1, 0, 0, 64, 64);
      constexpr uint32_t ID_PV = make_idesc(1, 1, 1, 1, 128, 64);
      // S^T cursor
      WorkIter ws = work_begin<false>(p);
      Item is;
      bool s_have = false, s_end = false, s_q = false;
      int32_t s_nh = 0, s_hh = 0, s_item = -1;
      int s_d = 0;
      uint32_t s_g = 0;
      // PV cursor
      WorkIter wv = work_begin<false>(p);
      Item iv;
      bool v_have = false, v_end = false;
      int32_t v_nh = 0, v_hh = 0;
      uint32_t v_g = 0;
      uint64_t t_idle = 0;
      bool idle = false;
      while (true) {
        if (*abort_flag) break;
        bool prog = false;
        if (!s_have && !s_end) {
          if (work_next<false>(p, ws, is)) {
            s_have = true;
            s_q = false;
            s_nh = n_halves(p, is);
            s_hh = 0;
            ++s_item;
          } else {
            s_end = true;
          }
        }
        if (s_have && !s_q && mbar_test_wait(bar(B_QFULL), s_item & 1)) {
          fence_async_smem();
          tc_fence_after();
          s_q = true;
          prog = true;
          if (s_nh == 0) {
            mma_commit(bar(B_QEMPTY));
            s_have = false;
          }
        }
        if (s_have && s_q && s_g <= v_g + 1) {
          const int b = s_g & 1;
          const uint32_t par = (s_g >> 1) & 1;
          const uint32_t ds = tmem + TM_S + 64u * b;
          while (s_d < NSUB && mbar_test_wait(bar(b_full(b, s_d)), par)) {
            fence_async_smem();
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t a = make_sdesc(kv_addr(b, s_d) + kk * 32, 16, 1024);
              const uint64_t bq = make_sdesc(base + OFF_Q + s_d * SUB_Q + kk * 32, 16, 1024);
              mma_f16(ds, a, bq, ID_S, (s_d | kk) != 0);
            }
            ++s_d;
            prog = true;
          }
          if (s_d == NSUB) {
            mma_commit(bar(b_sfull(b)));
            if (++s_hh == s_nh) {
              mma_commit(bar(B_QEMPTY));
              s_have = false;
            }
            s_d = 0;
            ++s_g;
          }
        }
        while (!v_have && !v_end) {
          if (work_next<false>(p, wv, iv)) {
            v_nh = n_halves(p, iv);
            v_hh = 0;
            v_have = v_nh > 0;
          } else {
            v_end = true;
          }
        }
        if (v_have && v_g < s_g) {
          const int b = v_g & 1;
          if (mbar_test_wait(bar(b_pfull(b)), (v_g >> 1) & 1)) {
            tc_fence_after();
#pragma unroll 1
            for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = make_sdesc(kv_addr(b, 2 * mb) + kk * 2048, SUB_H, 1024);
                const uint64_t bp = make_sdesc(kv_addr(b, 8) + kk * 2048, SUB_H, 1024);
                mma_f16(tmem + 64u * mb, a, bp, ID_PV, (v_hh > 0 || kk > 0));
              }
              mma_commit(bar(b_empty(b, mb)));
            }
            mma_commit(bar(b_pvdone(b)));
            ++v_g;
            if (++v_hh == v_nh) v_have = false;
            prog = true;
          }
        }
        if (s_end && !s_have && v_end && !v_have) break;
        if (prog) {
          idle = false;
          continue;
        }
        __nanosleep(20);  // leave the issue slots of this sub-partition to the softmax warps
        if (!idle) {
          idle = true;
          t_idle = globaltimer_ns();
        } else if (globaltimer_ns() - t_idle > p.wait_ns) {
          *abort_flag = 1;
          atomicOr(p.status, DEVERR_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ================================================================= softmax / output warps
    const int quad = warp & 3, hh4 = warp >> 2;
    const int side = lane >> 4;                              // half-warp: heads +0..7 or +8..15
    const int kq = quad * 16 + (lane & 15);                  // key of the half (S^T row)
    const int key_o = quad * 32 + lane;                      // O^T lane: dim of a block
    const int st = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t hcol = static_cast<uint32_t>(HPW) * hh4;  // the warp's 16 heads
    const uint32_t h8 = hcol + 8u * side;                    // this thread's 8 heads
    const bool head_lane = lane < HPW;
    uint32_t gh = 0;
    bool ok = true;
    WorkIter wk = work_begin<false>(p);
    Item it;
    while (ok && work_next<false>(p, wk, it)) {
      const int32_t* idx_row = p.idx + static_cast<int64_t>(it.irow) * p.k;
      const int32_t nh = n_halves(p, it);
      const int32_t key0 = it.j0 * TILE;
      if (quad == 0 && head_lane) m_run[hcol + lane] = -INFINITY;
      named_bar(1, SM_THREADS);
      bool fail = false;
      float lsum[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) lsum[h] = 0.f;
      for (int32_t hh = 0; hh < nh; ++hh, ++gh) {
        const int b = gh & 1;
        const uint32_t par = (gh >> 1) & 1;
        const int32_t jj = key0 + hh * HALF + kq;
        const int32_t v = jj < p.k ? idx_row[jj] : -1;
        const bool valid = kv_row<false>(p, it.irow, v, 0) >= 0;
        {
          const bool got = mbar_wait(bar(b_sfull(b)), par, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
        }
        tc_fence_after();
        float z[8];
        if (!fail) {
          uint32_t x[8];
          DSA_TMEM_LD_16X2_X8(tmem + TM_S + 64u * b + hcol + lane_off, x);
#pragma unroll
          for (int h = 0; h < 8; ++h) z[h] = valid ? __uint_as_float(x[h]) * p.scale_log2 : -INFINITY;
        } else {
#pragma unroll
          for (int h = 0; h < 8; ++h) z[h] = -INFINITY;
        }
        volatile int* need = need_flags + (gh & 1);
        bool exceed = false;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_run + h8 + 4 * c);
          exceed |= (z[4 * c] > m4.x + 8.f) | (z[4 * c + 1] > m4.y + 8.f) | (z[4 * c + 2] > m4.z + 8.f) |
                    (z[4 * c + 3] > m4.w + 8.f);
        }
        if (__any_sync(0xffffffffu, exceed) && lane == 0) *need = 1;
        if (named_bar_or(1, SM_THREADS, fail)) {
          ok = false;
          break;
        }
        if (st == 0) need_flags[(gh + 1) & 1] = 0;
        const bool resc = *need != 0;
        if (resc) {
          const float wmax = half_reduce8<true>(z, lane);
          if ((lane & 1) == 0) red[quad * 64 + h8 + ((lane & 15) >> 1)] = wmax;
          named_bar(1, SM_THREADS);
          if (quad == 0 && head_lane) {
            const int h = hcol + lane;
            const float tmax = fmaxf(fmaxf(red[h], red[64 + h]), fmaxf(red[128 + h], red[192 + h]));
            const float mo = m_run[h];
            float a = 1.f;
            if (tmax > -INFINITY && (mo == -INFINITY || tmax > mo + 8.f)) {
              a = (mo == -INFINITY) ? 0.f : ex2_approx(mo - tmax);
              m_run[h] = tmax;
            }
            alpha[h] = a;
          }
          named_bar(1, SM_THREADS);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const float4 a4 = *reinterpret_cast<const float4*>(alpha + h8 + 4 * c);
            lsum[4 * c] *= a4.x;
            lsum[4 * c + 1] *= a4.y;
            lsum[4 * c + 2] *= a4.z;
            lsum[4 * c + 3] *= a4.w;
          }
        }
        {
          const float4 ma = *reinterpret_cast<const float4*>(m_run + h8);
          const float4 mb4 = *reinterpret_cast<const float4*>(m_run + h8 + 4);
          const float m8[8] = {ma.x, ma.y, ma.z, ma.w, mb4.x, mb4.y, mb4.z, mb4.w};
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_approx(z[2 * e] - (m8[2 * e] == -INFINITY ? 0.f : m8[2 * e]));
            const float p1 = ex2_approx(z[2 * e + 1] - (m8[2 * e + 1] == -INFINITY ? 0.f : m8[2 * e + 1]));
            lsum[2 * e] += p0;
            lsum[2 * e + 1] += p1;
            pk[e] = pack_pair(p0, p1, false);
          }
          *reinterpret_cast<uint4*>(smem + OFF_KV + b * BUF_BYTES + 8 * SUB_H + sw128_off(kq, h8 >> 3)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (resc && hh > 0) {
          // O^T *= alpha once PV of the previous half (the other buffer) is done
          const uint32_t pg = gh - 1;
          const bool got = mbar_wait(bar(b_pvdone(pg & 1)), (pg >> 1) & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
          tc_fence_after();
#pragma unroll 1
          for (int mb = 0; mb < 4 && !fail; ++mb) {
            uint32_t x[HPW];
            const uint32_t ta = tmem + 64u * mb + hcol + lane_off;
            tmem_ld_heads<HPW>(ta, x);
#pragma unroll
            for (int c = 0; c < HPW; ++c) x[c] = __float_as_uint(__uint_as_float(x[c]) * alpha[hcol + c]);
            tmem_st_heads<HPW>(ta, x);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(b_pfull(b)));
      }
      if (!ok) break;
      // ---- end of item: wait for the last PV, reduce row sums, write the output
      if (nh > 0) {
        const uint32_t pg = gh - 1;
        const bool got = mbar_wait(bar(b_pvdone(pg & 1)), (pg >> 1) & 1, abort_flag, p.status, p.wait_ns);
        fail = __any_sync(0xffffffffu, fail || !got);
        tc_fence_after();
      }
      {
        const float wsum = half_reduce8<false>(lsum, lane);
        if ((lane & 1) == 0) red[quad * 64 + h8 + ((lane & 15) >> 1)] = wsum;
      }
      if (named_bar_or(1, SM_THREADS, fail)) break;
      if (quad == 0 && head_lane) {
        const int h = hcol + lane;
        l_tot[h] = red[h] + red[64 + h] + red[128 + h] + red[192 + h];
      }
      named_bar(1, SM_THREADS);
      if (it.direct) {
        uint16_t* orow = p.out + static_cast<int64_t>(it.row) * 64 * 512;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t x[HPW];
          if (nh > 0) {
            tmem_ld_heads<HPW>(tmem + 64u * mb + hcol + lane_off, x);
          } else {
#pragma unroll
            for (int c = 0; c < HPW; ++c) x[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < HPW; ++c) {
            const int h = hcol + c;
            const float l = l_tot[h];
            const float o = l > 0.f ? __uint_as_float(x[c]) / l : 0.f;
            const __nv_bfloat16 ob = __float2bfloat16_rn(o);
            orow[h * 512 + mb * 128 + key_o] = *reinterpret_cast<const uint16_t*>(&ob);
          }
        }
        if (p.lse && quad == 0 && head_lane) {
          const int h = hcol + lane;
          const float l = l_tot[h];
          p.lse[static_cast<int64_t>(it.row) * 64 + h] =
              l > 0.f ? (m_run[h] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      } else {
        const int64_t pr = static_cast<int64_t>(it.row) * p.n_split + it.split;
        float* po = p.part_o + pr * 64 * 512;
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t x[HPW];
          if (nh > 0) {
            tmem_ld_heads<HPW>(tmem + 64u * mb + hcol + lane_off, x);
          } else {
#pragma unroll
            for (int c = 0; c < HPW; ++c) x[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < HPW; ++c) po[(hcol + c) * 512 + mb * 128 + key_o] = __uint_as_float(x[c]);
        }
        if (quad == 0 && head_lane) {
          const int h = hcol + lane;
          p.part_ml[pr * 128 + h] = m_run[h];
          p.part_ml[pr * 128 + 64 + h] = l_tot[h];
        }
      }
      tc_fence_before();
      named_bar(1, SM_THREADS);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace db
}  // namespace mla
}  // namespace dsa

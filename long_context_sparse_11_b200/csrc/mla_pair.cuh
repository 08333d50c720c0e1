// Step a6 for many query rows over a dense bf16 latent cache (causal prefill): sparse MLA run by
// a pair of CTAs (a thread-block cluster of 2) that splits every selected latent row by its dims.
//
// Why a pair.  With 64 heads a 128-key tile of full 576-dim rows takes 144 KB of shared memory
// next to the 72 KB query row, so one CTA holds a single tile and the gather of tile j+1 cannot
// start before tile j has gone through S, softmax and PV.  Split by dims over two CTAs, each CTA
// holds 288 dims of a key (256 value dims + 32 RoPE dims: 576 B) and of the query row, so a tile
// is 72 KB and two tiles fit: the gather of tile j+1 runs under the math of tile j.
//
// CTA c of the pair holds value dims [256c, 256c+256) and RoPE dims [512+32c, 512+32c+32).
//   S^T partial:  S_c[key, head] = KV[key, dims_c] . Q[head, dims_c]      (M=128 keys, N=64, K=288)
//   The full logits are S = S_0 + S_1.  CTA c owns heads [32c, 32c+32): it sends the peer the
//   partials of the peer's heads and receives the partials of its own (16 KB each way per tile,
//   through distributed shared memory), runs the online softmax of its own heads, and writes
//   their P^T columns into both CTAs' P^T tile.
//   O^T_c[dim, head] += V^T[dims_c, key] . P^T[key, head]                (M=128 dims x 2, N=64)
//   Each CTA thus accumulates its own 256 output dims of all 64 heads; a head's running-max
//   rescale factor travels with its P^T columns, and its final row sum at the end of the row.
//
// Shared memory per CTA: Q (4 swizzled 64-dim sub-tiles + one 32-dim no-swizzle sub-tile, 36 KB),
// two KV tiles (72 KB each, same layout over 128 keys), P^T (128 keys x 64 heads, 16 KB), the
// received partial logits (128 keys x 32 heads fp32, 16 KB), barriers and per-head state.
//
// Warps: SM_WARPS softmax / output warps (warp w: TMEM lane quadrant w%4, HPW own heads from
// HPW*(w/4) of the CTA's 32), then 7 gather warps (query row and KV tiles by cp.async), then the
// TMEM owner + MMA issuer.
//
// Every wait is bounded (mbar_wait); the softmax warps agree on a failure at
// their per-tile barrier (named_bar_or) and leave together.  Both CTAs meet at a cluster barrier
// before either exits, so no CTA writes into the shared memory of one that has gone.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace dsa {
namespace mlap {

constexpr int TILE = 128;
constexpr int NSUB = 4;                      // swizzled 64-dim value sub-tiles per CTA
constexpr int SUB_KV = 128 * 128;            // 16 KB
constexpr int ROPE_KV = 128 * 64;            // 8 KB: 32 RoPE dims x 128 keys, no swizzle
constexpr int TILE_BYTES = NSUB * SUB_KV + ROPE_KV;  // 72 KB
constexpr int SUB_Q = 64 * 128;              // 8 KB
constexpr int ROPE_Q = 64 * 64;              // 4 KB
constexpr int Q_BYTES = NSUB * SUB_Q + ROPE_Q;       // 36 KB
constexpr int P_BYTES = 128 * 128;           // P^T [128 keys][64 heads] bf16, swizzled
constexpr int RECV_BYTES = 128 * 128;        // [128 keys][32 heads] fp32 partial logits
constexpr int PRECV_BYTES = 128 * 64 + 32 * 4 + 4;   // the peer's P^T columns, rescale factors, flag

constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + Q_BYTES;
constexpr int OFF_P = OFF_KV + 2 * TILE_BYTES;
constexpr int OFF_RECV = OFF_P + P_BYTES;
constexpr int OFF_MISC = OFF_RECV + RECV_BYTES;

// barriers (8 bytes each, from OFF_MISC)
constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2 /* [2][5] */, B_KEMPTY = 12 /* [2] */,
              B_SFULL = 14 /* [2] */, B_PFULL = 16, B_PRECV = 17, B_SRECV = 18, B_RECVFREE = 19, B_PVDONE = 20,
              B_LRECV = 21, N_BARS = 22;
constexpr int M_TMEM = N_BARS * 8;
constexpr int M_ABORT = M_TMEM + 4;
constexpr int M_NEED = M_TMEM + 8;           // int[2]: a head's max moved, per tile parity
constexpr int M_PFLAG = M_TMEM + 16;         // int: the peer rescaled some head this tile (peer-written)
constexpr int M_DUMMY = M_TMEM + 20;         // int: target of the peer's "receive buffer free" store
constexpr int M_MRUN = 256;                  // float[32] own heads, log2 units
constexpr int M_ALPHA = M_MRUN + 128;        // float[32] own heads
constexpr int M_LOWN = M_ALPHA + 128;        // float[32] own heads
constexpr int M_PALPHA = M_LOWN + 128;       // float[32] the peer's heads (peer-written)
constexpr int M_PL = M_PALPHA + 128;         // float[32] the peer's heads' row sums (peer-written)
constexpr int M_RED = M_PL + 128;            // float[4 quadrants][32 heads]
constexpr int MISC_BYTES = M_RED + 512;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "pair tile layout exceeds the shared memory of one CTA");

#ifndef DSA_MLAP_SM_WARPS
#define DSA_MLAP_SM_WARPS 16
#endif
constexpr int SM_WARPS = DSA_MLAP_SM_WARPS, GA_WARPS = 7;  // softmax warps: 16 (8 heads each) or 8 (16)
constexpr int SM_THREADS = SM_WARPS * 32, GA_THREADS = GA_WARPS * 32;
constexpr int MMA_WARP = SM_WARPS + GA_WARPS;
constexpr int THREADS = (MMA_WARP + 1) * 32;
constexpr int TMEM_COLS = 256;
constexpr uint32_t TM_O = 0, TM_S = 128;     // O^T blocks at 0, 64; S^T buffers at 128, 192
constexpr int HPW = 32 / (SM_WARPS / 4);     // own heads per softmax warp
constexpr int OCOLS = 64 / (SM_WARPS / 4);   // O^T columns (heads) per softmax thread
static_assert(HPW == 8 || HPW == 16, "softmax warps: 16 or 8");

struct Params {
  const uint16_t* q;      // [n_q,64,576] bf16
  const uint8_t* kv;      // [n_tokens, row_stride] bf16
  const int32_t* idx;     // [n_q, k]
  uint16_t* out;          // [n_q,64,512] bf16
  float* lse;             // [n_q,64] or null
  int64_t row_stride;     // elements
  int64_t n_tokens;
  int32_t n_q;
  int32_t k;
  int64_t valid0;         // >= 0: idx row i holds min(k, valid0 + i) valid entries first; < 0: k
  float scale_log2;
  int* status;
  uint64_t wait_ns;
};

__device__ __forceinline__ int32_t row_tiles(const Params& p, int32_t row) {
  int64_t v = p.k;
  if (p.valid0 >= 0) v = min(static_cast<int64_t>(p.k), p.valid0 + row);
  return static_cast<int32_t>((max(v, static_cast<int64_t>(0)) + TILE - 1) / TILE);
}

// Byte offset of 16-byte chunk c (0..3) of row r in a no-swizzle K-major region of 4 chunks per
// row: core matrices of 8 rows x 16 B, 4 of them along K per 8-row group.
__host__ __device__ __forceinline__ uint32_t noswz_off(uint32_t r, uint32_t c) {
  return (r >> 3) * 512u + c * 128u + (r & 7u) * 16u;
}

// Max (or sum) over the 32 lanes for 8 per-lane values; every lane ends with the result for
// value index head8_of_lane(lane).
template <bool MAX>
__device__ __forceinline__ float warp_reduce8(const float (&v)[8], int lane) {
  float a[4], b2[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[4 + i] : v[i], give = hi ? v[i] : v[4 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 16);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 8;
    const float keep = hi ? a[2 + i] : a[i], give = hi ? a[i] : a[2 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 8);
    b2[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
  float c;
  {
    const bool hi = lane & 4;
    const float keep = hi ? b2[1] : b2[0], give = hi ? b2[0] : b2[1];
    const float o = __shfl_xor_sync(0xffffffffu, give, 4);
    c = MAX ? fmaxf(keep, o) : keep + o;
  }
  float o = __shfl_xor_sync(0xffffffffu, c, 2);
  c = MAX ? fmaxf(c, o) : c + o;
  o = __shfl_xor_sync(0xffffffffu, c, 1);
  return MAX ? fmaxf(c, o) : c + o;
}
__device__ __forceinline__ int head8_of_lane(int lane) {
  return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

// Max (or sum) over the 32 lanes for 16 per-lane values; lanes 2i and 2i+1 end with value i.
template <bool MAX>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16], int lane) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[8 + i] : v[i], give = hi ? v[i] : v[8 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 16);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int w = 8, bit = 8; w >= 2; w >>= 1, bit >>= 1) {
#pragma unroll
    for (int i = 0; i < w / 2; ++i) {
      const bool hi = lane & bit;
      const float keep = hi ? a[w / 2 + i] : a[i], give = hi ? a[i] : a[w / 2 + i];
      const float o = __shfl_xor_sync(0xffffffffu, give, bit);
      a[i] = MAX ? fmaxf(keep, o) : keep + o;
    }
  }
  const float o = __shfl_xor_sync(0xffffffffu, a[0], 1);
  return MAX ? fmaxf(a[0], o) : a[0] + o;
}

// The per-warp head reduction for HPW values and where its results sit.
template <bool MAX>
__device__ __forceinline__ float reduce_heads(const float (&v)[HPW], int lane) {
  if constexpr (HPW == 8) return warp_reduce8<MAX>(v, lane);
  else return warp_reduce16<MAX>(v, lane);
}
__device__ __forceinline__ int reduced_head(int lane) { return HPW == 8 ? head8_of_lane(lane) : lane >> 1; }
__device__ __forceinline__ bool reduced_writer(int lane) { return HPW == 8 ? (lane & 3) == 0 : (lane & 1) == 0; }

template <int N>
__device__ __forceinline__ void tmem_ld2(uint32_t ta, uint32_t tb, uint32_t (&a)[N], uint32_t (&b)[N]) {
  if constexpr (N == 8) {
    DSA_TMEM_LD_X8_NOWAIT(ta, a);
    DSA_TMEM_LD_X8_NOWAIT(tb, b);
    DSA_TMEM_WAIT_LD_X8X2(a, b);
  } else {
    DSA_TMEM_LD_X16(ta, a);
    DSA_TMEM_LD_X16(tb, b);
  }
}

__global__ void __launch_bounds__(THREADS, 1) sparse_mla_pair_kernel(Params p) {
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
  volatile int* peer_flag = reinterpret_cast<volatile int*>(misc + M_PFLAG);
  float* m_run = reinterpret_cast<float*>(misc + M_MRUN);
  float* alpha = reinterpret_cast<float*>(misc + M_ALPHA);
  float* l_own = reinterpret_cast<float*>(misc + M_LOWN);
  volatile float* p_alpha = reinterpret_cast<volatile float*>(misc + M_PALPHA);
  volatile float* p_l = reinterpret_cast<volatile float*>(misc + M_PL);
  float* red = reinterpret_cast<float*>(misc + M_RED);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (cluster_size() != 2) {  // launched without its CTA pair: touch no peer memory
    if (threadIdx.x == 0) atomicOr(p.status, DEVERR_LAUNCH);
    return;
  }
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const uint32_t cid = cluster_id_x(), ncl = cluster_count_x();

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), GA_THREADS);
    mbar_init(bar(B_QEMPTY), 1);
    for (int b = 0; b < 2; ++b) {
      for (int d = 0; d <= NSUB; ++d) mbar_init(bar(B_KFULL + 5 * b + d), GA_THREADS);
      mbar_init(bar(B_KEMPTY + b), 1);
      mbar_init(bar(B_SFULL + b), 1);
    }
    mbar_init(bar(B_PFULL), SM_THREADS);
    // barriers fed by the peer's st.async bytes: one local arrival (the arming) + the bytes
    mbar_init(bar(B_PRECV), 1);
    mbar_init(bar(B_SRECV), 1);
    mbar_init(bar(B_RECVFREE), 1);
    mbar_init(bar(B_LRECV), 1);
    mbar_init(bar(B_PVDONE), 2);  // PV completion of this CTA and of the peer (multicast commits)
    *abort_flag = 0;
    need_flags[0] = 0;
    need_flags[1] = 0;
    fence_mbar_init();
    // arm the first phase of every barrier the peer's stores complete
    mbar_arrive_expect_tx(bar(B_SRECV), RECV_BYTES);
    mbar_arrive_expect_tx(bar(B_PRECV), PRECV_BYTES);
    mbar_arrive_expect_tx(bar(B_RECVFREE), 4);
    mbar_arrive_expect_tx(bar(B_LRECV), 128);
  }
  if (warp == MMA_WARP) tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers exist before any remote arrival
  const uint32_t tmem = *tmem_holder;

  if (warp >= SM_WARPS && warp < MMA_WARP) {
    // ================================================================= gather warps
    const int g = threadIdx.x - SM_THREADS;
    const int dim0 = 256 * static_cast<int>(rank), rope0 = 512 + 32 * static_cast<int>(rank);
    uint32_t gtile = 0;
    bool ok = true;
    for (int32_t row = cid, it_n = 0; ok && row < p.n_q; row += ncl, ++it_n) {
      // ---- this CTA's dims of the query row
      if (!mbar_wait(bar(B_QEMPTY), (it_n & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + static_cast<int64_t>(row) * 64 * 576);
      for (int c = g; c < 64 * 36; c += GA_THREADS) {
        const int h = c / 36, part = c % 36;
        if (part < 32) {
          cp_async16(base + OFF_Q + (part >> 3) * SUB_Q + sw128_off(h, part & 7), qsrc + h * 1152 + dim0 * 2 + part * 16,
                     16);
        } else {
          cp_async16(base + OFF_Q + NSUB * SUB_Q + noswz_off(h, part - 32), qsrc + h * 1152 + rope0 * 2 + (part - 32) * 16,
                     16);
        }
      }
      cp_async_arrive_noinc(bar(B_QFULL));
      const int32_t n_tiles = row_tiles(p, row);
      const int32_t* idx_row = p.idx + static_cast<int64_t>(row) * p.k;
      for (int32_t t = 0; t < n_tiles; ++t, ++gtile) {
        const uint32_t b = gtile & 1;
        // this thread's keys and sources: value chunks c = g + i*GA (key c/8, chunk c%8), RoPE
        // chunks c = g + i*GA (key c/4, chunk c%4)
        constexpr int MV = (1024 + GA_THREADS - 1) / GA_THREADS, MR = (512 + GA_THREADS - 1) / GA_THREADS;
        const uint8_t* sv[MV];
        uint32_t nv[MV];
        const uint8_t* sr[MR];
        uint32_t nr[MR];
#pragma unroll
        for (int i = 0; i < MV; ++i) {
          const int c = g + i * GA_THREADS;
          int64_t r = -1;
          if (c < 1024) {
            const int32_t jj = t * TILE + (c >> 3);
            const int32_t v = jj < p.k ? idx_row[jj] : -1;
            if (v >= 0 && v < p.n_tokens) r = v;
            else if (v >= p.n_tokens) atomicOr(p.status, DEVERR_BOUNDS);
          }
          sv[i] = p.kv + (r >= 0 ? r : 0) * p.row_stride * 2 + dim0 * 2 + (c & 7) * 16;
          nv[i] = r >= 0 ? 16u : 0u;
        }
#pragma unroll
        for (int i = 0; i < MR; ++i) {
          const int c = g + i * GA_THREADS;
          int64_t r = -1;
          if (c < 512) {
            const int32_t jj = t * TILE + (c >> 2);
            const int32_t v = jj < p.k ? idx_row[jj] : -1;
            if (v >= 0 && v < p.n_tokens) r = v;
          }
          sr[i] = p.kv + (r >= 0 ? r : 0) * p.row_stride * 2 + rope0 * 2 + (c & 3) * 16;
          nr[i] = r >= 0 ? 16u : 0u;
        }
        if (!mbar_wait(bar(B_KEMPTY + b), ((gtile >> 1) & 1) ^ 1, abort_flag, p.status, p.wait_ns)) {
          ok = false;
          break;
        }
        const uint32_t tb = base + OFF_KV + b * TILE_BYTES;
        for (int d = 0; d < NSUB; ++d) {
#pragma unroll
          for (int i = 0; i < MV; ++i) {
            const int c = g + i * GA_THREADS;
            if (c < 1024) cp_async16(tb + d * SUB_KV + sw128_off(c >> 3, c & 7), sv[i] + d * 128, nv[i]);
          }
          cp_async_arrive_noinc(bar(B_KFULL + 5 * b + d));
        }
#pragma unroll
        for (int i = 0; i < MR; ++i) {
          const int c = g + i * GA_THREADS;
          if (c < 512) cp_async16(tb + NSUB * SUB_KV + noswz_off(c >> 2, c & 3), sr[i], nr[i]);
        }
        cp_async_arrive_noinc(bar(B_KFULL + 5 * b + NSUB));
      }
    }
  } else if (warp == MMA_WARP) {
    // ================================================================= MMA issuer
    // Two cursors over the CTA's tile sequence: S^T of tile s (as its sub-tiles land) and PV of
    // tile v < s (once its P^T is complete), issued in whichever order they become ready, so that
    // PV of one tile never waits for the gather of the next.  S^T(s) writes the S buffer of
    // tile s - 2, so it waits until PV(s - 2) has been issued (its softmax is done).
    if (lane == 0) {
      constexpr uint32_t ID_S = make_idesc(1, 1, 0, 0, 128, 64);
      constexpr uint32_t ID_PV = make_idesc(1, 1, 1, 1, 128, 64);
      struct Cursor {
        int32_t row, it_n, t, n_tiles;
        uint32_t g;
      };
      auto first_row = [&](Cursor& c) {
        c.row = cid;
        c.it_n = 0;
        c.t = 0;
        c.g = 0;
        c.n_tiles = c.row < p.n_q ? row_tiles(p, c.row) : 0;
      };
      auto next_row = [&](Cursor& c) {
        c.row += ncl;
        ++c.it_n;
        c.t = 0;
        c.n_tiles = c.row < p.n_q ? row_tiles(p, c.row) : 0;
      };
      Cursor cs, cv;
      first_row(cs);
      first_row(cv);
      while (cv.row < p.n_q && cv.t >= cv.n_tiles) next_row(cv);  // PV skips rows without tiles
      bool q_ready = false;
      int d_next = 0;  // next sub-tile of S^T(cs.g)
      uint64_t t_idle = globaltimer_ns();
      while (cv.row < p.n_q || cs.row < p.n_q) {
        bool progress = false;
        // ---- S side
        if (cs.row < p.n_q && cs.g <= cv.g + 1) {
          if (!q_ready) {
            if (mbar_try_wait(bar(B_QFULL), cs.it_n & 1)) {
              fence_async_smem();
              tc_fence_after();
              q_ready = true;
              progress = true;
              if (cs.n_tiles == 0) {  // nothing to attend: release the query row at once
                mma_commit(bar(B_QEMPTY));
                next_row(cs);
                q_ready = false;
              }
            }
          } else {
            const uint32_t b = cs.g & 1;
            const uint32_t ds = tmem + TM_S + 64u * b;
            const uint32_t tb = base + OFF_KV + b * TILE_BYTES;
            while (d_next <= NSUB && mbar_try_wait(bar(B_KFULL + 5 * b + d_next), (cs.g >> 1) & 1)) {
              fence_async_smem();  // cp.async writes -> MMA reads
              tc_fence_after();
              const int d = d_next;
              if (d < NSUB) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t a = make_sdesc(tb + d * SUB_KV + kk * 32, 16, 1024);
                  const uint64_t bd = make_sdesc(base + OFF_Q + d * SUB_Q + kk * 32, 16, 1024);
                  mma_f16(ds, a, bd, ID_S, (d | kk) != 0);
                }
              } else {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                  const uint64_t a = make_sdesc_noswz(tb + NSUB * SUB_KV + kk * 256, 128, 512);
                  const uint64_t bd = make_sdesc_noswz(base + OFF_Q + NSUB * SUB_Q + kk * 256, 128, 512);
                  mma_f16(ds, a, bd, ID_S, 1);
                }
              }
              ++d_next;
              progress = true;
            }
            if (d_next > NSUB) {
              mma_commit(bar(B_SFULL + b));
              d_next = 0;
              ++cs.g;
              if (++cs.t == cs.n_tiles) {
                mma_commit(bar(B_QEMPTY));
                next_row(cs);
                q_ready = false;
              }
            }
          }
        }
        // ---- PV side
        if (cv.g < cs.g && mbar_try_wait(bar(B_PFULL), cv.g & 1)) {
          fence_async_smem();  // P^T written by the generic proxy (also by the peer) -> MMA reads
          tc_fence_after();
          const uint32_t tb = base + OFF_KV + (cv.g & 1) * TILE_BYTES;
#pragma unroll 1
          for (int mb = 0; mb < 2; ++mb) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = make_sdesc(tb + 2 * mb * SUB_KV + kk * 2048, SUB_KV, 1024);
              const uint64_t bd = make_sdesc(base + OFF_P + kk * 2048, SUB_KV, 1024);
              mma_f16(tmem + TM_O + 64u * mb, a, bd, ID_PV, (cv.t > 0 || kk > 0));
            }
          }
          mma_commit(bar(B_KEMPTY + (cv.g & 1)));
          mma_commit_multicast(bar(B_PVDONE), 0x3);
          ++cv.g;
          if (++cv.t == cv.n_tiles) {
            next_row(cv);
            while (cv.row < p.n_q && cv.t >= cv.n_tiles) next_row(cv);
          }
          progress = true;
        }
        const uint64_t now = globaltimer_ns();
        if (progress) {
          t_idle = now;
        } else {
          if (*abort_flag) break;
          if (now - t_idle > p.wait_ns) {
            *abort_flag = 1;
            atomicOr(p.status, DEVERR_TIMEOUT);
            break;
          }
        }
      }
    }
  } else {
    // ================================================================= softmax / output warps
    // Exchanges with the peer are st.async stores whose bytes complete a transaction count on a
    // barrier of the receiving CTA; each receiving barrier is armed (arrive + expect_tx) by this
    // CTA's thread 0 once the previous phase has completed, so no cluster-scope fence is needed.
    const int quad = warp & 3, hg = warp >> 2;
    const int key = quad * 32 + lane;                  // TMEM lane: key of S^T, dim of an O^T block
    const int st = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t own_col = 32u * rank + HPW * hg;    // own heads' columns in S^T
    const uint32_t peer_col = 32u * peer + HPW * hg;   // the peer's heads' columns in S^T
    const int oh = HPW * hg;                           // own head index (0..31) of value 0
    const uint32_t peer_base = map_to_cta(base, peer);
    const uint32_t peer_recv = peer_base + OFF_RECV + key * 128 + oh * 4;
    const uint32_t peer_bar = peer_base + OFF_MISC;    // the peer's barrier 0
    const bool head_lane = quad == 0 && reduced_writer(lane);   // holds a reduced value (reduced_head)
    uint32_t gtile = 0;
    bool ok = true;
    for (int32_t row = cid, it_n = 0; ok && row < p.n_q; row += ncl, ++it_n) {
      const int32_t n_tiles = row_tiles(p, row);
      const int32_t* idx_row = p.idx + static_cast<int64_t>(row) * p.k;
      if (quad == 0 && lane < HPW) m_run[oh + lane] = -INFINITY;
      named_bar(1, SM_THREADS);
      bool fail = false;
      float lsum[HPW];
#pragma unroll
      for (int i = 0; i < HPW; ++i) lsum[i] = 0.f;
      int32_t v_next = n_tiles > 0 && key < p.k ? idx_row[key] : -1;
      for (int32_t t = 0; t < n_tiles; ++t, ++gtile) {
        const uint32_t b = gtile & 1;
        const int32_t v = v_next;
        {  // the next tile's index, loaded under this tile's work
          const int32_t jn = (t + 1) * TILE + key;
          v_next = t + 1 < n_tiles && jn < p.k ? idx_row[jn] : -1;
        }
        const bool valid = v >= 0 && v < p.n_tokens;
        // ---- 1. this CTA's partial logits
        {
          const bool got = mbar_wait(bar(B_SFULL + b), (gtile >> 1) & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
        }
        tc_fence_after();
        uint32_t xp[HPW], xo[HPW];
        if (!fail) tmem_ld2<HPW>(tmem + TM_S + 64u * b + peer_col + lane_off, tmem + TM_S + 64u * b + own_col + lane_off, xp, xo);
        // ---- 2. the peer's heads' partials into the peer's receive buffer, once it has read the
        // previous ones
        if (gtile > 0) {
          const bool got = mbar_wait(bar(B_RECVFREE), (gtile - 1) & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
          if (st == 0) mbar_arrive_expect_tx(bar(B_RECVFREE), 4);
        }
        if (!fail) {
#pragma unroll
          for (int c = 0; c < HPW / 4; ++c)
            st_async_v4(peer_recv + 16 * c, xp[4 * c], xp[4 * c + 1], xp[4 * c + 2], xp[4 * c + 3],
                        peer_bar + 8u * B_SRECV);
        }
        // ---- 3. the peer's partials of this CTA's heads
        float z[HPW];
        {
          const bool got = mbar_wait(bar(B_SRECV), gtile & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
          if (st == 0) mbar_arrive_expect_tx(bar(B_SRECV), RECV_BYTES);
        }
        if (!fail) {
#pragma unroll
          for (int c = 0; c < HPW / 4; ++c) {
            const float4 r4 = *reinterpret_cast<const float4*>(smem + OFF_RECV + key * 128 + oh * 4 + 16 * c);
            z[4 * c] = valid ? (__uint_as_float(xo[4 * c]) + r4.x) * p.scale_log2 : -INFINITY;
            z[4 * c + 1] = valid ? (__uint_as_float(xo[4 * c + 1]) + r4.y) * p.scale_log2 : -INFINITY;
            z[4 * c + 2] = valid ? (__uint_as_float(xo[4 * c + 2]) + r4.z) * p.scale_log2 : -INFINITY;
            z[4 * c + 3] = valid ? (__uint_as_float(xo[4 * c + 3]) + r4.w) * p.scale_log2 : -INFINITY;
          }
        } else {
#pragma unroll
          for (int i = 0; i < HPW; ++i) z[i] = -INFINITY;
        }
        // ---- 4. lazy running max of the own heads (reduced only when a logit passes it by > 8)
        volatile int* need = need_flags + (gtile & 1);
        bool exceed = false;
#pragma unroll
        for (int c = 0; c < HPW / 4; ++c) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_run + oh + 4 * c);
          exceed |= (z[4 * c] > m4.x + 8.f) | (z[4 * c + 1] > m4.y + 8.f) | (z[4 * c + 2] > m4.z + 8.f) |
                    (z[4 * c + 3] > m4.w + 8.f);
        }
        if (__any_sync(0xffffffffu, exceed) && lane == 0) *need = 1;
        if (named_bar_or(1, SM_THREADS, fail)) {
          ok = false;
          break;
        }
        // every thread has read its received partials: the peer may send the next ones
        if (st == 0) st_async_b32(peer_base + OFF_MISC + M_DUMMY, 0u, peer_bar + 8u * B_RECVFREE);
        if (st == 0) need_flags[(gtile + 1) & 1] = 0;
        const bool resc_own = *need != 0;
        if (resc_own) {
          const float wmax = reduce_heads<true>(z, lane);
          if (reduced_writer(lane)) red[quad * 32 + oh + reduced_head(lane)] = wmax;
          named_bar(1, SM_THREADS);
          if (head_lane) {
            const int h = oh + reduced_head(lane);
            const float tmax = fmaxf(fmaxf(red[h], red[32 + h]), fmaxf(red[64 + h], red[96 + h]));
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
          for (int c = 0; c < HPW / 4; ++c) {
            const float4 a4 = *reinterpret_cast<const float4*>(alpha + oh + 4 * c);
            lsum[4 * c] *= a4.x;
            lsum[4 * c + 1] *= a4.y;
            lsum[4 * c + 2] *= a4.z;
            lsum[4 * c + 3] *= a4.w;
          }
        }
        // ---- 5. probabilities of the own heads -> HPW/8 16-byte chunks of this key's P^T row
        uint32_t pk[HPW / 2];
#pragma unroll
        for (int c = 0; c < HPW / 4; ++c) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_run + oh + 4 * c);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 4 * c + 2 * e;
            const float p0 = ex2_approx(z[h] - (mm[2 * e] == -INFINITY ? 0.f : mm[2 * e]));
            const float p1 = ex2_approx(z[h + 1] - (mm[2 * e + 1] == -INFINITY ? 0.f : mm[2 * e + 1]));
            lsum[h] += p0;
            lsum[h + 1] += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[h / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        }
        // ---- 6. P^T columns of the own heads (and their rescale factors) into both CTAs' P^T,
        // once PV of the previous tile is done in both
        if (gtile > 0) {
          const bool got = mbar_wait(bar(B_PVDONE), (gtile - 1) & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
        }
        if (!fail) {
#pragma unroll
          for (int c = 0; c < HPW / 8; ++c) {
            const uint32_t poff = sw128_off(key, (32u * rank + oh) / 8 + c);
            *reinterpret_cast<uint4*>(smem + OFF_P + poff) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            st_async_v4(peer_base + OFF_P + poff, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3],
                        peer_bar + 8u * B_PRECV);
          }
          if (head_lane) {
            const int h = oh + reduced_head(lane);
            st_async_b32(peer_base + OFF_MISC + M_PALPHA + 4u * h, __float_as_uint(resc_own ? alpha[h] : 1.f),
                         peer_bar + 8u * B_PRECV);
          }
          if (st == 0) st_async_b32(peer_base + OFF_MISC + M_PFLAG, resc_own ? 1u : 0u, peer_bar + 8u * B_PRECV);
        }
        // ---- 7. the peer's P^T columns and rescale factors
        {
          const bool got = mbar_wait(bar(B_PRECV), gtile & 1, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);
          if (st == 0) mbar_arrive_expect_tx(bar(B_PRECV), PRECV_BYTES);
        }
        const bool peer_resc = *peer_flag != 0;
        if ((resc_own || peer_resc) && t > 0 && !fail) {
          // O^T (this CTA's dims on lanes, all 64 heads on columns) *= alpha of each head; PV of
          // the previous tile is done (step 6)
          tc_fence_after();
#pragma unroll 1
          for (int blk = 0; blk < 2 * OCOLS / 16; ++blk) {
            const int mb = blk / (OCOLS / 16), part = blk % (OCOLS / 16);
            uint32_t x[16];
            const uint32_t ta = tmem + TM_O + 64u * mb + OCOLS * hg + 16u * part + lane_off;
            DSA_TMEM_LD_X16(ta, x);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int h = OCOLS * hg + 16 * part + c;
              const bool mine = (h >> 5) == static_cast<int>(rank);
              const float a = mine ? (resc_own ? alpha[h & 31] : 1.f) : p_alpha[h & 31];
              x[c] = __float_as_uint(__uint_as_float(x[c]) * a);
            }
            DSA_TMEM_ST_X16(ta, x);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL));
      }
      if (!ok) break;
      // ---- end of the row: wait for the last PV in both CTAs, exchange the row sums, write out
      if (n_tiles > 0) {
        const bool got = mbar_wait(bar(B_PVDONE), (gtile - 1) & 1, abort_flag, p.status, p.wait_ns);
        fail = __any_sync(0xffffffffu, fail || !got);
        tc_fence_after();
      }
      {
        const float wsum = reduce_heads<false>(lsum, lane);
        if (reduced_writer(lane)) red[quad * 32 + oh + reduced_head(lane)] = wsum;
      }
      if (named_bar_or(1, SM_THREADS, fail)) break;
      if (head_lane) {
        const int h = oh + reduced_head(lane);
        const float l = red[h] + red[32 + h] + red[64 + h] + red[96 + h];
        l_own[h] = l;
        st_async_b32(peer_base + OFF_MISC + M_PL + 4u * h, __float_as_uint(l), peer_bar + 8u * B_LRECV);
        if (p.lse) {
          p.lse[static_cast<int64_t>(row) * 64 + 32 * rank + h] =
              l > 0.f ? (m_run[h] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      }
      {
        const bool got = mbar_wait(bar(B_LRECV), it_n & 1, abort_flag, p.status, p.wait_ns);
        fail = __any_sync(0xffffffffu, fail || !got);
        if (st == 0) mbar_arrive_expect_tx(bar(B_LRECV), 128);
      }
      if (named_bar_or(1, SM_THREADS, fail)) break;  // l_own complete; the peer's sums arrived
      uint16_t* orow = p.out + static_cast<int64_t>(row) * 64 * 512 + 256 * rank;
#pragma unroll 1
      for (int blk = 0; blk < 2 * OCOLS / 16; ++blk) {
        const int mb = blk / (OCOLS / 16), part = blk % (OCOLS / 16);
        uint32_t x[16];
        if (n_tiles > 0) {
          DSA_TMEM_LD_X16(tmem + TM_O + 64u * mb + OCOLS * hg + 16u * part + lane_off, x);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) x[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int h = OCOLS * hg + 16 * part + c;
          const float l = (h >> 5) == static_cast<int>(rank) ? l_own[h & 31] : p_l[h & 31];
          const float o = l > 0.f ? __uint_as_float(x[c]) / l : 0.f;
          const __nv_bfloat16 ob = __float2bfloat16_rn(o);
          orow[h * 512 + mb * 128 + key] = *reinterpret_cast<const uint16_t*>(&ob);
        }
      }
      tc_fence_before();
      named_bar(1, SM_THREADS);  // m_run / l_own / red are reused by the next row
    }
    // the peer's last "receive buffer free" store lands here before this CTA may exit
    if (ok && gtile > 0) mbar_wait(bar(B_RECVFREE), (gtile - 1) & 1, abort_flag, p.status, p.wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the peer may still write its shared memory
  tc_fence_after();
  if (warp == MMA_WARP) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace mlap
}  // namespace dsa

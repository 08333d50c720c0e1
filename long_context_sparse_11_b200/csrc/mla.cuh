// Step a6 (+ a7 paged address translation / FP8 dequant, a8 MTP rows): sparse MLA
// attention of one query row (64 heads) over its selected latent rows.
//
// Both contractions run "transposed" so that every tcgen05.mma is M = 128 and the
// 64 x 512 fp32 output fits in 256 TMEM columns:
//   S^T[key, head]  = KV[key, 0:576] . Q[head, 0:576]        M = 128 keys,  N = 64 heads
//   O^T[dim, head] += V^T[dim, key]  . P^T[key, head]        M = 128 dims (x4), N = 64 heads
// S^T puts one key on each TMEM lane, so masking, the per-key FP8 scale and the P^T row are
// thread-local to the softmax thread of that lane; only the per-head max and sum cross lanes
// (shuffle transpose-reduce + a shared-memory step over the 4 lane quadrants).  The running
// max is updated lazily (only when a head's max grows by more than 2^8), so O^T is rarely
// rescaled in TMEM.
//
// Shared memory: Q as 9 K-major 64-dim sub-tiles [64 heads x 128 B] (72 KB) and one
// 128-key KV tile as 9 sub-tiles [128 keys x 128 B] (144 KB), 128-byte swizzled.  The same
// KV bytes are the K-major A operand of S^T and the MN-major A operand (V^T) of O^T; once
// S^T has completed, the RoPE sub-tile (dims 512..575) receives P^T [128 keys x 64 heads],
// the MN-major B operand of the second MMA.
//
// Pipelining with one KV tile: every sub-tile has its own "full" barrier and every pair of
// sub-tiles (one 128-dim block of V) its own "empty" barrier, committed when the PV MMAs of
// that block complete.  The gather of tile j+1 therefore streams into the sub-tiles that
// PV(j) has finished with while PV(j) still runs on the others, and S^T(j+1) starts as soon
// as its first sub-tile lands.  CTAs are persistent over (query row, key split) items, or,
// for short decode batches, over equal stream-K ranges of the (row, key tile) sequence whose
// cut rows are merged by the combine kernel.
//
// Rows are gathered with 16-byte cp.async whose completion the hardware reports to the
// sub-tile's barrier (bf16 cache), or with 16-byte loads + e4m3 -> f16 conversion (paged FP8
// cache; the MMAs then run kind::f16 on f16 operands, exact for e4m3 values; the per-token
// scale is applied to the logits and folded into P^T).
//
// Warps 0..SM_WARPS-1: softmax / output (warp w: lane quadrant w%4, HPW heads from HPW*(w/4)),
// and on the FP8 path part of the gather; the next GA_WARPS (7) warps: query rows and the KV gather; the
// last warp: TMEM owner + MMA issuer.
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
constexpr int N_BARS = 18;
constexpr int M_TMEM = N_BARS * 8;
constexpr int M_ABORT = M_TMEM + 4;
constexpr int M_NEED = M_TMEM + 8;   // int[2]: "a head's max moved" flag per tile parity
constexpr int M_MRUN = 256;          // float[64], log2 units
constexpr int M_ALPHA = M_MRUN + 256;
constexpr int M_LTOT = M_ALPHA + 256;
constexpr int M_RED = M_LTOT + 256;  // float[4 quadrants][64 heads]
constexpr int MISC_BYTES = M_RED + 1024;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
#ifndef DSA_MLA_SM_WARPS
#define DSA_MLA_SM_WARPS 16
#endif
// softmax warps: 4 lane quadrants x (64 / HPW) head groups; with 8 (16 warps in all, 4 per SM
// sub-partition) each thread may use 128 registers, with 16 (24 warps) 80
#ifndef DSA_MLA_GA_WARPS
#define DSA_MLA_GA_WARPS 7
#endif
constexpr int SM_WARPS = DSA_MLA_SM_WARPS, GA_WARPS = DSA_MLA_GA_WARPS;
constexpr int HPW = 64 / (SM_WARPS / 4);  // heads per softmax warp
static_assert(HPW == 16 || HPW == 32, "softmax warps: 8 or 16");
constexpr int SM_THREADS = SM_WARPS * 32, GA_THREADS = GA_WARPS * 32;
// Threads that gather KV rows.  bf16 cache: the gather warps alone (cp.async issue is the
// limit, and the softmax warps would join only after their softmax, late for the first
// sub-tiles).  FP8 cache: the softmax warps help with the load + convert + store.
template <bool PAGED>
__host__ __device__ constexpr bool sm_gather() { return PAGED; }
template <bool PAGED>
__host__ __device__ constexpr int n_gather() { return sm_gather<PAGED>() ? SM_THREADS + GA_THREADS : GA_THREADS; }
constexpr int MMA_WARP = SM_WARPS + GA_WARPS;
constexpr int THREADS = (MMA_WARP + 1) * 32;
constexpr int TMEM_COLS = 512;
constexpr uint32_t TM_S = 256;  // S^T buffers at columns 256, 320

// barrier indices
constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 3, B_PVDONE = 4, B_FULL = 5, B_EMPTY = 14;

struct Params {
  const uint16_t* q;         // [n_q,64,576] bf16, or its f16 copy when q_f16 is set (paged only)
  const uint8_t* kv;         // dense bf16 [n_tokens,row_stride] or paged e4m3 [n_pages,64,576]
  const float* kv_scale;     // paged: [n_pages*64]
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* idx;        // [n_idx_rows, k]
  uint16_t* out;             // [n_q,64,512] bf16
  float* lse;                // [n_q,64] or null
  float* part_o;             // partials [n_q*n_split,64,512] fp32 (row r, slot s at r*n_split+s)
  float* part_ml;            // [n_q*n_split,2,64] (m in log2 units, l)
  int64_t row_stride;        // elements (dense)
  int64_t n_tokens;
  int32_t n_q;
  int32_t rows_per_idx;
  int32_t k;
  int32_t n_split;          // slots per row (equal splits, or at most this many stream-K fragments)
  int32_t stream_k;          // (kernels instantiated with SK) 1: CTA c takes the contiguous tile range [c*G/grid, (c+1)*G/grid) of the
                             // n_q x tiles_per_row tiles in row order; rows cut by a range boundary
                             // leave partials per fragment, whole rows are written directly
  int64_t valid0;            // >= 0: idx row i holds its valid entries first, min(k, valid0 + i) of
                             // them (causal prefill); tiles past them are skipped.  < 0: k
  int32_t max_pages;
  int32_t n_pages;
  float scale_log2;          // softmax_scale * log2(e)
  int* status;
  uint64_t wait_ns;
  int32_t q_f16;             // paged: 1 when q was converted to f16 before the launch (q_to_f16_kernel)
};

// Max (or sum) over the 32 lanes of a warp for 32 per-lane values; lane l ends with the
// result for value index l.
template <bool MAX>
__device__ __forceinline__ float warp_reduce32(const float (&v)[32], int lane) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[16 + i] : v[i];
    const float give = hi ? v[i] : v[16 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 16);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int w = 16, bit = 8; w >= 2; w >>= 1, bit >>= 1) {
#pragma unroll
    for (int i = 0; i < w / 2; ++i) {
      const bool hi = lane & bit;
      const float keep = hi ? a[w / 2 + i] : a[i];
      const float give = hi ? a[i] : a[w / 2 + i];
      const float o = __shfl_xor_sync(0xffffffffu, give, bit);
      a[i] = MAX ? fmaxf(keep, o) : keep + o;
    }
  }
  return a[0];
}

// Max (or sum) over the 32 lanes of a warp for 16 per-lane values; lanes 2i and 2i+1 end with
// the result for value index i.
template <bool MAX>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16], int lane) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float keep = hi ? v[8 + i] : v[i];
    const float give = hi ? v[i] : v[8 + i];
    const float o = __shfl_xor_sync(0xffffffffu, give, 16);
    a[i] = MAX ? fmaxf(keep, o) : keep + o;
  }
#pragma unroll
  for (int w = 8, bit = 8; w >= 2; w >>= 1, bit >>= 1) {
#pragma unroll
    for (int i = 0; i < w / 2; ++i) {
      const bool hi = lane & bit;
      const float keep = hi ? a[w / 2 + i] : a[i];
      const float give = hi ? a[i] : a[w / 2 + i];
      const float o = __shfl_xor_sync(0xffffffffu, give, bit);
      a[i] = MAX ? fmaxf(keep, o) : keep + o;
    }
  }
  const float o = __shfl_xor_sync(0xffffffffu, a[0], 1);
  return MAX ? fmaxf(a[0], o) : a[0] + o;
}

// Per-warp head reduction for HPW values: the result for head index i of the warp's group is
// held by lane reduce_lane(i) (32 values: lane i; 16 values: lanes 2i, 2i+1).
template <bool MAX, int N>
__device__ __forceinline__ float warp_reduce_heads(const float (&v)[N], int lane) {
  if constexpr (N == 32) return warp_reduce32<MAX>(v, lane);
  else return warp_reduce16<MAX>(v, lane);
}
template <int N>
__device__ __forceinline__ int reduce_head_of_lane(int lane) { return N == 32 ? lane : lane >> 1; }
template <int N>
__device__ __forceinline__ bool reduce_lane_writes(int lane) { return N == 32 || (lane & 1) == 0; }

template <int N>
__device__ __forceinline__ void tmem_ld_heads(uint32_t taddr, uint32_t (&x)[N]) {
  if constexpr (N == 32) { DSA_TMEM_LD_X32(taddr, x); }
  else { DSA_TMEM_LD_X16(taddr, x); }
}
template <int N>
__device__ __forceinline__ void tmem_st_heads(uint32_t taddr, const uint32_t (&x)[N]) {
  if constexpr (N == 32) { DSA_TMEM_ST_X32(taddr, x); }
  else { DSA_TMEM_ST_X16(taddr, x); }
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

// Work item -> (query row, idx row, first tile, number of tiles, partial slot, written directly).
struct Item {
  int32_t row, irow, j0, n_tiles, split;
  bool direct;
};

// Stream-K: the CTA owning global tile g of G tiles split over `grid` CTAs.
__host__ __device__ __forceinline__ int64_t sk_owner(int64_t g, int64_t G, int64_t grid) {
  return ((g + 1) * grid - 1) / G;
}

// The CTA's sequence of items: strided (row, split) items, or its stream-K tile range.
struct WorkIter {
  int64_t a, b;
};
template <bool SK>
__device__ __forceinline__ WorkIter work_begin(const Params& p) {
  WorkIter w;
  if constexpr (SK) {
    const int64_t G = static_cast<int64_t>(p.n_q) * ((p.k + TILE - 1) / TILE);
    w.a = static_cast<int64_t>(blockIdx.x) * G / gridDim.x;
    w.b = static_cast<int64_t>(blockIdx.x + 1) * G / gridDim.x;
  } else {
    w.a = blockIdx.x;
    w.b = static_cast<int64_t>(p.n_q) * p.n_split;
  }
  return w;
}

__device__ __forceinline__ Item make_item(const Params& p, int32_t item);

template <bool SK>
__device__ __forceinline__ bool work_next(const Params& p, WorkIter& w, Item& it) {
  if (w.a >= w.b) return false;
  if constexpr (!SK) {
    it = make_item(p, static_cast<int32_t>(w.a));
    w.a += gridDim.x;
    return true;
  }
  const int32_t tpr = (p.k + TILE - 1) / TILE;
  const int64_t G = static_cast<int64_t>(p.n_q) * tpr;
  it.row = static_cast<int32_t>(w.a / tpr);
  it.irow = it.row / p.rows_per_idx;
  it.j0 = static_cast<int32_t>(w.a % tpr);
  it.n_tiles = static_cast<int32_t>(min(static_cast<int64_t>(tpr - it.j0), w.b - w.a));
  it.direct = it.j0 == 0 && it.n_tiles == tpr;
  it.split = static_cast<int32_t>(blockIdx.x - sk_owner(static_cast<int64_t>(it.row) * tpr, G, gridDim.x));
  w.a += it.n_tiles;
  return true;
}

__device__ __forceinline__ Item make_item(const Params& p, int32_t item) {
  Item it;
  it.row = item / p.n_split;
  it.split = item % p.n_split;
  it.direct = p.n_split == 1;
  it.irow = it.row / p.rows_per_idx;
  const int32_t all = (p.k + TILE - 1) / TILE;
  const int32_t tps = (all + p.n_split - 1) / p.n_split;
  int32_t used = all;
  if (p.valid0 >= 0) {
    const int64_t v = min(static_cast<int64_t>(p.k), p.valid0 + it.irow);
    used = static_cast<int32_t>((max(v, static_cast<int64_t>(0)) + TILE - 1) / TILE);
  }
  it.j0 = it.split * tps;
  it.n_tiles = max(0, min(it.j0 + tps, used) - it.j0);
  return it;
}

__device__ __forceinline__ uint32_t pack_pair(float a, float b, bool f16) {
  if (f16) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// e4m3 x16 (one 16-byte chunk) -> two 16-byte chunks of f16 (exact).
__device__ __forceinline__ void e4m3x16_to_f16(uint4 raw, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t r[8];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[q4] & 0xFFFFu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[q4] >> 16), __NV_E4M3);
    r[2 * q4] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    r[2 * q4 + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
  }
  o0 = make_uint4(r[0], r[1], r[2], r[3]);
  o1 = make_uint4(r[4], r[5], r[6], r[7]);
}

template <bool PAGED, bool SK>
__global__ void __launch_bounds__(THREADS, 1) sparse_mla_kernel(Params p) {
  grid_dependency_sync();
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
  constexpr bool SM_GATHER = sm_gather<PAGED>();
  constexpr int NG = n_gather<PAGED>();

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), GA_THREADS);
    mbar_init(bar(B_QEMPTY), 1);
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_PFULL), SM_THREADS);
    mbar_init(bar(B_PVDONE), 1);
    // every gathering thread that owns a chunk arrives once per sub-tile (FP8: 512 parts per tile)
    for (int d = 0; d < NSUB; ++d) mbar_init(bar(B_FULL + d), PAGED ? (NG < 512 ? NG : 512) : NG);
    for (int g = 0; g < 4; ++g) mbar_init(bar(B_EMPTY + g), 1);
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

  // One thread's share (g in [0, NG)) of a KV tile: 16-byte chunks c = g, g + NG, ... of every
  // 64-dim sub-tile, chunk c = (key c/8, 16 bytes c%8) for the bf16 cache, or (key c/4, 16 e4m3
  // values c%4) for the paged FP8 cache.  `prepare` reads the tile's indices (issued early so
  // their latency hides behind other work); `issue` writes the sub-tiles in order, each pair
  // once PV of the previous tile has released it.  bf16: cp.async, and the hardware arrives on
  // the sub-tile's "full" barrier when this thread's copies have landed (the thread never waits
  // for them; the MMA issuer fences the async proxy after the barrier).
  // 16-byte chunks per sub-tile: 1,024 for the bf16 cache (128 keys x 8), 512 parts for FP8 (128 x 4)
  constexpr int MAXC = ((PAGED ? 512 : 1024) + NG - 1) / NG;
  struct Plan {
    const uint8_t* src[MAXC];
    uint32_t nb[MAXC], dst[MAXC];
  };
  auto prepare = [&](const Item& it, int32_t t, int g) -> Plan {
    Plan pl;
    const int32_t j = it.j0 + t;
    const int32_t seq_len = PAGED ? p.seq_lens[it.irow] : 0;
    const int32_t* idx_row = p.idx + static_cast<int64_t>(it.irow) * p.k;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = g + i * NG;
      const int key = PAGED ? (c >> 2) : (c >> 3), sub = PAGED ? (c & 3) : (c & 7);
      const int lim = PAGED ? 512 : 1024;
      int64_t r = -1;
      if (c < lim) {
        const int32_t jj = j * TILE + key;
        const int32_t v = jj < p.k ? idx_row[jj] : -1;
        r = kv_row<PAGED>(p, it.irow, v, seq_len);
      }
      if (PAGED) {
        pl.src[i] = p.kv + (r >= 0 ? r : 0) * 576 + sub * 16;
        pl.dst[i] = c < lim ? static_cast<uint32_t>(key * 4 + sub) : 0xFFFFFFFFu;
      } else {
        pl.src[i] = p.kv + (r >= 0 ? r : 0) * p.row_stride * 2 + sub * 16;
        pl.dst[i] = c < lim ? sw128_off(key, sub) : 0xFFFFFFFFu;
      }
      pl.nb[i] = r >= 0 ? 16u : 0u;
    }
    return pl;
  };
  auto issue = [&](const Plan& pl, uint32_t gtile) -> bool {
    const uint32_t par = (gtile & 1) ^ 1;
    if (!PAGED) {
      for (int d = 0; d < NSUB; ++d) {
        if ((d & 1) == 0 &&
            !mbar_wait(bar(d < 8 ? B_EMPTY + d / 2 : B_PVDONE), par, abort_flag, p.status, p.wait_ns))
          return false;
#pragma unroll
        for (int i = 0; i < MAXC; ++i)
          if (pl.dst[i] != 0xFFFFFFFFu)
            cp_async16(base + OFF_KV + d * SUB_KV + pl.dst[i], pl.src[i] + d * 128, pl.nb[i]);
        cp_async_arrive_noinc(bar(B_FULL + d));
      }
    } else {
      // each part: 16 e4m3 values of every sub-tile, all 9 loaded before the first wait (loads do
      // not touch shared memory), converted to f16 and stored once the sub-tile pair is free
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        if (pl.dst[i] == 0xFFFFFFFFu) continue;
        const int key = pl.dst[i] >> 2, part = pl.dst[i] & 3;
        uint4 raw[NSUB];
#pragma unroll
        for (int d = 0; d < NSUB; ++d)
          raw[d] = pl.nb[i] ? __ldg(reinterpret_cast<const uint4*>(pl.src[i] + d * 64)) : make_uint4(0, 0, 0, 0);
        const bool last = i + 1 == MAXC || pl.dst[i + 1 < MAXC ? i + 1 : i] == 0xFFFFFFFFu;
        // no early return inside the unrolled loop, so raw[] stays in registers
        bool free_ok = true;
#pragma unroll
        for (int d = 0; d < NSUB; ++d) {
          if ((d & 1) == 0 && free_ok)
            free_ok = mbar_wait(bar(d < 8 ? B_EMPTY + d / 2 : B_PVDONE), par, abort_flag, p.status, p.wait_ns);
          if (!free_ok) continue;
          uint4 o0, o1;
          e4m3x16_to_f16(raw[d], o0, o1);
          *reinterpret_cast<uint4*>(smem + OFF_KV + d * SUB_KV + sw128_off(key, 2 * part)) = o0;
          *reinterpret_cast<uint4*>(smem + OFF_KV + d * SUB_KV + sw128_off(key, 2 * part + 1)) = o1;
          if (last) {
            fence_async_smem();
            mbar_arrive(bar(B_FULL + d));
          }
        }
        if (!free_ok) return false;
      }
    }
    return true;
  };

  if (warp >= SM_WARPS && warp < MMA_WARP) {
    // ================================================================= gather warps
    const int gq = threadIdx.x - SM_THREADS;  // query-row loader index
    uint32_t gtile = 0;
    bool ok = true;
    WorkIter wk = work_begin<SK>(p);
    Item it;
    for (int32_t it_n = 0; ok && work_next<SK>(p, wk, it); ++it_n) {
      // ---- query row -> 9 K-major sub-tiles (bf16 copy, or bf16 -> f16 for the FP8 cache path)
      if (!mbar_wait(bar(B_QEMPTY), (it_n & 1) ^ 1, abort_flag, p.status, p.wait_ns)) break;
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q + static_cast<int64_t>(it.row) * 64 * 576);
      constexpr int QCH = 64 * 72;  // 16-byte chunks of one query row
      if (!PAGED) {
        for (int c = gq; c < QCH; c += GA_THREADS) {
          const int h = c / 72, ch = c % 72;
          cp_async16(base + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7), qsrc + h * 1152 + ch * 16, 16);
        }
      } else if (p.q_f16) {
        // rows converted to f16 before the launch: copied as they are
        for (int c = gq; c < QCH; c += GA_THREADS) {
          const int h = c / 72, ch = c % 72;
          cp_async16(base + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7), qsrc + h * 1152 + ch * 16, 16);
        }
      } else {
        // every chunk copied at once (one memory latency per row), then converted bf16 -> f16 in
        // place by the thread that copied it; values that f16 cannot hold (|q| >= 65520 rounds to
        // infinity) are reported through the status word
        for (int c = gq; c < QCH; c += GA_THREADS) {
          const int h = c / 72, ch = c % 72;
          cp_async16(base + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7), qsrc + h * 1152 + ch * 16, 16);
        }
        cp_async_wait_all();
        bool out_of_range = false;
        for (int c = gq; c < QCH; c += GA_THREADS) {
          const int h = c / 72, ch = c % 72;
          uint4* chunk = reinterpret_cast<uint4*>(smem + OFF_Q + (ch >> 3) * SUB_Q + sw128_off(h, ch & 7));
          const uint4 raw = *chunk;
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
            out_of_range |= fmaxf(fabsf(lo), fabsf(hi)) >= 65520.f;
            o[i] = pack_pair(lo, hi, true);
          }
          *chunk = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (out_of_range) atomicOr(p.status, DEVERR_RANGE);
      }
      if (!PAGED || p.q_f16) {
        cp_async_arrive_noinc(bar(B_QFULL));
      } else {
        fence_async_smem();
        mbar_arrive(bar(B_QFULL));
      }
      const int g = SM_GATHER ? threadIdx.x : gq;
      for (int32_t t = 0; t < it.n_tiles && ok; ++t, ++gtile) ok = issue(prepare(it, t, g), gtile);
    }
  } else if (warp == MMA_WARP) {
    // ================================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t FMT = PAGED ? 0u : 1u;  // f16 operands for the FP8 cache, else bf16
      constexpr uint32_t ID_S = make_idesc(FMT, FMT, 0, 0, 128, 64);
      constexpr uint32_t ID_PV = make_idesc(FMT, FMT, 1, 1, 128, 64);
      uint32_t gtile = 0;
      bool ok = true;
      WorkIter wk = work_begin<SK>(p);
      Item it;
      for (int32_t it_n = 0; ok && work_next<SK>(p, wk, it); ++it_n) {
        if (!mbar_wait(bar(B_QFULL), it_n & 1, abort_flag, p.status, p.wait_ns)) break;
        // cp.async (generic proxy) writes -> tcgen05.mma (async proxy) reads.  Rows converted in
        // the kernel were fenced by the threads that stored them, before they arrived.
        if (!PAGED || p.q_f16) fence_async_smem();
        tc_fence_after();
        if (it.n_tiles == 0) mma_commit(bar(B_QEMPTY));
        for (int32_t t = 0; t < it.n_tiles && ok; ++t, ++gtile) {
          const uint32_t par = gtile & 1;
          const uint32_t ds = tmem + TM_S + 64u * par;
          for (int d = 0; d < NSUB; ++d) {
            if (!mbar_wait(bar(B_FULL + d), par, abort_flag, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            if (!PAGED) fence_async_smem();  // as after the query barrier
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t a = make_sdesc(base + OFF_KV + d * SUB_KV + kk * 32, 16, 1024);
              const uint64_t b = make_sdesc(base + OFF_Q + d * SUB_Q + kk * 32, 16, 1024);
              mma_f16(ds, a, b, ID_S, (d | kk) != 0);
            }
          }
          if (!ok) break;
          mma_commit(bar(B_SFULL));
          if (t == it.n_tiles - 1) mma_commit(bar(B_QEMPTY));
          if (!mbar_wait(bar(B_PFULL), par, abort_flag, p.status, p.wait_ns)) break;
          tc_fence_after();
#pragma unroll 1
          for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = make_sdesc(base + OFF_KV + 2 * mb * SUB_KV + kk * 2048, SUB_KV, 1024);
              const uint64_t b = make_sdesc(base + OFF_P + kk * 2048, SUB_KV, 1024);
              mma_f16(tmem + 64u * mb, a, b, ID_PV, (t > 0 || kk > 0));
            }
            mma_commit(bar(B_EMPTY + mb));
          }
          mma_commit(bar(B_PVDONE));
        }
      }
    }
  } else {
    // ================================================================= softmax / output warps
    const int quad = warp & 3, hh = warp >> 2;
    const int key = quad * 32 + lane;                 // TMEM lane: key of S^T, dim of an O^T block
    const int st = warp * 32 + lane;                  // 0..SM_THREADS-1
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t hcol = static_cast<uint32_t>(HPW) * hh;
    const bool head_lane = lane < HPW;                // lanes that own one of the warp's heads
    uint32_t gtile = 0;
    bool ok = true;
    WorkIter wk = work_begin<SK>(p);
    Item it;
    // A failed (timed-out) wait is recorded in `fail` and acted on at the next named_bar_or, where
    // all softmax threads see the same OR and leave together: none is then left waiting at a
    // later barrier for one that has gone.  Before a warp-collective TMEM access the lanes of a
    // warp agree on `fail` first (__any_sync).  A failed wait always comes with the CTA's abort
    // flag set, so the waits that follow it return at once.
    while (ok && work_next<SK>(p, wk, it)) {
      const int32_t seq_len = PAGED ? p.seq_lens[it.irow] : 0;
      const int32_t* idx_row = p.idx + static_cast<int64_t>(it.irow) * p.k;
      if (quad == 0 && head_lane) m_run[hcol + lane] = -INFINITY;
      named_bar(1, SM_THREADS);
      bool fail = false;
      if (SM_GATHER && it.n_tiles > 0) fail = !issue(prepare(it, 0, threadIdx.x), gtile);
      float lsum[HPW];
#pragma unroll
      for (int h = 0; h < HPW; ++h) lsum[h] = 0.f;
      for (int32_t t = 0; t < it.n_tiles; ++t, ++gtile) {
        const uint32_t par = gtile & 1;
        const int32_t jj = (it.j0 + t) * TILE + key;
        const int32_t v = jj < p.k ? idx_row[jj] : -1;
        const int64_t prow = kv_row<PAGED>(p, it.irow, v, seq_len);
        const bool valid = prow >= 0;
        Plan next_plan;  // indices of the next tile, loaded while this tile's softmax runs
        if (SM_GATHER && t + 1 < it.n_tiles) next_plan = prepare(it, t + 1, threadIdx.x);
        const float kscale = PAGED ? (valid ? p.kv_scale[prow] : 0.f) : 1.f;
        {
          const bool got = mbar_wait(bar(B_SFULL), par, abort_flag, p.status, p.wait_ns);
          fail = __any_sync(0xffffffffu, fail || !got);   // warp-uniform: the TMEM load is collective
        }
        tc_fence_after();
        float z[HPW];
        if (!fail) {
          uint32_t x[HPW];
          tmem_ld_heads<HPW>(tmem + TM_S + 64u * par + hcol + lane_off, x);
          const float zs = p.scale_log2 * kscale;
#pragma unroll
          for (int h = 0; h < HPW; ++h) z[h] = valid ? __uint_as_float(x[h]) * zs : -INFINITY;
        } else {
#pragma unroll
          for (int h = 0; h < HPW; ++h) z[h] = -INFINITY;
        }
        // Lazy running max: the cross-lane reduction is needed only when some logit exceeds
        // its head's running max by more than 8 (log2 units) -- always on an item's first tile.
        volatile int* need = need_flags + (gtile & 1);
        bool exceed = false;
#pragma unroll
        for (int c = 0; c < HPW / 4; ++c) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_run + hcol + 4 * c);
          exceed |= (z[4 * c] > m4.x + 8.f) | (z[4 * c + 1] > m4.y + 8.f) | (z[4 * c + 2] > m4.z + 8.f) |
                    (z[4 * c + 3] > m4.w + 8.f);
        }
        if (__any_sync(0xffffffffu, exceed) && lane == 0) *need = 1;
        if (named_bar_or(1, SM_THREADS, fail)) {
          ok = false;
          break;
        }
        if (st == 0) need_flags[(gtile + 1) & 1] = 0;  // the next tile's flag: its readers are done
        const bool resc = *need != 0;
        if (resc) {
          const float wmax = warp_reduce_heads<true, HPW>(z, lane);
          if (reduce_lane_writes<HPW>(lane)) red[quad * 64 + hcol + reduce_head_of_lane<HPW>(lane)] = wmax;
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
          for (int c = 0; c < HPW / 4; ++c) {
            const float4 a4 = *reinterpret_cast<const float4*>(alpha + hcol + 4 * c);
            lsum[4 * c] *= a4.x;
            lsum[4 * c + 1] *= a4.y;
            lsum[4 * c + 2] *= a4.z;
            lsum[4 * c + 3] *= a4.w;
          }
        }
        // probabilities 8 heads at a time -> one 16-byte chunk of this key's P^T row
#pragma unroll
        for (int c = 0; c < HPW / 8; ++c) {
          float m8[8];
          const float4 ma = *reinterpret_cast<const float4*>(m_run + hcol + 8 * c);
          const float4 mb = *reinterpret_cast<const float4*>(m_run + hcol + 8 * c + 4);
          m8[0] = ma.x, m8[1] = ma.y, m8[2] = ma.z, m8[3] = ma.w;
          m8[4] = mb.x, m8[5] = mb.y, m8[6] = mb.z, m8[7] = mb.w;
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = 8 * c + 2 * e;
            // z = -inf for masked keys, so the probability is exactly 0
            const float p0 = ex2_approx(z[h] - (m8[2 * e] == -INFINITY ? 0.f : m8[2 * e]));
            const float p1 = ex2_approx(z[h + 1] - (m8[2 * e + 1] == -INFINITY ? 0.f : m8[2 * e + 1]));
            lsum[h] += p0;
            lsum[h + 1] += p1;
            pk[e] = pack_pair(p0 * kscale, p1 * kscale, PAGED);
          }
          *reinterpret_cast<uint4*>(smem + OFF_P + sw128_off(key, (HPW / 8) * hh + c)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (resc && t > 0) {
          // O^T (dims on lanes, heads on columns) *= alpha; PV of the previous tile is done
          const bool got = mbar_wait(bar(B_PVDONE), par ^ 1, abort_flag, p.status, p.wait_ns);
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
        mbar_arrive(bar(B_PFULL));
        if (SM_GATHER && t + 1 < it.n_tiles && !fail) fail = !issue(next_plan, gtile + 1);
      }
      if (!ok) break;
      // ---- end of item: wait for the last PV, reduce row sums, write the output
      if (it.n_tiles > 0) {
        const bool got = mbar_wait(bar(B_PVDONE), (gtile - 1) & 1, abort_flag, p.status, p.wait_ns);
        fail = __any_sync(0xffffffffu, fail || !got);
        tc_fence_after();
      }
      {
        const float wsum = warp_reduce_heads<false, HPW>(lsum, lane);
        if (reduce_lane_writes<HPW>(lane)) red[quad * 64 + hcol + reduce_head_of_lane<HPW>(lane)] = wsum;
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
          if (it.n_tiles > 0) {
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
            orow[h * 512 + mb * 128 + key] = *reinterpret_cast<const uint16_t*>(&ob);
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
          if (it.n_tiles > 0) {
            tmem_ld_heads<HPW>(tmem + 64u * mb + hcol + lane_off, x);
          } else {
#pragma unroll
            for (int c = 0; c < HPW; ++c) x[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < HPW; ++c) po[(hcol + c) * 512 + mb * 128 + key] = __uint_as_float(x[c]);
        }
        if (quad == 0 && head_lane) {
          const int h = hcol + lane;
          p.part_ml[pr * 128 + h] = m_run[h];
          p.part_ml[pr * 128 + 64 + h] = l_tot[h];
        }
      }
      tc_fence_before();
      named_bar(1, SM_THREADS);  // m_run / l_tot / red are reused by the next item
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) tmem_dealloc(tmem, TMEM_COLS);
}

// The FP8 path multiplies in f16 (exact for e4m3 keys and values).  When a call cuts every query
// row over many CTAs, each of them would convert the same row from bf16 to f16, so the rows of
// all of a group's layers are converted here once, in one launch (blockIdx.y = layer), into the
// group's workspace.  8 values per thread and step.  A value that f16 cannot hold (|q| >= 65520
// rounds to infinity) sets DEVERR_RANGE, as the conversion inside the attention kernel does.
struct QConvert {
  const uint4* src[4];
  uint4* dst[4];
};
__global__ void __launch_bounds__(256) q_to_f16_kernel(const __grid_constant__ QConvert qc, int64_t n_chunks, int* status) {
  grid_dependency_sync();
  const uint4* __restrict__ q = qc.src[blockIdx.y];
  uint4* __restrict__ q16 = qc.dst[blockIdx.y];
  bool out_of_range = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n_chunks;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    const uint4 raw = q[i];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      out_of_range |= fmaxf(fabsf(lo), fabsf(hi)) >= 65520.f;
      o[j] = pack_pair(lo, hi, true);
    }
    q16[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (out_of_range) atomicOr(status, DEVERR_RANGE);
}

// Combine split-KV partials: one CTA of 128 threads per (row, head), 4 dims per thread.  Equal
// splits: n_split slots per row.  Stream-K (grid > 0): the row's fragments came from CTAs
// sk_owner(first tile) .. sk_owner(last tile); a row inside one CTA was written directly.  A row
// has at most MAX_SLOTS fragments (one per 128-key tile of k <= 2048); their weights are formed
// once in shared memory by one warp.  The memory latencies, not the arithmetic, set the time of
// this short kernel, so the first EARLY slots' partial rows are loaded before the weights, together
// with the row sums and maxima, and any further slots in batches of EARLY with their loads first.
constexpr int MAX_SLOTS = 16;
// EARLY = 4 keeps the registers low (38) for a grid of many waves; EARLY = MAX_SLOTS (80 registers,
// every slot at once) suits a grid of few rows cut into many slots, which fits in one wave.
template <int EARLY>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int32_t n_split,
                                                      uint16_t* __restrict__ out, float* __restrict__ lse,
                                                      int32_t tiles_per_row, int64_t sk_tiles, int32_t sk_grid) {
  grid_dependency_sync();
  __shared__ float wgt_s[MAX_SLOTS];
  __shared__ float tot_s[2];  // max (log2 units), sum of weighted row sums
  const int32_t row = blockIdx.x, h = blockIdx.y, t = threadIdx.x;
  int32_t n_slots = n_split;
  if (sk_grid > 0) {
    const int64_t g0 = static_cast<int64_t>(row) * tiles_per_row;
    n_slots = static_cast<int32_t>(sk_owner(g0 + tiles_per_row - 1, sk_tiles, sk_grid) -
                                   sk_owner(g0, sk_tiles, sk_grid) + 1);
    if (n_slots == 1) return;
  }
  n_slots = min(n_slots, MAX_SLOTS);
  const int64_t pr0 = static_cast<int64_t>(row) * n_split;
  auto load_o = [&](int s) {
    return *reinterpret_cast<const float4*>(part_o + ((pr0 + s) * 64 + h) * 512 + 4 * t);
  };
  // the first slots' partial rows in flight before their weights are known, with the row sums and
  // maxima: one memory latency instead of three in a chain (row sum, max, then the rows)
  float4 o[EARLY];
#pragma unroll
  for (int s = 0; s < EARLY; ++s) o[s] = s < n_slots ? load_o(s) : make_float4(0.f, 0.f, 0.f, 0.f);
  if (t < 32) {
    const int64_t pr = pr0 + t;
    const float l_raw = t < n_slots ? part_ml[pr * 128 + 64 + h] : 0.f;
    const float m_raw = t < n_slots ? part_ml[pr * 128 + h] : -INFINITY;
    const bool live = l_raw > 0.f;
    const float m = live ? m_raw : -INFINITY;
    const float l = live ? l_raw : 0.f;
    float M = m;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w = live ? exp2f(m - M) : 0.f;
    float L = w * l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (t < MAX_SLOTS) wgt_s[t] = w;
    if (t == 0) {
      tot_s[0] = M;
      tot_s[1] = L;
    }
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // a slot without keys (weight 0) holds no written row: it never enters acc
  auto add = [&](float w, const float4& v) {
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  };
#pragma unroll
  for (int s = 0; s < EARLY; ++s)
    if (s < n_slots && wgt_s[s] > 0.f) add(wgt_s[s], o[s]);
  // rows cut into more slots (few rows over many CTAs): the rest in batches of EARLY, loads first
  for (int s0 = EARLY; s0 < n_slots; s0 += EARLY) {
#pragma unroll
    for (int u = 0; u < EARLY; ++u)
      o[u] = s0 + u < n_slots && wgt_s[s0 + u] > 0.f ? load_o(s0 + u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < EARLY; ++u)
      if (s0 + u < n_slots && wgt_s[s0 + u] > 0.f) add(wgt_s[s0 + u], o[u]);
  }
  const float M = tot_s[0], L = tot_s[1];
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

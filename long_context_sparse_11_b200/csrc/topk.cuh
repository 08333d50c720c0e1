// Step a4: exact per-row Top-k by radix selection on CUDA cores.
//
// Each candidate s of a row gets the 64-bit composite key  (f32_key(score) << 32) | ~s,
// so "larger composite" means "larger score, then lower position"; composites are unique
// and the Top-k set is the k largest composites.  Selection walks six digits of the
// composite (12, 12, 8 bits of the score key, then 12, 12, 8 bits of ~s).  At each digit
// a histogram over the elements still matching the chosen prefix gives the bin T that
// contains the k_rem-th largest; elements above T are emitted, the prefix is extended by
// T, and the walk stops as soon as the elements matching the prefix are exactly k_rem.
//
// Row mode (one CTA per row): the row is read twice from global memory (histogram of the
// first digit, then emit / collect the threshold bin into shared memory); later digits
// run on the shared-memory candidates.  Segmented mode (few long rows): several CTAs per
// row build the first-digit histogram (or the paged indexer builds it in its epilogue), then
// several CTAs per row emit / collect in parallel through a global workspace, and the last of
// them to finish resolves the remaining digits.
#pragma once
#include "ptx.cuh"

namespace dsa {
namespace topk {

constexpr int THREADS = 1024;
constexpr int BINS = 4096;
constexpr int CAND_CAP = 6144;  // shared-memory candidates of the threshold bin
constexpr int SEG_THREADS = 512;

struct Smem {
  uint32_t hist[BINS];
  uint32_t cand_key[CAND_CAP];
  int32_t cand_idx[CAND_CAP];
  uint32_t warp_sum[32];
  int32_t out_cnt;
  int32_t cand_cnt;
  uint32_t sel_bin;
  uint32_t sel_above;
  uint32_t sel_eq;
};

__device__ __forceinline__ uint64_t composite(uint32_t key, int32_t idx) {
  return (static_cast<uint64_t>(key) << 32) | static_cast<uint64_t>(~static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int digit_shift(int lvl) {
  // levels: bits [52,64), [40,52), [32,40), [20,32), [8,20), [0,8)
  const int sh[6] = {52, 40, 32, 20, 8, 0};
  return sh[lvl];
}
__device__ __forceinline__ int digit_bits(int lvl) { return (lvl == 2 || lvl == 5) ? 8 : 12; }

// Block-wide: find bin T with above(T) < k_rem <= above(T) + hist[T], above(T) = sum of
// bins > T.  Writes sel_bin / sel_above / sel_eq.  All threads of the block must call.
template <int NT>
__device__ void find_threshold(const uint32_t* hist, uint32_t k_rem, uint32_t* warp_sum, uint32_t* sel_bin,
                               uint32_t* sel_above, uint32_t* sel_eq) {
  constexpr int PER = BINS / NT;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  uint32_t v = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) v += hist[t * PER + i];
  uint32_t incl = v;  // sum over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
    if (lane + off < 32) incl += y;
  }
  if (lane == 0) warp_sum[w] = incl;
  __syncthreads();
  uint32_t above_warp = 0;
  for (int u = w + 1; u < NT / 32; ++u) above_warp += warp_sum[u];
  const uint32_t excl = incl - v + above_warp;  // sum of bins owned by higher threads
  if (excl < k_rem && k_rem <= excl + v) {
    uint32_t acc = excl;
    for (int i = PER - 1; i >= 0; --i) {
      const uint32_t h = hist[t * PER + i];
      if (acc + h >= k_rem) {
        *sel_bin = t * PER + i;
        *sel_above = acc;
        *sel_eq = h;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
}

// Element sources for the digit walk.
struct RowSrc {
  const float* p;
  int32_t n;
  __device__ __forceinline__ int32_t size() const { return n; }
  __device__ __forceinline__ uint64_t comp(int32_t i) const { return composite(f32_key(p[i]), i); }
  __device__ __forceinline__ int32_t index(int32_t i) const { return i; }
};
struct CandSrc {
  const uint32_t* keys;
  const int32_t* idx;
  int32_t n;
  __device__ __forceinline__ int32_t size() const { return n; }
  __device__ __forceinline__ uint64_t comp(int32_t i) const { return composite(keys[i], idx[i]); }
  __device__ __forceinline__ int32_t index(int32_t i) const { return idx[i]; }
};

struct CandSrcL2 {  // candidates written by other CTAs of the grid: read at L2, past this SM's L1
  const uint32_t* keys;
  const int32_t* idx;
  int32_t n;
  __device__ __forceinline__ int32_t size() const { return n; }
  __device__ __forceinline__ uint64_t comp(int32_t i) const { return composite(__ldcg(keys + i), __ldcg(idx + i)); }
  __device__ __forceinline__ int32_t index(int32_t i) const { return __ldcg(idx + i); }
};

// Walk digits lvl0..5 over `src`, emitting into out[0..k) through the shared counter.
template <int NT, class Src, class S>
__device__ void walk_digits(const Src& src, int lvl0, uint64_t pfx, uint64_t pmask, uint32_t k_rem, S& sm,
                            int32_t* out, int32_t kmax) {
  const int t = threadIdx.x;
  for (int lvl = lvl0; lvl < 6 && k_rem > 0; ++lvl) {
    const int sh = digit_shift(lvl);
    const uint32_t dmask = (1u << digit_bits(lvl)) - 1u;
    for (int b = t; b < BINS; b += NT) sm.hist[b] = 0;
    __syncthreads();
    const int32_t n = src.size();
    for (int32_t i = t; i < n; i += NT) {
      const uint64_t c = src.comp(i);
      if ((c & pmask) == pfx) atomicAdd(&sm.hist[(c >> sh) & dmask], 1u);
    }
    __syncthreads();
    find_threshold<NT>(sm.hist, k_rem, sm.warp_sum, &sm.sel_bin, &sm.sel_above, &sm.sel_eq);
    const uint32_t T = sm.sel_bin, above = sm.sel_above, eq = sm.sel_eq;
    const uint64_t new_pfx = pfx | (static_cast<uint64_t>(T) << sh);
    const uint64_t new_mask = pmask | (static_cast<uint64_t>(dmask) << sh);
    const bool take_eq = (eq == k_rem - above);
    for (int32_t i = t; i < n; i += NT) {
      const uint64_t c = src.comp(i);
      if ((c & pmask) != pfx) continue;
      const uint32_t d = static_cast<uint32_t>((c >> sh) & dmask);
      if (d > T || (take_eq && d == T)) {
        const int32_t pos = atomicAdd(&sm.out_cnt, 1);
        if (pos < kmax) out[pos] = src.index(i);
      }
    }
    __syncthreads();
    if (take_eq) break;
    k_rem -= above;
    pfx = new_pfx;
    pmask = new_mask;
  }
}

// Candidates of row r: row_len[r] (device array) or causal_len0 + r, capped at `cap`.
__device__ __forceinline__ int32_t row_length(int32_t r, const int32_t* row_len, int64_t causal_len0, int64_t cap) {
  int64_t n = row_len ? static_cast<int64_t>(row_len[r]) : causal_len0 + r;
  n = n < 0 ? 0 : n;
  return static_cast<int32_t>(n > cap ? cap : n);
}

// ------------------------------------------------------------------------------- row mode

__global__ void __launch_bounds__(THREADS) topk_row_kernel(const float* __restrict__ scores, int64_t ld,
                                                           int32_t n_rows, const int32_t* __restrict__ row_len,
                                                           int64_t causal_len0, int64_t cap, int32_t k,
                                                           int32_t* __restrict__ idx_out) {
  grid_dependency_sync();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int32_t r = blockIdx.x;
  if (r >= n_rows) return;
  const int t = threadIdx.x;
  const float* row = scores + static_cast<int64_t>(r) * ld;
  int32_t* out = idx_out + static_cast<int64_t>(r) * k;
  const int32_t n = row_length(r, row_len, causal_len0, cap);
  if (t == 0) {
    sm.out_cnt = 0;
    sm.cand_cnt = 0;
  }
  if (n <= k) {
    for (int32_t i = t; i < k; i += THREADS) out[i] = i < n ? i : -1;
    return;
  }
  for (int b = t; b < BINS; b += THREADS) sm.hist[b] = 0;
  __syncthreads();
  // pass 1: histogram of the top 12 key bits (vectorised, row start is 16-byte aligned)
  const int32_t n4 = n & ~3;
  for (int32_t i = t * 4; i < n4; i += THREADS * 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
    atomicAdd(&sm.hist[f32_key(v.x) >> 20], 1u);
    atomicAdd(&sm.hist[f32_key(v.y) >> 20], 1u);
    atomicAdd(&sm.hist[f32_key(v.z) >> 20], 1u);
    atomicAdd(&sm.hist[f32_key(v.w) >> 20], 1u);
  }
  for (int32_t i = n4 + t; i < n; i += THREADS) atomicAdd(&sm.hist[f32_key(row[i]) >> 20], 1u);
  __syncthreads();
  find_threshold<THREADS>(sm.hist, static_cast<uint32_t>(k), sm.warp_sum, &sm.sel_bin, &sm.sel_above, &sm.sel_eq);
  const uint32_t T = sm.sel_bin, above = sm.sel_above, eq = sm.sel_eq;
  const uint32_t k_rem = static_cast<uint32_t>(k) - above;
  const bool take_eq = (eq == k_rem);
  const bool collect = !take_eq && eq <= static_cast<uint32_t>(CAND_CAP);
  // pass 2: emit bins above T, collect bin T
  auto visit = [&](float f, int32_t i) {
    const uint32_t key = f32_key(f);
    const uint32_t d = key >> 20;
    if (d > T || (take_eq && d == T)) {
      const int32_t pos = atomicAdd(&sm.out_cnt, 1);
      if (pos < k) out[pos] = i;
    } else if (collect && d == T) {
      const int32_t c = atomicAdd(&sm.cand_cnt, 1);
      if (c < CAND_CAP) {
        sm.cand_key[c] = key;
        sm.cand_idx[c] = i;
      }
    }
  };
  for (int32_t i = t * 4; i < n4; i += THREADS * 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
    visit(v.x, i);
    visit(v.y, i + 1);
    visit(v.z, i + 2);
    visit(v.w, i + 3);
  }
  for (int32_t i = n4 + t; i < n; i += THREADS) visit(row[i], i);
  __syncthreads();
  if (take_eq) return;
  const uint64_t pfx = static_cast<uint64_t>(T) << 52;
  const uint64_t pmask = static_cast<uint64_t>(0xFFF) << 52;
  if (collect) {
    CandSrc src{sm.cand_key, sm.cand_idx, min(sm.cand_cnt, CAND_CAP)};
    walk_digits<THREADS>(src, 1, pfx, pmask, k_rem, sm, out, k);
  } else {
    RowSrc src{row, n};
    walk_digits<THREADS>(src, 1, pfx, pmask, k_rem, sm, out, k);
  }
}

// --------------------------------------------------------------------------- segmented mode
// Workspace per row: hist[4096] u32, counters[4] i32 (out, cand), then cand keys/idx [gcap].

struct SegWs {
  uint32_t* hist;     // [rows][BINS]
  int32_t* counters;  // [rows][4]
  uint32_t* cand_key; // [rows][gcap]
  int32_t* cand_idx;  // [rows][gcap]
  int32_t gcap;
};

__global__ void __launch_bounds__(SEG_THREADS) topk_seg_hist_kernel(const float* __restrict__ scores, int64_t ld,
                                                                    const int32_t* __restrict__ row_len,
                                                                    int64_t causal_len0, int64_t cap, int32_t k,
                                                                    int32_t seg_len, SegWs ws) {
  grid_dependency_sync();
  __shared__ uint32_t hist[BINS];
  const int32_t r = blockIdx.y;
  const int32_t n = row_length(r, row_len, causal_len0, cap);
  if (n <= k) return;
  const int32_t beg = blockIdx.x * seg_len;
  if (beg >= n) return;
  const int32_t end = min(n, beg + seg_len);
  const int t = threadIdx.x;
  for (int b = t; b < BINS; b += SEG_THREADS) hist[b] = 0;
  __syncthreads();
  const float* row = scores + static_cast<int64_t>(r) * ld;
  for (int32_t i = beg + t * 4; i + 3 < end; i += SEG_THREADS * 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(row + i));
    atomicAdd(&hist[f32_key(v.x) >> 20], 1u);
    atomicAdd(&hist[f32_key(v.y) >> 20], 1u);
    atomicAdd(&hist[f32_key(v.z) >> 20], 1u);
    atomicAdd(&hist[f32_key(v.w) >> 20], 1u);
  }
  const int32_t tail = beg + ((end - beg) & ~3);
  for (int32_t i = tail + t; i < end; i += SEG_THREADS) atomicAdd(&hist[f32_key(row[i]) >> 20], 1u);
  __syncthreads();
  uint32_t* g = ws.hist + static_cast<int64_t>(r) * BINS;
  for (int b = t; b < BINS; b += SEG_THREADS)
    if (hist[b]) atomicAdd(&g[b], hist[b]);
}

// Filter and resolve in one launch.  Every CTA of a row emits the elements above the threshold
// bin of the row's first-digit histogram and collects the threshold bin's elements into the row's
// global candidate list; the last CTA of the row to finish (counted on counters[2], after a
// device-scope fence of each CTA's writes) then resolves the remaining digits over those candidates.
struct FilterSmem {
  static constexpr int SEL_BUF = 2048, CAND_BUF = 1024;
  uint32_t hist[BINS];
  uint32_t warp_sum[32];
  int32_t out_cnt;
  uint32_t sel_bin, sel_above, sel_eq;
  int32_t s_sel[SEL_BUF];
  uint32_t s_ckey[CAND_BUF];
  int32_t s_cidx[CAND_BUF];
  int32_t s_cnt[2], s_base[2];
  int32_t last;
};

__global__ void __launch_bounds__(SEG_THREADS) topk_seg_filter_kernel(const float* __restrict__ scores, int64_t ld,
                                                                      const int32_t* __restrict__ row_len,
                                                                      int64_t causal_len0, int64_t cap, int32_t k,
                                                                      int32_t seg_len, SegWs ws,
                                                                      int32_t* __restrict__ idx_out) {
  grid_dependency_sync();
  // The segment's selections and threshold-bin candidates are gathered in shared memory and
  // placed in the row's arrays with one global reservation each per CTA: a per-element atomic
  // on the row's counter serialises about k same-address atomics per row.
  __shared__ FilterSmem sm;
  constexpr int SEL_BUF = FilterSmem::SEL_BUF, CAND_BUF = FilterSmem::CAND_BUF;
  const int32_t r = blockIdx.y;
  const int t = threadIdx.x;
  const int32_t n = row_length(r, row_len, causal_len0, cap);
  int32_t* out = idx_out + static_cast<int64_t>(r) * k;
  if (n <= k) {  // every candidate is selected, the rest is padding
    if (blockIdx.x == 0)
      for (int32_t i = t; i < k; i += SEG_THREADS) out[i] = i < n ? i : -1;
    return;
  }
  const int32_t beg = blockIdx.x * seg_len;
  if (beg >= n) return;
  const int32_t n_segs = (n + seg_len - 1) / seg_len;  // CTAs of this row that reach the end
  const int32_t end = min(n, beg + seg_len);
  const uint32_t* g = ws.hist + static_cast<int64_t>(r) * BINS;
  for (int b = t; b < BINS; b += SEG_THREADS) sm.hist[b] = g[b];
  if (t == 0) sm.s_cnt[0] = sm.s_cnt[1] = 0;
  __syncthreads();
  find_threshold<SEG_THREADS>(sm.hist, static_cast<uint32_t>(k), sm.warp_sum, &sm.sel_bin, &sm.sel_above,
                              &sm.sel_eq);
  const uint32_t T = sm.sel_bin, above = sm.sel_above, eq = sm.sel_eq;
  const bool take_eq = (eq == static_cast<uint32_t>(k) - above);
  const bool collect = !take_eq && eq <= static_cast<uint32_t>(ws.gcap);
  const float* row = scores + static_cast<int64_t>(r) * ld;
  int32_t* cnt = ws.counters + static_cast<int64_t>(r) * 4;
  uint32_t* ck = ws.cand_key + static_cast<int64_t>(r) * ws.gcap;
  int32_t* ci = ws.cand_idx + static_cast<int64_t>(r) * ws.gcap;
  auto visit = [&](float f, int32_t i) {
    const uint32_t key = f32_key(f);
    const uint32_t d = key >> 20;
    if (d > T || (take_eq && d == T)) {
      const int32_t p = atomicAdd(&sm.s_cnt[0], 1);
      if (p < SEL_BUF) {
        sm.s_sel[p] = i;
      } else {  // overflow (a segment holding more than SEL_BUF selections): place directly
        const int32_t pos = atomicAdd(&cnt[0], 1);
        if (pos < k) out[pos] = i;
      }
    } else if (collect && d == T) {
      const int32_t p = atomicAdd(&sm.s_cnt[1], 1);
      if (p < CAND_BUF) {
        sm.s_ckey[p] = key;
        sm.s_cidx[p] = i;
      } else {
        const int32_t c = atomicAdd(&cnt[1], 1);
        if (c < ws.gcap) {
          ck[c] = key;
          ci[c] = i;
        }
      }
    }
  };
  // 16-byte loads, two in flight per thread (segments start at multiples of 4 and rows are
  // 16-byte aligned), then the unaligned tail one by one
  const int32_t end4 = beg + ((end - beg) & ~3);
  int32_t i = beg + t * 4;
  for (; i + SEG_THREADS * 4 < end4; i += SEG_THREADS * 8) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + i));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + i + SEG_THREADS * 4));
    visit(a.x, i);
    visit(a.y, i + 1);
    visit(a.z, i + 2);
    visit(a.w, i + 3);
    const int32_t j = i + SEG_THREADS * 4;
    visit(b.x, j);
    visit(b.y, j + 1);
    visit(b.z, j + 2);
    visit(b.w, j + 3);
  }
  if (i < end4) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + i));
    visit(a.x, i);
    visit(a.y, i + 1);
    visit(a.z, i + 2);
    visit(a.w, i + 3);
  }
  for (int32_t u = end4 + t; u < end; u += SEG_THREADS) visit(row[u], u);
  __syncthreads();
  const int32_t n_sel = min(sm.s_cnt[0], SEL_BUF), n_cand = min(sm.s_cnt[1], CAND_BUF);
  if (t == 0) {
    sm.s_base[0] = n_sel > 0 ? atomicAdd(&cnt[0], n_sel) : 0;
    sm.s_base[1] = n_cand > 0 ? atomicAdd(&cnt[1], n_cand) : 0;
  }
  __syncthreads();
  for (int32_t j = t; j < n_sel; j += SEG_THREADS) {
    const int32_t pos = sm.s_base[0] + j;
    if (pos < k) out[pos] = sm.s_sel[j];
  }
  for (int32_t j = t; j < n_cand; j += SEG_THREADS) {
    const int32_t c = sm.s_base[1] + j;
    if (c < ws.gcap) {
      ck[c] = sm.s_ckey[j];
      ci[c] = sm.s_cidx[j];
    }
  }
  // ---- the row's last CTA resolves the threshold bin
  __threadfence();
  __syncthreads();
  if (t == 0) sm.last = atomicAdd(&cnt[2], 1) == n_segs - 1;
  __syncthreads();
  if (!sm.last || take_eq) return;  // take_eq: the filter emitted the whole Top-k
  __threadfence();
  const uint32_t k_rem = static_cast<uint32_t>(k) - above;
  if (t == 0) sm.out_cnt = static_cast<int32_t>(above);
  const uint64_t pfx = static_cast<uint64_t>(T) << 52;
  const uint64_t pmask = static_cast<uint64_t>(0xFFF) << 52;
  __syncthreads();
  if (collect) {
    CandSrcL2 src{ck, ci, min(__ldcg(&cnt[1]), ws.gcap)};
    walk_digits<SEG_THREADS>(src, 1, pfx, pmask, k_rem, sm, out, k);
  } else {
    RowSrc src{row, n};
    walk_digits<SEG_THREADS>(src, 1, pfx, pmask, k_rem, sm, out, k);
  }
}

}  // namespace topk
}  // namespace dsa

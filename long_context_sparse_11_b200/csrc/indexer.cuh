// Steps a2 + a3: lightweight-indexer scores on the 5th-generation tensor cores.
//
//   I[r, s] = sk[s] * sum_h w'[r,h] * max(0, q[r,h,:] . k[s,:]),   w' = w * sq
//
// Layout of the contraction: the 128 keys of a tile are the M rows (one TMEM lane per
// key), and (query, head) pairs are the N columns: 8 queries x 32 heads = 256 columns in
// prefill, 1 query x 32 heads in decode.  The head sum is then a per-thread loop over 32
// consecutive TMEM columns, with no cross-lane traffic.  K = 128: 8 MMAs of K=16 (bf16)
// or 4 of K=32 (e4m3).
//
// Warp roles (one CTA per work unit = query block x chunk of key tiles):
//   warp 0      TMA producer: query tile once, then key tiles into a STAGES-deep ring
//   warp 1      TMEM owner and single-thread MMA issuer
//   warps 2..   epilogue: tcgen05.ld -> ReLU / weights / scale / causal mask -> scores
// Prefill runs two query groups (16 queries) per key tile so a key tile feeds 2 MMAs, each
// into its own 256-column accumulator; the epilogue of one overlaps the MMA of the other.
#pragma once
#include "ptx.cuh"

namespace dsa {
namespace idx {

constexpr int BLOCK_KEYS = 128;
constexpr int UNIT_TILES = 32;  // key tiles per work unit (default; decode may use fewer)

// ReLU split between two pipes.  max(x, 0) runs on the ALU pipe, the epilogue's busiest; for P
// of the 16 head pairs the epilogue instead forms x + |x| = 2 max(x, 0) with one
// add on the FMA pipe and the staged weight of those heads is halved, so w * max(x, 0) is
// reproduced exactly (0.5 w * 2x = w * x for every finite accumulator x).  The P pairs are
// spread evenly over the 16.
#ifndef DSA_IDX_RELU_FMA_PAIRS_BF16
#define DSA_IDX_RELU_FMA_PAIRS_BF16 8
#endif
#ifndef DSA_IDX_RELU_FMA_PAIRS_E4M3
#define DSA_IDX_RELU_FMA_PAIRS_E4M3 8
#endif
template <int P>
__host__ __device__ constexpr bool relu_on_fma(int pair) {
  return ((pair + 1) * P) / 16 != (pair * P) / 16;
}

template <bool FP8, bool PAGED>
struct Cfg {
  static constexpr int NQ = PAGED ? 1 : 8;        // queries per accumulator
  static constexpr int NGROUP = PAGED ? 1 : 2;    // accumulators fed by one key tile
  static constexpr int N = NQ * 32;
  static constexpr int NBUF = PAGED ? 4 : 2;      // TMEM accumulator ring
  static constexpr int TMEM_COLS = PAGED ? 128 : 512;
  static constexpr int KH = FP8 ? 1 : 2;          // 128-byte K halves per row
  static constexpr int KSTEPS = FP8 ? 4 : 8;
  // decode keeps 3 stages so that its 16 KB score histogram still leaves room for 3 CTAs per SM
  static constexpr int STAGES = PAGED ? 3 : (FP8 ? 4 : 2);
  static constexpr int EPI_WARPS = PAGED ? 4 : 16;
  static constexpr int RELU_FMA_PAIRS = FP8 ? DSA_IDX_RELU_FMA_PAIRS_E4M3 : DSA_IDX_RELU_FMA_PAIRS_BF16;
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int Q_HALF_BYTES = N * 128;    // one K half of one query group
  static constexpr int Q_BYTES = NGROUP * KH * Q_HALF_BYTES;
  static constexpr int KEY_HALF_BYTES = BLOCK_KEYS * 128;
  static constexpr int KEY_STAGE_BYTES = KH * KEY_HALF_BYTES;
  static constexpr int W_FLOATS = NGROUP * NQ * 32;
  static constexpr uint32_t IDESC = FP8 ? make_idesc(0, 0, 0, 0, 128, N) : make_idesc(1, 1, 0, 0, 128, N);
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_W = OFF_K + STAGES * KEY_STAGE_BYTES;
  static constexpr int HIST_BINS = 4096;  // decode: first-digit histogram of the scores for the Top-k
  static constexpr int OFF_HIST = OFF_W + W_FLOATS * 4;
  static constexpr int OFF_BAR = OFF_HIST + (PAGED ? HIST_BINS * 4 : 0);
  static constexpr int N_BARS = 2 * STAGES + 2 * NBUF + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
};

struct Params {
  const float* q_scale;     // [n_q,32] (e4m3) or null
  const float* w;           // [n_q,32]
  const float* key_scale;   // dense [n_tokens] / paged [n_pages*64] (e4m3) or null
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* scores;
  int64_t ld;
  int64_t n_tokens;
  int32_t n_q;
  int32_t q_pos0;
  int32_t max_pages;
  int32_t n_pages;
  int32_t unit_tiles;       // key tiles per CTA
  uint32_t* hist;           // paged only, or null: [n_q][4096] counts of f32_key(score) >> 20, added to
  int* status;
  uint64_t wait_ns;
};

template <bool FP8, bool PAGED>
__global__ void __launch_bounds__(Cfg<FP8, PAGED>::THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k, Params p) {
  grid_dependency_sync();
  using C = Cfg<FP8, PAGED>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  const uint32_t bar0 = base + C::OFF_BAR;
  auto key_full = [&](int s) { return bar0 + 8u * s; };
  auto key_empty = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto acc_full = [&](int b) { return bar0 + 8u * (2 * C::STAGES + b); };
  auto acc_empty = [&](int b) { return bar0 + 8u * (2 * C::STAGES + C::NBUF + b); };
  const uint32_t q_full = bar0 + 8u * (2 * C::STAGES + 2 * C::NBUF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: rows and key-tile range
  int32_t r0 = 0, b = 0, len = 0;
  if (PAGED) {
    b = blockIdx.y;
    len = p.seq_lens[b];
    len = len < 0 ? 0 : min(len, p.max_pages * 64);
  } else {
    r0 = blockIdx.y * (C::NQ * C::NGROUP);
    const int32_t rlast = min(r0 + C::NQ * C::NGROUP, p.n_q) - 1;
    const int64_t l = min(static_cast<int64_t>(p.q_pos0) + rlast + 1, p.n_tokens);
    len = static_cast<int32_t>(l);
  }
  const int32_t n_tiles = (len + BLOCK_KEYS - 1) / BLOCK_KEYS;
  const int32_t kt0 = blockIdx.x * p.unit_tiles;
  const int32_t kt1 = min(kt0 + p.unit_tiles, n_tiles);
  if (kt0 >= kt1) return;  // uniform across the CTA

  // group g needs tile kt iff some of its rows has a candidate in the tile
  auto group_needed = [&](int kt, int g) -> bool {
    if (PAGED) return true;
    const int32_t rg = r0 + g * C::NQ;
    if (rg >= p.n_q) return false;
    const int64_t maxpos = static_cast<int64_t>(p.q_pos0) + min(rg + C::NQ, p.n_q) - 1;
    return static_cast<int64_t>(kt) * BLOCK_KEYS <= maxpos;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(key_full(s), 1);
      mbar_init(key_empty(s), 1);
    }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), C::EPI_WARPS);
    }
    mbar_init(q_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  if (PAGED && p.hist)
    for (int i = threadIdx.x; i < C::HIST_BINS; i += C::THREADS) hist_s[i] = 0u;
  // per-(query, head) weights, folded with the query scale
  if (warp >= 2) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < C::W_FLOATS; i += C::EPI_WARPS * 32) {
      const int qq = i >> 5, h = i & 31;
      const int32_t row = PAGED ? b : r0 + qq;
      float v = 0.f;
      if (row < p.n_q) {
        v = p.w[static_cast<int64_t>(row) * 32 + h];
        if (FP8) v *= p.q_scale[static_cast<int64_t>(row) * 32 + h];
        if (relu_on_fma<C::RELU_FMA_PAIRS>(h >> 1)) v *= 0.5f;
      }
      w_s[i] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
      for (int g = 0; g < C::NGROUP; ++g)
        for (int kh = 0; kh < C::KH; ++kh) {
          const int y = PAGED ? b * 32 : (r0 + g * C::NQ) * 32;
          tma_load_2d(base + C::OFF_Q + (g * C::KH + kh) * C::Q_HALF_BYTES, &map_q, q_full, kh * 64, y);
        }
      for (int kt = kt0, i = 0; kt < kt1; ++kt, ++i) {
        const int s = i % C::STAGES;
        const uint32_t ph = (i / C::STAGES) & 1;
        if (!mbar_wait(key_empty(s), ph ^ 1, abort_flag, p.status, p.wait_ns)) break;
        const uint32_t dst = base + C::OFF_K + s * C::KEY_STAGE_BYTES;
        if (PAGED) {
          int32_t phys[2];
          uint32_t bytes = 0;
          for (int pg = 0; pg < 2; ++pg) {
            const int32_t lp = kt * 2 + pg;
            phys[pg] = -1;
            if (lp * 64 < len && lp < p.max_pages) {
              const int32_t v = p.block_table[static_cast<int64_t>(b) * p.max_pages + lp];
              if (v >= 0 && v < p.n_pages) {
                phys[pg] = v;
                bytes += 64 * 128;
              } else {
                atomicOr(p.status, DEVERR_BOUNDS);
              }
            }
          }
          if (bytes == 0) {  // nothing valid to load: release the stage without data
            mbar_arrive(key_full(s));
          } else {
            mbar_arrive_expect_tx(key_full(s), bytes);
            for (int pg = 0; pg < 2; ++pg)
              if (phys[pg] >= 0) tma_load_2d(dst + pg * 64 * 128, &map_k, key_full(s), 0, phys[pg] * 64);
          }
        } else {
          mbar_arrive_expect_tx(key_full(s), C::KEY_STAGE_BYTES);
          for (int kh = 0; kh < C::KH; ++kh)
            tma_load_2d(dst + kh * C::KEY_HALF_BYTES, &map_k, key_full(s), kh * 64, kt * BLOCK_KEYS);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (mbar_wait(q_full, 0, abort_flag, p.status, p.wait_ns)) {
        tc_fence_after();
        int job = 0;
        for (int kt = kt0, i = 0; kt < kt1; ++kt, ++i) {
          const int s = i % C::STAGES;
          if (!mbar_wait(key_full(s), (i / C::STAGES) & 1, abort_flag, p.status, p.wait_ns)) break;
          tc_fence_after();
          bool ok = true;
          for (int g = 0; g < C::NGROUP; ++g) {
            if (!group_needed(kt, g)) continue;
            const int bf = job % C::NBUF;
            if (!mbar_wait(acc_empty(bf), ((job / C::NBUF) & 1) ^ 1, abort_flag, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + bf * C::N;
            const uint32_t kbase = base + C::OFF_K + s * C::KEY_STAGE_BYTES;
            const uint32_t qbase = base + C::OFF_Q + g * C::KH * C::Q_HALF_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const int half = FP8 ? 0 : kk / 4;
              const uint32_t koff = (FP8 ? kk : kk % 4) * 32;
              const uint64_t a = make_sdesc(kbase + half * C::KEY_HALF_BYTES + koff, 16, 1024);
              const uint64_t bd = make_sdesc(qbase + half * C::Q_HALF_BYTES + koff, 16, 1024);
              if (FP8)
                mma_f8(d, a, bd, C::IDESC, kk > 0);
              else
                mma_f16(d, a, bd, C::IDESC, kk > 0);
            }
            mma_commit(acc_full(bf));
            ++job;
          }
          if (!ok) break;
          mma_commit(key_empty(s));
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int e = warp - 2;
    const int quad = warp & 3;
    const int part = e / 4;                      // prefill: which queries of the group
    constexpr int QPW = PAGED ? 1 : C::NQ / (C::EPI_WARPS / 4);  // queries per warp per accumulator
    const int key_in_tile = quad * 32 + lane;
    int job = 0;
    bool ok = true;
    for (int kt = kt0; kt < kt1 && ok; ++kt) {
      const int64_t s_abs = static_cast<int64_t>(kt) * BLOCK_KEYS + key_in_tile;
      float sk = 1.f;
      if (FP8 && s_abs < len) {
        if (PAGED) {
          const int32_t lp = static_cast<int32_t>(s_abs >> 6);
          const int32_t v = p.block_table[static_cast<int64_t>(b) * p.max_pages + lp];
          sk = (v >= 0 && v < p.n_pages) ? p.key_scale[static_cast<int64_t>(v) * 64 + (s_abs & 63)] : 0.f;
        } else {
          sk = p.key_scale[s_abs];
        }
      }
      for (int g = 0; g < C::NGROUP; ++g) {
        if (!group_needed(kt, g)) continue;
        const int bf = job % C::NBUF;
        // every lane must take the same branch: the TMEM loads below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(acc_full(bf), (job / C::NBUF) & 1, abort_flag, p.status,
                                               p.wait_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // head sum of one query from registers: ReLU, per-head weight, packed FMA on head pairs
        auto score = [&](const uint32_t (&x)[32], int qq) {
          const float4* wv = reinterpret_cast<const float4*>(w_s + (g * C::NQ + qq) * 32);
          // two independent chains of packed FMAs (heads 0-1, 4-5, ... and 2-3, 6-7, ...), so
          // that consecutive FMAs of one query do not wait on each other
          float2 a2 = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            const float4 ww = wv[h4];
            float r[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float v = __uint_as_float(x[4 * h4 + u]);
              r[u] = relu_on_fma<C::RELU_FMA_PAIRS>(2 * h4 + u / 2) ? v + fabsf(v) : fmaxf(v, 0.f);
            }
            // packed fp32 FMA on head pairs (the compiler's own pairing of the operands)
            a2 = __ffma2_rn(make_float2(ww.x, ww.y), make_float2(r[0], r[1]), a2);
            b2 = __ffma2_rn(make_float2(ww.z, ww.w), make_float2(r[2], r[3]), b2);
          }
          float acc = (a2.x + a2.y) + (b2.x + b2.y);
          if (FP8) acc *= sk;
          if (PAGED) {
            if (s_abs < len) {
              p.scores[static_cast<int64_t>(b) * p.ld + s_abs] = acc;
              if (p.hist) atomicAdd(&hist_s[f32_key(acc) >> 20], 1u);
            }
          } else {
            const int32_t row = r0 + g * C::NQ + qq;
            if (row < p.n_q && s_abs <= static_cast<int64_t>(p.q_pos0) + row && s_abs < p.n_tokens)
              p.scores[static_cast<int64_t>(row) * p.ld + s_abs] = acc;
          }
        };
        const uint32_t trow = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + bf * C::N;
        const int q0 = PAGED ? 0 : part * QPW;
        uint32_t xa[32], xb[32];
        if constexpr (QPW == 2) {
          // both queries' accumulators in flight at once: one TMEM load latency per group
          DSA_TMEM_LD_X32_NOWAIT(trow + q0 * 32, xa);
          DSA_TMEM_LD_X32_NOWAIT(trow + (q0 + 1) * 32, xb);
          DSA_TMEM_WAIT_LD2(xa, xb);
          score(xa, q0);
          score(xb, q0 + 1);
        } else {
          // TMEM loads run one query ahead of the math
          DSA_TMEM_LD_X32_NOWAIT(trow + q0 * 32, xa);
#pragma unroll
          for (int j = 0; j < QPW; j += 2) {
            DSA_TMEM_WAIT_LD(xa);
            if (j + 1 < QPW) DSA_TMEM_LD_X32_NOWAIT(trow + (q0 + j + 1) * 32, xb);
            score(xa, q0 + j);
            if (j + 1 < QPW) {
              DSA_TMEM_WAIT_LD(xb);
              if (j + 2 < QPW) DSA_TMEM_LD_X32_NOWAIT(trow + (q0 + j + 2) * 32, xa);
              score(xb, q0 + j + 1);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty(bf));
        ++job;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (PAGED && p.hist) {  // this CTA's counts into the sequence's histogram
    uint32_t* g = p.hist + static_cast<int64_t>(b) * C::HIST_BINS;
    for (int i = threadIdx.x; i < C::HIST_BINS; i += C::THREADS)
      if (hist_s[i]) atomicAdd(&g[i], hist_s[i]);
  }
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace idx
}  // namespace dsa

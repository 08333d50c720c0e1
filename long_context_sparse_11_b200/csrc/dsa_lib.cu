// Host side of the C ABI declared in include/dsa.h: argument validation, tensor-map
// encoding, launch configuration and the IndexShare group orchestration.  All device
// memory is owned by the caller; the only library state is one device status word per
// device, per-device launch attributes, and the thread-local error text.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <vector>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/dsa.h"
#include "gemm.cuh"
#include "indexer.cuh"
#include "mla.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "splitn.cuh"
#include "topk.cuh"

namespace dsa {

__device__ int g_status_word;  // DEVERR_* bits, cleared by dsa_sync_status

// Test hook: an mbarrier that expects two arrivals but gets one; the bounded wait runs out.
__global__ void debug_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 2);
    fence_mbar_init();
    mbar_arrive(smem_u32(&bar));
    mbar_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
  }
}

namespace {

thread_local std::string t_err;
int64_t g_wait_ns = 2000000000LL;
std::atomic<int64_t> g_launches{0};

void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Programmatic dependent launch for the kernels of a group (each starts with grid_dependency_sync):
// a kernel's launch overlaps the completion of the previous kernel of the stream, which matters for
// decode steps of a few hundred short kernels.  DSA_PDL=0 in the environment launches them plainly
// (same results, for timing the difference).
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DSA_PDL");
    return e == nullptr || std::atoi(e) != 0;
  }();
  return on;
}
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  // a failed launch is left for the caller's cudaGetLastError, like a <<<>>> launch
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

void trace(void** ev, int i, cudaStream_t st) {
  if (ev && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st);
}

dsa_status fail(dsa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

dsa_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DSA_OK;
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DSA_TRY(x)                       \
  do {                                   \
    const dsa_status _s = (x);           \
    if (_s != DSA_OK) return _s;         \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceState {
  bool ready = false;
  int sms = 148;
  int* status = nullptr;
};

DeviceState g_dev[64];
std::mutex g_mu;

dsa_status device_state(DeviceState** out) {
  int dev = 0;
  DSA_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= 64) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    DSA_TRY(cuda_check(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "attr"));
    DSA_TRY(cuda_check(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "attr"));
    if (major != 10 || minor != 0)
      return fail(DSA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev,
                  major, minor);
    DSA_TRY(cuda_check(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev), "attr"));
    void* sym = nullptr;
    DSA_TRY(cuda_check(cudaGetSymbolAddress(&sym, g_status_word), "cudaGetSymbolAddress(status)"));
    d.status = static_cast<int*>(sym);
    DSA_TRY(cuda_check(cudaFuncSetAttribute(idx::indexer_kernel<false, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            idx::Cfg<false, false>::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(idx::indexer_kernel<true, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            idx::Cfg<true, false>::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(idx::indexer_kernel<true, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            idx::Cfg<true, true>::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(mla::sparse_mla_kernel<false, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, mla::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(mla::sparse_mla_kernel<true, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, mla::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(mla::sparse_mla_kernel<false, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, mla::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(mla::sparse_mla_kernel<true, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, mla::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(gemm::gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            gemm::SMEM_BYTES),
                       "smem attr"));
    DSA_TRY(cuda_check(cudaFuncSetAttribute(topk::topk_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(sizeof(topk::Smem))),
                       "smem attr"));
    d.ready = true;
  }
  *out = &d;
  return DSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D tiled map with 128-byte swizzle: [outer rows x inner elements], row stride in bytes.
dsa_status make_map(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer,
                    uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------- validation

dsa_status check_view(const dsa_cache_view* v, int32_t dim, const char* name) {
  if (!v) return fail(DSA_ERR_INVALID_ARG, "%s: null cache view", name);
  if (!v->data || !aligned16(v->data)) return fail(DSA_ERR_INVALID_ARG, "%s: data null or not 16-byte aligned", name);
  if (v->dim != dim) return fail(DSA_ERR_UNSUPPORTED, "%s: dim %d, expected %d", name, v->dim, dim);
  if (v->dtype != DSA_BF16 && v->dtype != DSA_E4M3) return fail(DSA_ERR_INVALID_ARG, "%s: bad dtype", name);
  const int64_t es = v->dtype == DSA_BF16 ? 2 : 1;
  if (v->n_tokens < 0) return fail(DSA_ERR_INVALID_ARG, "%s: n_tokens < 0", name);
  if (v->dtype == DSA_E4M3 && (!v->scale || !aligned16(v->scale)))
    return fail(DSA_ERR_INVALID_ARG, "%s: e4m3 cache needs a 16-byte aligned scale array", name);
  if (v->block_table) {
    if (v->dtype != DSA_E4M3) return fail(DSA_ERR_UNSUPPORTED, "%s: paged caches must be e4m3", name);
    if (v->row_stride != dim) return fail(DSA_ERR_INVALID_ARG, "%s: paged row_stride must equal dim", name);
    if (!v->seq_lens) return fail(DSA_ERR_INVALID_ARG, "%s: paged cache needs seq_lens", name);
    if (v->max_pages <= 0 || v->batch <= 0) return fail(DSA_ERR_INVALID_ARG, "%s: bad max_pages/batch", name);
    if (v->n_tokens % DSA_PAGE) return fail(DSA_ERR_INVALID_ARG, "%s: n_tokens must be pages*64", name);
    if (v->n_tokens / DSA_PAGE > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "%s: too many pages", name);
  } else {
    if (v->row_stride < dim || (v->row_stride * es) % 16)
      return fail(DSA_ERR_INVALID_ARG, "%s: row_stride %lld invalid", name, static_cast<long long>(v->row_stride));
    if (v->n_tokens > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "%s: n_tokens too large", name);
  }
  return DSA_OK;
}

// ---------------------------------------------------------------------------- launches

dsa_status launch_indexer(const void* q, int32_t q_dtype, const float* q_scale, const float* w, int32_t n_q,
                          int32_t q_pos0, const dsa_cache_view* keys, float* scores, int64_t ld,
                          cudaStream_t st, uint32_t* hist = nullptr) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  const bool fp8 = q_dtype == DSA_E4M3;
  const bool paged = keys->block_table != nullptr;
  idx::Params p{};
  p.q_scale = q_scale;
  p.w = w;
  p.key_scale = keys->scale;
  p.block_table = keys->block_table;
  p.seq_lens = keys->seq_lens;
  p.scores = scores;
  p.ld = ld;
  p.n_tokens = keys->n_tokens;
  p.n_q = n_q;
  p.q_pos0 = q_pos0;
  p.max_pages = keys->max_pages;
  p.n_pages = static_cast<int32_t>(keys->n_tokens / DSA_PAGE);
  p.status = ds->status;
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  p.unit_tiles = idx::UNIT_TILES;
  p.hist = keys->block_table ? hist : nullptr;
  CUtensorMap mq, mk;
  const uint64_t qrows = static_cast<uint64_t>(n_q) * 32;
  if (paged) {
    DSA_TRY(make_map(&mq, q, false, 128, qrows, 128, 128, 32));
    DSA_TRY(make_map(&mk, keys->data, false, 128, static_cast<uint64_t>(keys->n_tokens), 128, 128, 64));
    const int64_t max_len = static_cast<int64_t>(keys->max_pages) * DSA_PAGE;
    const int64_t tiles = (max_len + idx::BLOCK_KEYS - 1) / idx::BLOCK_KEYS;
    // few long sequences: shorter units, so that the grid still covers the SMs several times over
    // (units sized to fill exactly one wave of resident CTAs measured slower on a 1M-token sequence)
    int32_t unit = idx::UNIT_TILES;
    while (unit > 4 && static_cast<int64_t>(n_q) * ((tiles + unit - 1) / unit) < 4LL * ds->sms) unit /= 2;
    p.unit_tiles = unit;
    dim3 grid(static_cast<unsigned>((tiles + unit - 1) / unit), static_cast<unsigned>(n_q));
    using C = idx::Cfg<true, true>;
    launch_pdl(idx::indexer_kernel<true, true>, grid, C::THREADS, C::SMEM_BYTES, st, mq, mk, p);
    count_launch();
  } else {
    const int64_t max_len = std::min<int64_t>(static_cast<int64_t>(q_pos0) + n_q, keys->n_tokens);
    const int64_t tiles = (max_len + idx::BLOCK_KEYS - 1) / idx::BLOCK_KEYS;
    if (tiles <= 0) return DSA_OK;
    if (fp8) {
      using C = idx::Cfg<true, false>;
      DSA_TRY(make_map(&mq, q, false, 128, qrows, 128, 128, 256));
      DSA_TRY(make_map(&mk, keys->data, false, 128, static_cast<uint64_t>(keys->n_tokens),
                       static_cast<uint64_t>(keys->row_stride), 128, 128));
      dim3 grid(static_cast<unsigned>((tiles + idx::UNIT_TILES - 1) / idx::UNIT_TILES),
                static_cast<unsigned>((n_q + 15) / 16));
      launch_pdl(idx::indexer_kernel<true, false>, grid, C::THREADS, C::SMEM_BYTES, st, mq, mk, p);
      count_launch();
    } else {
      using C = idx::Cfg<false, false>;
      DSA_TRY(make_map(&mq, q, true, 128, qrows, 256, 64, 256));
      DSA_TRY(make_map(&mk, keys->data, true, 128, static_cast<uint64_t>(keys->n_tokens),
                       static_cast<uint64_t>(keys->row_stride) * 2, 64, 128));
      dim3 grid(static_cast<unsigned>((tiles + idx::UNIT_TILES - 1) / idx::UNIT_TILES),
                static_cast<unsigned>((n_q + 15) / 16));
      launch_pdl(idx::indexer_kernel<false, false>, grid, C::THREADS, C::SMEM_BYTES, st, mq, mk, p);
      count_launch();
    }
  }
  return cuda_check(cudaGetLastError(), "indexer launch");
}

// Top-k launch plan: row mode unless the rows are too few to fill the GPU and long.
struct TopkPlan {
  bool segmented = false;
  int32_t segs = 1;
  int32_t seg_len = 0;
  int32_t gcap = 0;
  size_t ws = 0;
};

TopkPlan plan_topk(int32_t n_rows, int64_t max_len, int32_t k, int sms) {
  TopkPlan pl;
  if (n_rows <= 0 || max_len <= k || n_rows >= 2 * sms || max_len <= 32768) return pl;
  pl.segmented = true;
  const int64_t by_len = (max_len + 8191) / 8192;  // at least 8K candidates per segment
  int64_t segs = (4LL * sms + n_rows - 1) / n_rows;
  segs = std::max<int64_t>(1, std::min(segs, by_len));
  pl.segs = static_cast<int32_t>(segs);
  pl.seg_len = static_cast<int32_t>(align_up(static_cast<size_t>((max_len + segs - 1) / segs), 4));
  pl.gcap = static_cast<int32_t>(std::max<int64_t>(topk::CAND_CAP, std::min<int64_t>(max_len, 1 << 16)));
  pl.ws = static_cast<size_t>(n_rows) * (topk::BINS * 4 + 16 + static_cast<size_t>(pl.gcap) * 8) + 256;
  return pl;
}

// hist_ready: the caller zeroed the workspace head (histograms + counters) and filled the
// first-digit histograms itself (the paged indexer does, in its epilogue), so the segmented plan
// skips its histogram pass.
dsa_status launch_topk(const float* scores, int64_t ld, int32_t n_rows, const int32_t* row_len,
                       int64_t causal_len0, int64_t max_len, int32_t k, int32_t* idx_out, void* ws,
                       size_t ws_bytes, cudaStream_t st, bool hist_ready = false) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  const int64_t cap = std::min(ld, max_len);
  const TopkPlan pl = plan_topk(n_rows, cap, k, ds->sms);
  if (!pl.segmented) {
    launch_pdl(topk::topk_row_kernel, n_rows, topk::THREADS, sizeof(topk::Smem), st, scores, ld, n_rows, row_len,
                                                                             causal_len0, cap, k, idx_out);
    count_launch();
    return cuda_check(cudaGetLastError(), "topk launch");
  }
  if (!ws || ws_bytes < pl.ws)
    return fail(DSA_ERR_WORKSPACE, "topk needs %zu workspace bytes, got %zu", pl.ws, ws_bytes);
  uint8_t* b = static_cast<uint8_t*>(ws);
  topk::SegWs sw;
  sw.hist = reinterpret_cast<uint32_t*>(b);
  sw.counters = reinterpret_cast<int32_t*>(b + static_cast<size_t>(n_rows) * topk::BINS * 4);
  const size_t head = static_cast<size_t>(n_rows) * (topk::BINS * 4 + 16);
  sw.cand_key = reinterpret_cast<uint32_t*>(b + head);
  sw.cand_idx = reinterpret_cast<int32_t*>(b + head + static_cast<size_t>(n_rows) * pl.gcap * 4);
  sw.gcap = pl.gcap;
  dim3 grid(pl.segs, n_rows);
  if (!hist_ready) {
    DSA_TRY(cuda_check(cudaMemsetAsync(ws, 0, head, st), "topk workspace clear"));
    launch_pdl(topk::topk_seg_hist_kernel, grid, topk::SEG_THREADS, 0, st, scores, ld, row_len, causal_len0, cap, k,
                                                                   pl.seg_len, sw);
    count_launch();
  }
  launch_pdl(topk::topk_seg_filter_kernel, grid, topk::SEG_THREADS, 0, st, scores, ld, row_len, causal_len0, cap, k,
                                                                   pl.seg_len, sw, idx_out);
  count_launch();
  return cuda_check(cudaGetLastError(), "topk launch");
}

int32_t mla_splits(int32_t n_q, int32_t k, int sms) {
  // persistent CTAs take (row, split) items round-robin: aim for >= 2 items per SM when the
  // rows alone are too few, with equal tiles per split
  const int32_t tiles = (k + mla::TILE - 1) / mla::TILE;
  if (n_q >= 2 * sms || tiles <= 1) return 1;
  int32_t s = (2 * sms + n_q - 1) / n_q;
  s = std::min(s, tiles);
  // balance: equal tiles per split
  const int32_t tps = (tiles + s - 1) / s;
  return (tiles + tps - 1) / tps;
}

// Stream-K schedule for few rows (decode): grid and the most fragments any row is cut into.
struct StreamK {
  bool on = false;
  int32_t grid = 0, slots = 0, tiles_per_row = 0;
  int64_t tiles = 0;
};
StreamK plan_stream_k(int32_t n_q, int32_t k, int sms) {
  StreamK sk;
  const int32_t tpr = (k + mla::TILE - 1) / mla::TILE;
  if (n_q <= 0 || n_q >= 2 * sms || tpr <= 1) return sk;
  // worth it with several tiles per CTA (measured: 17 tiles per CTA 0.180 -> 0.160 ms per layer;
  // at 1 and 3.5 tiles per CTA equal splits were as fast or faster)
  if (static_cast<int64_t>(n_q) * tpr < 8LL * sms) return sk;
  sk.on = true;
  sk.tiles_per_row = tpr;
  sk.tiles = static_cast<int64_t>(n_q) * tpr;
  sk.grid = static_cast<int32_t>(std::min<int64_t>(sk.tiles, sms));
  for (int32_t r = 0; r < n_q; ++r) {
    const int64_t g0 = static_cast<int64_t>(r) * tpr;
    const int64_t s = mla::sk_owner(g0 + tpr - 1, sk.tiles, sk.grid) - mla::sk_owner(g0, sk.tiles, sk.grid) + 1;
    sk.slots = std::max(sk.slots, static_cast<int32_t>(s));
  }
  return sk;
}

size_t mla_ws_bytes(int32_t n_q, int32_t k, int sms) {
  // either schedule may run (stream-K unless the rows are causal prefill rows): room for both
  const int32_t s = std::max(mla_splits(n_q, k, sms), plan_stream_k(n_q, k, sms).slots);
  if (s <= 1) return 0;
  return static_cast<size_t>(n_q) * s * (64 * 512 * 4 + 128 * 4) + 256;
}

// A paged group converts its query rows to f16 once, ahead of the attention, when every row is cut
// over at least 8 CTAs (few rows): each of those CTAs would otherwise convert the same row.  Measured
// on decode: 6 rows x 16 splits and 32 rows x 8 splits gain; 160 rows (2-3 stream-K fragments per
// row) convert inside the kernel, where no extra launch or memory traffic is paid.
bool mla_query_prepass(int32_t n_q, int32_t k, int sms) {
  const StreamK sk = plan_stream_k(n_q, k, sms);
  const int32_t cuts = sk.on ? sk.slots : mla_splits(n_q, k, sms);
  return cuts >= 8;
}

dsa_status launch_mla(const void* q, const dsa_cache_view* kv, const int32_t* idx, int32_t n_q, int32_t rpi,
                      int32_t k, float softmax_scale, void* out, float* lse, void* ws, size_t ws_bytes,
                      cudaStream_t st, int64_t valid0 = -1, const void* q16 = nullptr) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  if (n_q == 0) return DSA_OK;
  const bool paged = kv->block_table != nullptr;
  mla::Params p{};
  p.q = static_cast<const uint16_t*>(q);
  p.kv = static_cast<const uint8_t*>(kv->data);
  p.kv_scale = kv->scale;
  p.block_table = kv->block_table;
  p.seq_lens = kv->seq_lens;
  p.idx = idx;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.row_stride = kv->row_stride;
  p.n_tokens = kv->n_tokens;
  p.n_q = n_q;
  p.rows_per_idx = rpi;
  p.k = k;
  p.max_pages = kv->max_pages;
  p.n_pages = static_cast<int32_t>(kv->n_tokens / DSA_PAGE);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.status = ds->status;
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  p.n_split = mla_splits(n_q, k, ds->sms);
  p.valid0 = valid0;
  if (paged && q16) {  // rows converted to f16 ahead of this launch
    p.q = static_cast<const uint16_t*>(q16);
    p.q_f16 = 1;
  }
  // few rows whose tiles all count (decode): contiguous tile ranges per CTA instead of equal splits
  const StreamK sk = valid0 < 0 ? plan_stream_k(n_q, k, ds->sms) : StreamK{};
  if (sk.on) {
    p.stream_k = 1;
    p.n_split = sk.slots;
  }
  if (p.n_split > 1) {
    const size_t need = mla_ws_bytes(n_q, k, ds->sms);
    if (!ws || ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "sparse MLA needs %zu workspace bytes", need);
    p.part_o = static_cast<float*>(ws);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                         static_cast<size_t>(n_q) * p.n_split * 64 * 512 * 4);
  }
  const unsigned grid = sk.on ? static_cast<unsigned>(sk.grid)
                              : static_cast<unsigned>(std::min<int64_t>(static_cast<int64_t>(n_q) * p.n_split,
                                                                        static_cast<int64_t>(ds->sms)));
  if (paged && sk.on) {
    launch_pdl(mla::sparse_mla_kernel<true, true>, grid, mla::THREADS, mla::SMEM_BYTES, st, p);
  } else if (paged) {
    launch_pdl(mla::sparse_mla_kernel<true, false>, grid, mla::THREADS, mla::SMEM_BYTES, st, p);
  } else if (sk.on) {
    launch_pdl(mla::sparse_mla_kernel<false, true>, grid, mla::THREADS, mla::SMEM_BYTES, st, p);
  } else {
    launch_pdl(mla::sparse_mla_kernel<false, false>, grid, mla::THREADS, mla::SMEM_BYTES, st, p);
  }
  count_launch();
  DSA_TRY(cuda_check(cudaGetLastError(), "sparse MLA launch"));
  if (p.n_split > 1) {
    // rows cut into more than 4 slots, few enough that all (row, head) blocks run in one wave
    // even at the occupancy of the all-slots variant (6 blocks per SM): every slot in flight
    const bool all_slots = p.n_split > 4 && static_cast<int64_t>(n_q) * 64 <= 6LL * ds->sms;
    if (all_slots)
      launch_pdl(mla::combine_kernel<mla::MAX_SLOTS>, dim3(n_q, 64), 128, 0, st,
          p.part_o, p.part_ml, p.n_split, p.out, p.lse, sk.tiles_per_row, sk.tiles, sk.on ? sk.grid : 0);
    else
      launch_pdl(mla::combine_kernel<4>, dim3(n_q, 64), 128, 0, st, p.part_o, p.part_ml, p.n_split, p.out, p.lse,
                                                           sk.tiles_per_row, sk.tiles, sk.on ? sk.grid : 0);
    count_launch();
    DSA_TRY(cuda_check(cudaGetLastError(), "combine launch"));
  }
  return DSA_OK;
}

// C[m, n] (fp32 or bf16, row stride ldc) = A[m, k] . B[n, k]^T, A and B bf16 with rows of k.
dsa_status launch_gemm(const void* A, const void* B, int32_t m, int32_t n, int32_t k, void* C, int64_t ldc,
                       bool out_bf16, cudaStream_t st) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  if (m == 0 || n == 0) return DSA_OK;
  CUtensorMap ma, mb;
  DSA_TRY(make_map(&ma, A, true, static_cast<uint64_t>(k), static_cast<uint64_t>(m), static_cast<uint64_t>(k) * 2, 64,
                   gemm::BM));
  DSA_TRY(make_map(&mb, B, true, static_cast<uint64_t>(k), static_cast<uint64_t>(n), static_cast<uint64_t>(k) * 2, 64,
                   gemm::BN));
  gemm::Params p{};
  p.c = C;
  p.ldc = ldc;
  p.m = m;
  p.n = n;
  p.k = k;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.status = ds->status;
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  dim3 grid(static_cast<unsigned>((n + gemm::BN - 1) / gemm::BN), static_cast<unsigned>((m + gemm::BM - 1) / gemm::BM));
  gemm::gemm_bf16_kernel<<<grid, gemm::THREADS, gemm::SMEM_BYTES, st>>>(ma, mb, p);
  count_launch();
  return cuda_check(cudaGetLastError(), "projection GEMM launch");
}

// ---------------------------------------------------------------------------- group plan

struct Chunk {
  int32_t row0, rows;  // query rows [row0, row0 + rows) of the group
  int64_t ld, max_len; // score row stride and longest candidate row of the chunk
};

struct GroupPlan {
  bool quant_q = false, quant_k = false;
  size_t off_q8 = 0, off_sq = 0, off_k8 = 0, off_sk = 0, off_scores = 0, off_topk = 0, off_mla = 0, total = 0;
  size_t off_q16 = 0, q16_layer_bytes = 0;  // f16 query rows of the paged layers (when converted ahead)
  std::vector<Chunk> chunks;
  size_t topk_ws = 0;
};

// Score block per query chunk: at least 64 MB (L2-sized), and large enough that the last
// chunks of a long prefill still hold kScoreMinRows rows (fewer, fuller launches), at most 1 GB.
constexpr int64_t kScoreBudgetFloats = 16LL << 20;
constexpr int64_t kScoreBudgetMaxFloats = 256LL << 20;
#ifndef DSA_SCORE_MIN_ROWS
#define DSA_SCORE_MIN_ROWS 2048
#endif
constexpr int64_t kScoreMinRows = DSA_SCORE_MIN_ROWS;

dsa_status plan_group(const dsa_group_args* a, int sms, GroupPlan* g) {
  const dsa_cache_view& kv = a->idx_keys;
  const bool paged = kv.block_table != nullptr;
  const int64_t n = a->n_idx_rows;
  g->quant_q = a->indexer_dtype == DSA_E4M3;
  g->quant_k = a->indexer_dtype == DSA_E4M3 && kv.dtype == DSA_BF16;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  if (g->quant_q) {
    g->off_q8 = take(static_cast<size_t>(n) * 32 * 128);
    g->off_sq = take(static_cast<size_t>(n) * 32 * 4);
  }
  if (g->quant_k) {
    g->off_k8 = take(static_cast<size_t>(kv.n_tokens) * 128);
    g->off_sk = take(static_cast<size_t>(kv.n_tokens) * 4);
  }
  // Query-row chunks whose [rows, ld] score block fits the budget: causal rows grow with the
  // position, so early chunks take more (shorter) rows than late ones.
  g->chunks.clear();
  size_t score_floats = 0;
  if (paged) {
    const int64_t len = static_cast<int64_t>(kv.max_pages) * DSA_PAGE;
    g->chunks.push_back({0, static_cast<int32_t>(n), len, len});
    score_floats = static_cast<size_t>(n) * len;
  } else {
    const int64_t longest = std::min<int64_t>(static_cast<int64_t>(a->q_pos0) + n, kv.n_tokens);
    const int64_t budget = std::min(kScoreBudgetMaxFloats, std::max(kScoreBudgetFloats, kScoreMinRows * longest));
    for (int64_t c0 = 0; c0 < n;) {
      const double a0 = static_cast<double>(a->q_pos0) + static_cast<double>(c0);
      int64_t c = static_cast<int64_t>((-a0 + std::sqrt(a0 * a0 + 4.0 * static_cast<double>(budget))) / 2.0);
      c = std::max<int64_t>(16, c / 16 * 16);
      c = std::min<int64_t>(c, n - c0);
      int64_t len = 0, ld = 0;
      for (;; c -= 16) {
        len = std::min<int64_t>(static_cast<int64_t>(a->q_pos0) + c0 + c, kv.n_tokens);
        ld = static_cast<int64_t>(align_up(static_cast<size_t>(std::max<int64_t>(len, 4)), 4));
        if (c <= 16 || c * ld <= budget) break;
      }
      g->chunks.push_back({static_cast<int32_t>(c0), static_cast<int32_t>(c), ld, len});
      score_floats = std::max(score_floats, static_cast<size_t>(c) * ld);
      c0 += c;
    }
  }
  g->topk_ws = 0;
  for (const Chunk& ch : g->chunks)
    g->topk_ws = std::max(g->topk_ws, plan_topk(ch.rows, ch.max_len, a->k, sms).ws);
  g->off_scores = take(score_floats * 4);
  g->off_topk = take(g->topk_ws);
  size_t mla_ws = 0;
  const int32_t nq = a->n_idx_rows * a->q_rows_per_idx_row;
  mla_ws = mla_ws_bytes(nq, a->k, sms);
  int n_paged = 0;
  for (int l = 0; l < a->n_layers; ++l) n_paged += a->kv[l].block_table != nullptr;
  if (n_paged > 0 && mla_query_prepass(nq, a->k, sms)) {
    g->q16_layer_bytes = static_cast<size_t>(nq) * 64 * 576 * 2;
    g->off_q16 = take(g->q16_layer_bytes * n_paged);
  }
  g->off_mla = take(mla_ws);
  g->total = off;
  return DSA_OK;
}

dsa_status check_group(const dsa_group_args* a) {
  if (!a) return fail(DSA_ERR_INVALID_ARG, "null group args");
  if (a->n_layers < 1 || a->n_layers > DSA_GROUP_MAX_LAYERS)
    return fail(DSA_ERR_INVALID_ARG, "n_layers %d not in [1,4]", a->n_layers);
  if (a->k < 1 || a->k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", a->k);
  if (a->n_idx_rows < 0 || a->q_rows_per_idx_row < 1) return fail(DSA_ERR_INVALID_ARG, "bad row counts");
  if (a->indexer_dtype != DSA_BF16 && a->indexer_dtype != DSA_E4M3)
    return fail(DSA_ERR_INVALID_ARG, "bad indexer_dtype");
  DSA_TRY(check_view(&a->idx_keys, 128, "idx_keys"));
  if (a->indexer_dtype == DSA_BF16 && a->idx_keys.dtype != DSA_BF16)
    return fail(DSA_ERR_UNSUPPORTED, "bf16 indexer needs bf16 keys");
  if (a->idx_keys.block_table && a->idx_keys.batch != a->n_idx_rows)
    return fail(DSA_ERR_INVALID_ARG, "paged indexer keys: batch %d != n_idx_rows %d", a->idx_keys.batch,
                a->n_idx_rows);
  if (!a->q_idx || !aligned16(a->q_idx) || !a->w || !aligned16(a->w))
    return fail(DSA_ERR_INVALID_ARG, "q_idx / w null or misaligned");
  for (int l = 0; l < a->n_layers; ++l) {
    DSA_TRY(check_view(&a->kv[l], 576, "kv"));
    if (!a->q[l] || !aligned16(a->q[l]) || !a->out[l] || !aligned16(a->out[l]))
      return fail(DSA_ERR_INVALID_ARG, "layer %d: q/out null or misaligned", l);
    if (a->lse[l] && !aligned16(a->lse[l])) return fail(DSA_ERR_INVALID_ARG, "layer %d: lse misaligned", l);
    if (!a->kv[l].block_table && a->kv[l].dtype != DSA_BF16)
      return fail(DSA_ERR_UNSUPPORTED, "dense latent caches must be bf16");
    if (a->kv[l].block_table && a->kv[l].batch != a->n_idx_rows)
      return fail(DSA_ERR_INVALID_ARG, "layer %d: paged batch != n_idx_rows", l);
  }
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

// ================================================================================= C ABI

extern "C" {

int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

size_t dsa_abi_sizeof(int32_t which) {
  switch (which) {
    case 0: return sizeof(dsa_cache_view);
    case 1: return sizeof(dsa_index_handle);
    case 2: return sizeof(dsa_group_args);
  }
  return 0;
}

const char* dsa_status_str(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported";
    case DSA_ERR_STALE_HANDLE: return "stale index handle";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_BOUNDS: return "index or page out of range";
    case DSA_ERR_RANGE: return "input value outside the supported range";
  }
  return "unknown status";
}

const char* dsa_last_error(void) { return t_err.c_str(); }

int64_t dsa_launch_count(void) { return g_launches.load(); }

int64_t dsa_set_wait_limit_ns(int64_t ns) {
  const int64_t old = g_wait_ns;
  if (ns > 0) g_wait_ns = ns;
  return old;
}

int32_t dsa_layer_is_full(int32_t layer) { return layer >= 0 && (layer < 2 || (layer - 2) % 4 == 0) ? 1 : 0; }
int32_t dsa_layer_producer(int32_t layer) {
  if (layer < 0) return -1;
  if (dsa_layer_is_full(layer)) return layer;
  return 2 + 4 * ((layer - 2) / 4);
}

dsa_status dsa_sync_status(void* stream) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  DSA_TRY(cuda_check(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize"));
  int v = 0;
  DSA_TRY(cuda_check(cudaMemcpy(&v, ds->status, sizeof(int), cudaMemcpyDeviceToHost), "read status"));
  const int zero = 0;
  DSA_TRY(cuda_check(cudaMemcpy(ds->status, &zero, sizeof(int), cudaMemcpyHostToDevice), "clear status"));
  if (v & DEVERR_TIMEOUT) return fail(DSA_ERR_TIMEOUT, "a bounded device wait ran out");
  if (v & DEVERR_BOUNDS) return fail(DSA_ERR_BOUNDS, "a kernel skipped an out-of-range index or page");
  if (v & DEVERR_RANGE)
    return fail(DSA_ERR_RANGE, "a query value of an attention over an e4m3 cache exceeds the f16 range");
  return DSA_OK;
}

dsa_status dsa_debug_bounded_wait(int64_t timeout_ns, void* stream) {
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return fail(DSA_ERR_INVALID_ARG, "timeout out of range");
  debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ds->status,
                                                                      static_cast<uint64_t>(timeout_ns));
  count_launch();
  return cuda_check(cudaGetLastError(), "debug wait launch");
}

dsa_status dsa_quant_e4m3(const void* x_bf16, int64_t n_vec, int32_t vec_len, uint8_t* codes, float* scale,
                          void* stream) {
  if (vec_len != 128) return fail(DSA_ERR_UNSUPPORTED, "vec_len %d (only 128)", vec_len);
  if (n_vec < 0) return fail(DSA_ERR_INVALID_ARG, "n_vec < 0");
  if (n_vec == 0) return DSA_OK;
  if (!x_bf16 || !codes || !scale || !aligned16(x_bf16) || !aligned16(codes) || !aligned16(scale))
    return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  const int64_t blocks = (n_vec + 7) / 8;
  if (blocks > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "n_vec too large");
  launch_pdl(quant_e4m3_kernel, static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream),
      static_cast<const uint16_t*>(x_bf16), n_vec, codes, scale);
  count_launch();
  return cuda_check(cudaGetLastError(), "quant launch");
}

dsa_status dsa_cache_write_e4m3(const void* x_bf16, int32_t n_rows, int32_t dim, const int32_t* seq,
                                const int32_t* pos, const int32_t* block_table, int32_t batch, int32_t max_pages,
                                int32_t n_pages, uint8_t* pool, float* pool_scale, void* stream) {
  if (dim != 128 && dim != 576) return fail(DSA_ERR_UNSUPPORTED, "cache write dim %d (128 or 576)", dim);
  if (n_rows < 0 || batch < 0 || max_pages < 0 || n_pages < 0) return fail(DSA_ERR_INVALID_ARG, "negative size");
  if (n_rows == 0) return DSA_OK;
  if (!x_bf16 || !aligned16(x_bf16) || !pos || !block_table || !pool || !aligned16(pool) || !pool_scale)
    return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  if (batch == 0 || max_pages == 0 || n_pages == 0) return fail(DSA_ERR_INVALID_ARG, "empty cache");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  const int64_t blocks = (static_cast<int64_t>(n_rows) + 7) / 8;
  launch_pdl(cache_write_e4m3_kernel, static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream),
      static_cast<const uint16_t*>(x_bf16), n_rows, dim, seq, pos, block_table, batch, max_pages, n_pages, pool,
      pool_scale, ds->status);
  count_launch();
  return cuda_check(cudaGetLastError(), "cache write launch");
}

dsa_status dsa_cache_write_e4m3_pools(int32_t n_pools, const void* const* x_bf16, const int32_t* dims,
                                      uint8_t* const* pools, float* const* pool_scales, int32_t n_rows,
                                      const int32_t* seq, const int32_t* pos, const int32_t* block_table, int32_t batch,
                                      int32_t max_pages, int32_t n_pages, void* stream) {
  if (n_pools < 0 || n_pools > CACHE_WRITE_MAX_POOLS)
    return fail(DSA_ERR_INVALID_ARG, "n_pools %d not in [0, %d]", n_pools, CACHE_WRITE_MAX_POOLS);
  if (n_rows < 0 || batch < 0 || max_pages < 0 || n_pages < 0) return fail(DSA_ERR_INVALID_ARG, "negative size");
  if (n_rows == 0 || n_pools == 0) return DSA_OK;
  if (!x_bf16 || !dims || !pools || !pool_scales || !pos || !block_table)
    return fail(DSA_ERR_INVALID_ARG, "null pointer");
  if (batch == 0 || max_pages == 0 || n_pages == 0) return fail(DSA_ERR_INVALID_ARG, "empty cache");
  CacheWritePools pp{};
  for (int32_t i = 0; i < n_pools; ++i) {
    if (dims[i] != 128 && dims[i] != 576) return fail(DSA_ERR_UNSUPPORTED, "pool %d: dim %d (128 or 576)", i, dims[i]);
    if (!x_bf16[i] || !aligned16(x_bf16[i]) || !pools[i] || !aligned16(pools[i]) || !pool_scales[i])
      return fail(DSA_ERR_INVALID_ARG, "pool %d: null or misaligned pointer", i);
    pp.x[i] = static_cast<const uint16_t*>(x_bf16[i]);
    pp.pool[i] = pools[i];
    pp.scale[i] = pool_scales[i];
    pp.dim[i] = dims[i];
  }
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  const dim3 grid(static_cast<unsigned>((static_cast<int64_t>(n_rows) + 7) / 8), static_cast<unsigned>(n_pools));
  launch_pdl(cache_write_e4m3_pools_kernel, grid, 256, 0, static_cast<cudaStream_t>(stream),
      pp, n_rows, seq, pos, block_table, batch, max_pages, n_pages, ds->status);
  count_launch();
  return cuda_check(cudaGetLastError(), "cache write launch");
}

dsa_status dsa_indexer_score(const void* q, int32_t q_dtype, const float* q_scale, const float* w, int32_t n_q,
                             int32_t q_pos0, const dsa_cache_view* keys, float* scores, int64_t ld_scores,
                             void* stream) {
  DSA_TRY(check_view(keys, 128, "keys"));
  if (n_q < 0 || q_pos0 < 0) return fail(DSA_ERR_INVALID_ARG, "n_q / q_pos0 negative");
  if (n_q == 0) return DSA_OK;
  if (q_dtype != keys->dtype) return fail(DSA_ERR_UNSUPPORTED, "q dtype must equal key dtype");
  if (!q || !aligned16(q) || !w || !aligned16(w) || !scores || !aligned16(scores))
    return fail(DSA_ERR_INVALID_ARG, "q / w / scores null or misaligned");
  if (q_dtype == DSA_E4M3 && (!q_scale || !aligned16(q_scale)))
    return fail(DSA_ERR_INVALID_ARG, "e4m3 queries need q_scale");
  if (ld_scores <= 0 || ld_scores % 4) return fail(DSA_ERR_INVALID_ARG, "ld_scores must be a positive multiple of 4");
  if (keys->block_table) {
    if (keys->batch != n_q) return fail(DSA_ERR_INVALID_ARG, "paged keys: batch != n_q");
    if (ld_scores < static_cast<int64_t>(keys->max_pages) * DSA_PAGE)
      return fail(DSA_ERR_INVALID_ARG, "ld_scores < max_pages*64");
  } else {
    if (ld_scores < std::min<int64_t>(static_cast<int64_t>(q_pos0) + n_q, keys->n_tokens))
      return fail(DSA_ERR_INVALID_ARG, "ld_scores shorter than the longest row");
  }
  return launch_indexer(q, q_dtype, q_scale, w, n_q, q_pos0, keys, scores, ld_scores,
                        static_cast<cudaStream_t>(stream));
}

size_t dsa_indexer_project_workspace_bytes(int32_t n_tokens) {
  return n_tokens <= 0 ? 0 : static_cast<size_t>(n_tokens) * 160 * 4 + 256;
}

dsa_status dsa_indexer_project(const void* cq, const void* x, const void* Wq, const void* Wkw, const float* gamma,
                               const float* beta, int32_t n_tokens, int32_t q_rank, int32_t hidden, void* q_out,
                               void* k_out, float* w_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_tokens < 0) return fail(DSA_ERR_INVALID_ARG, "n_tokens < 0");
  if (q_rank < 64 || q_rank % 64 || hidden < 64 || hidden % 64)
    return fail(DSA_ERR_UNSUPPORTED, "q_rank %d / hidden %d must be positive multiples of 64", q_rank, hidden);
  if (n_tokens == 0) return DSA_OK;
  const void* ptrs[] = {cq, x, Wq, Wkw, gamma, beta, q_out, k_out, w_out, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  if (workspace_bytes < dsa_indexer_project_workspace_bytes(n_tokens))
    return fail(DSA_ERR_WORKSPACE, "indexer projection needs %zu workspace bytes",
                dsa_indexer_project_workspace_bytes(n_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* kw = static_cast<float*>(workspace);
  DSA_TRY(launch_gemm(cq, Wq, n_tokens, 4096, q_rank, q_out, 4096, true, st));
  DSA_TRY(launch_gemm(x, Wkw, n_tokens, 160, hidden, kw, 160, false, st));
  gemm::key_norm_kernel<<<static_cast<unsigned>((n_tokens + 7) / 8), 256, 0, st>>>(
      kw, n_tokens, gamma, beta, 1e-6f, static_cast<uint16_t*>(k_out), w_out);
  count_launch();
  return cuda_check(cudaGetLastError(), "key norm launch");
}

size_t dsa_mla_latent_workspace_bytes(int32_t n_tokens) {
  return n_tokens <= 0 ? 0 : static_cast<size_t>(n_tokens) * 576 * 4 + 256;
}

dsa_status dsa_mla_latent(const void* x, const void* Wkv, const float* gamma, const int32_t* pos, int32_t n_tokens,
                          int32_t hidden, float theta, void* latent_out, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (n_tokens < 0) return fail(DSA_ERR_INVALID_ARG, "n_tokens < 0");
  if (hidden < 64 || hidden % 64) return fail(DSA_ERR_UNSUPPORTED, "hidden %d must be a positive multiple of 64", hidden);
  if (!(theta > 1.f)) return fail(DSA_ERR_INVALID_ARG, "theta must be > 1");
  if (n_tokens == 0) return DSA_OK;
  const void* ptrs[] = {x, Wkv, gamma, pos, latent_out, workspace};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  if (workspace_bytes < dsa_mla_latent_workspace_bytes(n_tokens))
    return fail(DSA_ERR_WORKSPACE, "latent projection needs %zu workspace bytes", dsa_mla_latent_workspace_bytes(n_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* y = static_cast<float*>(workspace);
  DSA_TRY(launch_gemm(x, Wkv, n_tokens, 576, hidden, y, 576, false, st));
  gemm::latent_norm_rope_kernel<<<static_cast<unsigned>((n_tokens + 7) / 8), 256, 0, st>>>(
      y, n_tokens, gamma, pos, 1e-6f, static_cast<double>(theta), static_cast<uint16_t*>(latent_out));
  count_launch();
  return cuda_check(cudaGetLastError(), "latent norm / rope launch");
}

dsa_status dsa_rope_query(void* q, const int32_t* pos, int32_t n_q, float theta, void* stream) {
  if (n_q < 0) return fail(DSA_ERR_INVALID_ARG, "n_q < 0");
  if (!(theta > 1.f)) return fail(DSA_ERR_INVALID_ARG, "theta must be > 1");
  if (n_q == 0) return DSA_OK;
  if (!q || !aligned16(q) || !pos) return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  gemm::rope_query_kernel<<<static_cast<unsigned>(n_q), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint16_t*>(q), n_q, pos, static_cast<double>(theta));
  count_launch();
  return cuda_check(cudaGetLastError(), "query rope launch");
}

dsa_status dsa_split_candidates(const float* scores, int64_t ld, int32_t n_rows, const int32_t* idx_local, int32_t k,
                                int32_t n_local, int32_t offset, float* cand_score, int32_t* cand_idx, void* stream) {
  if (k < 1 || k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", k);
  if (n_rows < 0 || n_local < 0 || offset < 0 || ld <= 0) return fail(DSA_ERR_INVALID_ARG, "bad sizes");
  if (static_cast<int64_t>(offset) + n_local > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "positions beyond int32");
  if (n_rows == 0) return DSA_OK;
  if (!scores || !idx_local || !cand_score || !cand_idx) return fail(DSA_ERR_INVALID_ARG, "null pointer");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  splitn::split_candidates_kernel<<<static_cast<unsigned>(n_rows), 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      scores, ld, idx_local, k, offset, n_local, cand_score, cand_idx, ds->status);
  count_launch();
  return cuda_check(cudaGetLastError(), "split candidates launch");
}

size_t dsa_split_merge_workspace_bytes(int32_t n_rows, int32_t n_cand, int32_t k) {
  return dsa_topk_workspace_bytes(n_rows, n_cand, k);
}

dsa_status dsa_split_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_rows, int32_t n_cand, int32_t k,
                           int32_t lo, int32_t hi, int32_t* idx_global, int32_t* idx_local, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (k < 1 || k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", k);
  if (n_rows < 0 || n_cand < 1 || n_cand % 4 || lo < 0 || hi < lo)
    return fail(DSA_ERR_INVALID_ARG, "bad sizes (n_cand must be a positive multiple of 4)");
  if (n_rows == 0) return DSA_OK;
  if (!cand_score || !aligned16(cand_score) || !cand_idx || !idx_global || !aligned16(idx_global) || !idx_local)
    return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // positions of the k best candidates of each row (every row holds n_cand: row length
  // causal_len0 + r capped at n_cand), written into idx_global, then mapped in place
  DSA_TRY(launch_topk(cand_score, n_cand, n_rows, nullptr, n_cand, n_cand, k, idx_global, workspace, workspace_bytes,
                      st));
  const int64_t total = static_cast<int64_t>(n_rows) * k;
  splitn::split_map_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(cand_idx, n_cand, k, n_rows,
                                                                                    idx_global, idx_local, lo, hi);
  count_launch();
  return cuda_check(cudaGetLastError(), "split map launch");
}

dsa_status dsa_combine_partials(const void* o_parts, const float* lse_parts, int32_t n_parts, int32_t n_q, void* out,
                                float* lse, void* stream) {
  if (n_parts < 1 || n_q < 0) return fail(DSA_ERR_INVALID_ARG, "bad sizes");
  if (n_q == 0) return DSA_OK;
  if (!o_parts || !aligned16(o_parts) || !lse_parts || !out || !aligned16(out))
    return fail(DSA_ERR_INVALID_ARG, "null or misaligned pointer");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  splitn::combine_parts_kernel<<<dim3(static_cast<unsigned>(n_q), 64), 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(o_parts), lse_parts, n_parts, n_q, static_cast<uint16_t*>(out), lse);
  count_launch();
  return cuda_check(cudaGetLastError(), "combine launch");
}

size_t dsa_topk_workspace_bytes(int32_t n_rows, int64_t max_len, int32_t k) {
  DeviceState* ds = nullptr;
  if (device_state(&ds) != DSA_OK) return 0;
  return plan_topk(n_rows, max_len, k, ds->sms).ws;
}

dsa_status dsa_topk(const float* scores, int64_t ld, int32_t n_rows, const int32_t* row_len, int64_t causal_len0,
                    int64_t max_len, int32_t k, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                    void* stream) {
  if (k < 1 || k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", k);
  if (n_rows < 0 || ld <= 0 || ld % 4 || max_len < 0 || ld > INT32_MAX)
    return fail(DSA_ERR_INVALID_ARG, "bad n_rows / ld / max_len");
  if (n_rows == 0) return DSA_OK;
  if (!scores || !aligned16(scores) || !idx_out || !aligned16(idx_out))
    return fail(DSA_ERR_INVALID_ARG, "scores / idx_out null or misaligned");
  if (!row_len && causal_len0 < 0) return fail(DSA_ERR_INVALID_ARG, "causal_len0 < 0");
  return launch_topk(scores, ld, n_rows, row_len, causal_len0, max_len, k, idx_out, workspace, workspace_bytes,
                     static_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_mla_workspace_bytes(int32_t n_q, int32_t k, const dsa_cache_view* kv) {
  (void)kv;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != DSA_OK) return 0;
  return mla_ws_bytes(n_q, k, ds->sms);
}

dsa_status dsa_sparse_mla_attn(const void* q, const dsa_cache_view* kv, const int32_t* idx, int32_t n_q,
                               int32_t q_rows_per_idx_row, int32_t k, float softmax_scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream) {
  DSA_TRY(check_view(kv, 576, "kv"));
  if (k < 1 || k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", k);
  if (n_q < 0 || q_rows_per_idx_row < 1 || n_q % q_rows_per_idx_row)
    return fail(DSA_ERR_INVALID_ARG, "n_q must be a non-negative multiple of q_rows_per_idx_row");
  if (n_q == 0) return DSA_OK;
  if (!q || !aligned16(q) || !idx || !aligned16(idx) || !out || !aligned16(out))
    return fail(DSA_ERR_INVALID_ARG, "q / idx / out null or misaligned");
  if (lse && !aligned16(lse)) return fail(DSA_ERR_INVALID_ARG, "lse misaligned");
  if (!(softmax_scale > 0.f)) return fail(DSA_ERR_INVALID_ARG, "softmax_scale must be > 0");
  if (kv->block_table) {
    if (kv->batch != n_q / q_rows_per_idx_row)
      return fail(DSA_ERR_INVALID_ARG, "paged kv: batch != n_q / q_rows_per_idx_row");
  } else if (kv->dtype != DSA_BF16) {
    return fail(DSA_ERR_UNSUPPORTED, "dense latent caches must be bf16");
  }
  return launch_mla(q, kv, idx, n_q, q_rows_per_idx_row, k, softmax_scale, out, lse, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream));
}

size_t dsa_group_workspace_bytes(const dsa_group_args* a) {
  if (check_group(a) != DSA_OK) return 0;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != DSA_OK) return 0;
  GroupPlan g;
  plan_group(a, ds->sms, &g);
  return g.total;
}

dsa_status indexshare_group_forward(const dsa_group_args* a, dsa_index_handle* h, int32_t reuse_only,
                                    void* stream) {
  DSA_TRY(check_group(a));
  if (!h || !h->idx || !aligned16(h->idx)) return fail(DSA_ERR_INVALID_ARG, "null handle or handle buffer");
  if (h->rows != a->n_idx_rows || h->k != a->k) {
    if (reuse_only)
      return fail(DSA_ERR_STALE_HANDLE, "handle holds %d x %d indices, call needs %d x %d", h->rows, h->k,
                  a->n_idx_rows, a->k);
    return fail(DSA_ERR_INVALID_ARG, "handle buffer is %d x %d, call needs %d x %d", h->rows, h->k, a->n_idx_rows,
                a->k);
  }
  if (reuse_only && !h->filled) return fail(DSA_ERR_STALE_HANDLE, "reuse of an unfilled index handle");
  // A fill invalidates the handle before anything can write h->idx; only a fill that enqueues
  // every one of its launches marks it filled again, so a fill that fails part-way leaves no mix
  // of old and new indices for a later reuse call to accept.
  if (!reuse_only) h->filled = 0;
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  GroupPlan g;
  DSA_TRY(plan_group(a, ds->sms, &g));
  if (g.total > 0 && (!a->workspace || a->workspace_bytes < g.total))
    return fail(DSA_ERR_WORKSPACE, "group needs %zu workspace bytes, got %zu", g.total, a->workspace_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  const int32_t n = a->n_idx_rows;
  void** ev = a->trace_events;
  trace(ev, 0, st);
  if (!reuse_only && n > 0) {
    // a1: FP8 prep
    const void* qi = a->q_idx;
    const float* qs = nullptr;
    dsa_cache_view keys = a->idx_keys;
    if (g.quant_q) {
      DSA_TRY(dsa_quant_e4m3(a->q_idx, static_cast<int64_t>(n) * 32, 128, ws + g.off_q8,
                             reinterpret_cast<float*>(ws + g.off_sq), st));
      qi = ws + g.off_q8;
      qs = reinterpret_cast<const float*>(ws + g.off_sq);
    }
    if (g.quant_k) {
      if (keys.row_stride != 128) return fail(DSA_ERR_UNSUPPORTED, "bf16 keys to quantise must be contiguous");
      DSA_TRY(dsa_quant_e4m3(keys.data, keys.n_tokens, 128, ws + g.off_k8,
                             reinterpret_cast<float*>(ws + g.off_sk), st));
      keys.data = ws + g.off_k8;
      keys.scale = reinterpret_cast<const float*>(ws + g.off_sk);
      keys.dtype = DSA_E4M3;
      keys.row_stride = 128;
    }
    const int32_t qdt = g.quant_q ? DSA_E4M3 : DSA_BF16;
    float* scores = reinterpret_cast<float*>(ws + g.off_scores);
    const bool paged = keys.block_table != nullptr;
    const size_t qrow_bytes = qdt == DSA_E4M3 ? 32 * 128 : 32 * 128 * 2;
    for (const Chunk& ch : g.chunks) {
      const int32_t c0 = ch.row0, cn = ch.rows;
      const uint8_t* qc = static_cast<const uint8_t*>(qi) + static_cast<size_t>(c0) * qrow_bytes;
      const float* qsc = qs ? qs + static_cast<size_t>(c0) * 32 : nullptr;
      // paged rows with a segmented Top-k: the indexer's epilogue builds the first-digit
      // histograms, so the Top-k skips that pass over the scores
      const TopkPlan tp = plan_topk(cn, std::min<int64_t>(ch.ld, ch.max_len), a->k, ds->sms);
      const bool fused_hist = paged && tp.segmented;
      if (fused_hist)
        DSA_TRY(cuda_check(cudaMemsetAsync(ws + g.off_topk, 0, static_cast<size_t>(cn) * (topk::BINS * 4 + 16), st),
                           "topk workspace clear"));
      DSA_TRY(launch_indexer(qc, qdt, qsc, a->w + static_cast<size_t>(c0) * 32, cn, a->q_pos0 + c0, &keys, scores,
                             ch.ld, st, fused_hist ? reinterpret_cast<uint32_t*>(ws + g.off_topk) : nullptr));
      DSA_TRY(launch_topk(scores, ch.ld, cn, paged ? keys.seq_lens : nullptr,
                          static_cast<int64_t>(a->q_pos0) + c0 + 1, ch.max_len, a->k,
                          h->idx + static_cast<size_t>(c0) * a->k, ws + g.off_topk, g.topk_ws, st, fused_hist));
    }
    h->generation += 1;
    h->filled = 1;
    h->producer_layer = a->first_layer;
  }
  trace(ev, 1, st);
  const int32_t nq = n * a->q_rows_per_idx_row;
  // indices computed by this call for a dense causal prefill: row i holds its min(k, q_pos0 + i + 1)
  // valid entries first, so the attention skips the tiles past them
  const int64_t valid0 = (!reuse_only && !a->idx_keys.block_table) ? static_cast<int64_t>(a->q_pos0) + 1 : -1;
  // paged layers' query rows to f16 in one launch, when the attention cuts every row over many CTAs
  // (inside layer 0's trace window: it is attention work)
  const void* q16[DSA_GROUP_MAX_LAYERS] = {};
  trace(ev, 2, st);
  if (g.q16_layer_bytes > 0 && nq > 0) {
    mla::QConvert qc{};
    int y = 0;
    for (int l = 0; l < a->n_layers; ++l) {
      if (!a->kv[l].block_table) continue;
      qc.src[y] = static_cast<const uint4*>(a->q[l]);
      qc.dst[y] = reinterpret_cast<uint4*>(ws + g.off_q16 + y * g.q16_layer_bytes);
      q16[l] = qc.dst[y];
      ++y;
    }
    const int64_t chunks = static_cast<int64_t>(nq) * 64 * 576 / 8;
    const unsigned gx = static_cast<unsigned>(std::min<int64_t>((chunks + 255) / 256, 2LL * ds->sms));
    launch_pdl(mla::q_to_f16_kernel, dim3(gx, static_cast<unsigned>(y)), 256, 0, st, qc, chunks, ds->status);
    count_launch();
    DSA_TRY(cuda_check(cudaGetLastError(), "query f16 launch"));
  }
  for (int l = 0; l < a->n_layers; ++l) {
    if (l > 0) trace(ev, 2 + 2 * l, st);
    DSA_TRY(launch_mla(a->q[l], &a->kv[l], h->idx, nq, a->q_rows_per_idx_row, a->k, a->softmax_scale, a->out[l],
                       a->lse[l], ws + g.off_mla, g.total - g.off_mla, st, valid0, q16[l]));
    trace(ev, 3 + 2 * l, st);
  }
  return DSA_OK;
}

}  // extern "C"

// ================================================================ Top-k without caller scratch
// The segmented Top-k with its scratch in a fixed device array of this file, for callers that
// cannot allocate device memory (see dsa_topk_no_alloc in include/dsa.h).

namespace dsa {
namespace {

constexpr int32_t kNoAllocGcap = 16384;
constexpr size_t kNoAllocRowHead = static_cast<size_t>(topk::BINS) * 4 + 16;
static_assert(DSA_TOPK_NO_ALLOC_SCRATCH_BYTES ==
                  DSA_TOPK_NO_ALLOC_MAX_ROWS * (kNoAllocRowHead + static_cast<size_t>(kNoAllocGcap) * 8),
              "scratch size and layout disagree");
static_assert(kNoAllocGcap >= topk::CAND_CAP, "global candidate capacity below the shared one");

// Host code must not use this name as a device address: it is looked up per device below.
static __device__ __align__(256) uint8_t g_topk_scratch[DSA_TOPK_NO_ALLOC_SCRATCH_BYTES];

uint8_t* g_topk_scratch_addr[64] = {};
std::mutex g_topk_scratch_mu;

// Once per device, with that device current: the array's device address.
dsa_status topk_scratch_address(uint8_t** out) {
  int dev = 0;
  DSA_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= 64) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_topk_scratch_mu);
  if (!g_topk_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess || !p) return cuda_check(e, "cudaGetSymbolAddress(top-k scratch)");
    g_topk_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_topk_scratch_addr[dev];
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_topk_no_alloc(const float* scores, int64_t ld, int32_t n_rows, const int32_t* row_len,
                                        int64_t causal_len0, int64_t max_len, int32_t k, int32_t* idx_out,
                                        void* stream) {
  if (k < 1 || k > DSA_MAX_K) return fail(DSA_ERR_INVALID_ARG, "k %d not in [1,2048]", k);
  if (n_rows < 0 || ld <= 0 || ld % 4 || max_len < 0 || ld > INT32_MAX)
    return fail(DSA_ERR_INVALID_ARG, "bad n_rows / ld / max_len");
  if (n_rows > DSA_TOPK_NO_ALLOC_MAX_ROWS)
    return fail(DSA_ERR_INVALID_ARG,
                "dsa_topk_no_alloc takes at most %d rows (fixed scratch of %u bytes), got %d; "
                "use dsa_topk with a workspace",
                DSA_TOPK_NO_ALLOC_MAX_ROWS, DSA_TOPK_NO_ALLOC_SCRATCH_BYTES, n_rows);
  if (n_rows == 0) return DSA_OK;
  if (!scores || !aligned16(scores) || !idx_out || !aligned16(idx_out))
    return fail(DSA_ERR_INVALID_ARG, "scores / idx_out null or misaligned");
  if (!row_len && causal_len0 < 0) return fail(DSA_ERR_INVALID_ARG, "causal_len0 < 0");
  DeviceState* ds = nullptr;
  DSA_TRY(device_state(&ds));
  uint8_t* scratch = nullptr;
  DSA_TRY(topk_scratch_address(&scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t cap = std::min(ld, max_len);
  const int64_t by_len = std::max<int64_t>(1, (cap + 8191) / 8192);
  const int64_t segs = std::max<int64_t>(1, std::min<int64_t>((4LL * ds->sms + n_rows - 1) / n_rows, by_len));
  const int32_t seg_len = static_cast<int32_t>(std::max<int64_t>(4, align_up(static_cast<size_t>((cap + segs - 1) / segs), 4)));
  topk::SegWs sw;
  sw.hist = reinterpret_cast<uint32_t*>(scratch);
  sw.counters = reinterpret_cast<int32_t*>(scratch + static_cast<size_t>(n_rows) * topk::BINS * 4);
  const size_t head = static_cast<size_t>(n_rows) * kNoAllocRowHead;
  sw.cand_key = reinterpret_cast<uint32_t*>(scratch + head);
  sw.cand_idx = reinterpret_cast<int32_t*>(scratch + head + static_cast<size_t>(n_rows) * kNoAllocGcap * 4);
  sw.gcap = kNoAllocGcap;
  // the histograms and counters of the previous call must not leak into this one
  DSA_TRY(cuda_check(cudaMemsetAsync(scratch, 0, head, st), "clear top-k scratch"));
  dim3 grid(static_cast<unsigned>(segs), static_cast<unsigned>(n_rows));
  launch_pdl(topk::topk_seg_hist_kernel, grid, topk::SEG_THREADS, 0, st, scores, ld, row_len, causal_len0, cap, k, seg_len,
                                                                 sw);
  launch_pdl(topk::topk_seg_filter_kernel, grid, topk::SEG_THREADS, 0, st, scores, ld, row_len, causal_len0, cap, k,
                                                                   seg_len, sw, idx_out);
  count_launch(2);
  return cuda_check(cudaGetLastError(), "no-alloc top-k launch");
}

/*
 * dsa.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention step with IndexShare.
 *
 * The operation, as the GLM-5.2 pages state it:
 *   - "Z.ai / 智谱 GLM-5.2 怎样让百万上下文真正跑起来" (ailearn.mscapital.top), section
 *     "一枚 Token，怎样穿过 78 层": MLA compresses the per-token KV; the indexer first scans
 *     the history and core attention reads only the Top-2,048 tokens; 64 attention heads,
 *     32 indexer heads, KV rank 512.
 *   - same page, section "IndexShare：四层共用一次搜索结果": Full layers compute the Top-k,
 *     the following 3 Shared layers reuse it (21 Full / 57 Shared of 78 layers).
 *   - same page, MTP section, and forum.sourcefind.cn "MTP推测解码改进": the first draft
 *     step computes the Top-k, later steps reuse it and the first step's KV (KV Share).
 *   - forum.sourcefind.cn "IndexShare：省掉3/4的索引计算": the lightweight indexer picks the
 *     top-k tokens per query, taking core attention from O(L^2) to O(Lk).
 * The pages give no formula; the readings used (ReLU-weighted head sum, causal set
 * including the query, 576 = 512 latent + 64 RoPE dims, per-token e4m3 scales) are
 * stated at each call below.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers (CUDA global memory) owned by the caller;
 *     the library never allocates, frees or retains device memory.  Scratch space is a
 *     caller-provided workspace whose size the *_workspace_bytes() calls return.
 *   - `stream` is a cudaStream_t (may be NULL = legacy default stream).  Every call only
 *     enqueues work and returns; results are ready when the stream reaches that point.
 *     The kernels of the indexer, Top-k, sparse MLA, quantisation and cache-write calls are
 *     launched with programmatic dependent launch: each may be launched before the previous
 *     work of the stream has finished, but waits for it before touching memory, so stream
 *     order holds as for plain launches (also inside a captured CUDA graph).  Setting
 *     DSA_PDL=0 in the environment before the first call launches them plainly.
 *   - Arguments are validated on the host before anything is launched; a failing check
 *     returns DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED and launches nothing.  The text
 *     of the last failure on the calling thread is returned by dsa_last_error().
 *   - Device pointers must be 16-byte aligned; row strides must be multiples of 16 bytes.
 *   - Device-side waits are bounded; a wait that runs out sets a device status word that
 *     dsa_sync_status() returns as DSA_ERR_TIMEOUT (the kernel exits instead of hanging).
 *   - bf16 tensors are passed as raw 16-bit patterns, e4m3 tensors as raw bytes (OCP e4m3fn).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 1
#define DSA_IDX_HEADS 32   /* indexer heads                         */
#define DSA_IDX_DIM 128    /* indexer head / key dims                */
#define DSA_HEADS 64       /* MLA query heads                        */
#define DSA_DQK 576        /* latent key width: 512 latent + 64 RoPE */
#define DSA_DV 512         /* latent value width                     */
#define DSA_PAGE 64        /* tokens per cache page                  */
#define DSA_MAX_K 2048     /* largest Top-k                          */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or stride            */
  DSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented combination (dtype, dims)      */
  DSA_ERR_STALE_HANDLE = 3, /* reuse of an index handle that is unfilled or mismatched  */
  DSA_ERR_TIMEOUT = 4,      /* a bounded device wait ran out (see dsa_sync_status)      */
  DSA_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed              */
  DSA_ERR_WORKSPACE = 6,    /* workspace missing or smaller than *_workspace_bytes()    */
  DSA_ERR_BOUNDS = 7,       /* a kernel met an out-of-range index or page and skipped it */
  DSA_ERR_RANGE = 8         /* an input value lies outside the range a kernel supports   */
} dsa_status;

typedef enum { DSA_BF16 = 0, DSA_E4M3 = 1 } dsa_dtype;

/*
 * A token-major cache (indexer keys: dim 128; latent KV: dim 576), dense or paged.
 *   dense  (block_table == NULL): data [n_tokens, row_stride] elements, token t at row t;
 *          e4m3 scale [n_tokens] fp32 (value = code * scale[t]).
 *   paged  (block_table != NULL): data [n_pages, 64, dim] (row_stride must equal dim),
 *          scale [n_pages, 64]; sequence b's token s lives in physical page
 *          block_table[b * max_pages + s / 64], slot s % 64; seq_lens[b] = tokens of b.
 *          n_tokens = n_pages * 64 (used for bounds checks of page ids).
 * bf16 caches have scale == NULL.  Paged caches are e4m3 only.
 */
typedef struct {
  const void* data;
  const float* scale;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int64_t row_stride;
  int64_t n_tokens;
  int32_t dim;
  int32_t dtype;     /* dsa_dtype */
  int32_t max_pages; /* paged: columns of block_table */
  int32_t batch;     /* paged: sequences (rows of block_table) */
} dsa_cache_view;

/*
 * Index-reuse handle: the Top-k of one Full layer, handed to the Shared layers that
 * follow it and to later MTP draft steps (page sections cited above).
 * idx: caller-owned device buffer [rows, k] int32 (row order within a row unspecified,
 * -1 = padding).  generation is bumped by every call that fills it; filled = 1 after.  A
 * filling call sets filled = 0 before it launches anything and back to 1 only once all of
 * its launches are enqueued, so a fill that fails leaves the handle unfilled.
 */
typedef struct {
  int32_t* idx;
  int32_t rows;
  int32_t k;
  int32_t filled;
  int32_t producer_layer;
  int64_t generation;
} dsa_index_handle;

/* ---------------------------------------------------------------------------------------
 * Step a1: per-vector FP8 e4m3 quantisation (FP8 indexer path; the pages state FP8 KV
 * cache support, "推理优化" on the wiki-for-amaranth page and the vLLM launch flag
 * fp8_ds_mla on forum.sourcefind.cn; the scale rule is this library's reading):
 *   scale[v] = amax(|x[v,:]|) / 448 (1 if amax == 0), codes = RNE_saturate(x / scale), all fp32.
 * x_bf16 [n_vec, vec_len] bf16 -> codes [n_vec, vec_len] uint8, scale [n_vec] fp32.
 * vec_len must be 128.
 */
dsa_status dsa_quant_e4m3(const void* x_bf16, int64_t n_vec, int32_t vec_len, uint8_t* codes, float* scale,
                          void* stream);

/* ---------------------------------------------------------------------------------------
 * Step a1 on the decode side: append new tokens to a paged FP8 cache (the FP8 KV cache of the
 * pages cited at dsa_quant_e4m3; the 64-token page is this library's choice, as for the paged
 * dsa_cache_view, since the pages give no block size).  Same pages and format as that view:
 * e4m3 codes [n_pages, 64, dim] + fp32 scales [n_pages, 64], one scale per token, rule as in
 * dsa_quant_e4m3 over the token's whole row.  Ownership: the caller owns every buffer; the call
 * writes only the rows' slots of pool and pool_scale, asynchronously on the stream.
 *   x_bf16      [n_rows, dim] bf16, dim 128 (indexer keys) or 576 (latent rows); 16-byte aligned
 *   seq         [n_rows] int32 sequence of each row, or NULL for row r -> sequence r
 *   pos         [n_rows] int32 position of each row in its sequence
 *   block_table [batch, max_pages] int32: slot of (b, t) = page block_table[b][t / 64], entry t % 64
 *   pool        [n_pages, 64, dim] uint8 (16-byte aligned), pool_scale [n_pages, 64] fp32: written
 *               at the rows' slots only
 * Each (sequence, position) may appear at most once per call.  Host-side errors: null or
 * misaligned pointers, dim not 128 / 576, negative sizes.  A row whose sequence, position or page
 * is out of range is skipped on the device and reported as DSA_ERR_BOUNDS by dsa_sync_status.
 */
dsa_status dsa_cache_write_e4m3(const void* x_bf16, int32_t n_rows, int32_t dim, const int32_t* seq,
                                const int32_t* pos, const int32_t* block_table, int32_t batch, int32_t max_pages,
                                int32_t n_pages, uint8_t* pool, float* pool_scale, void* stream);

/* The same write into several pools in one launch (a decode step appends its current token to
 * every layer's latent pool and every Full layer's key pool).  x_bf16, dims, pools and
 * pool_scales are HOST arrays of n_pools entries (device pointers inside; dims 128 or 576); all
 * pools share seq, pos, block_table, batch, max_pages and n_pages.  n_pools <= 128.  Errors as
 * above, per pool.
 */
#define DSA_CACHE_WRITE_MAX_POOLS 128
dsa_status dsa_cache_write_e4m3_pools(int32_t n_pools, const void* const* x_bf16, const int32_t* dims,
                                      uint8_t* const* pools, float* const* pool_scales, int32_t n_rows,
                                      const int32_t* seq, const int32_t* pos, const int32_t* block_table, int32_t batch,
                                      int32_t max_pages, int32_t n_pages, void* stream);

/* ---------------------------------------------------------------------------------------
 * Steps a2+a3: lightweight-indexer scores (forum.sourcefind.cn "IndexShare：省掉3/4的索引计算";
 * 32 heads, ailearn architecture card), with the ReLU, per-head weight and causal mask
 * fused into the tensor-core epilogue:
 *   I[r, s] = sk[s] * sum_h (w[r,h] * sq[r,h]) * max(0, q[r,h,:] . k[s,:])
 * (sk = sq = 1 for bf16).
 *   q        [n_q, 32, 128] bf16 or e4m3 (q_dtype must equal keys->dtype)
 *   q_scale  [n_q, 32] fp32 for e4m3, NULL for bf16
 *   w        [n_q, 32] fp32
 *   keys     dim 128.  Dense: query row r sits at position q_pos0 + r and its candidates
 *            are s in [0, min(q_pos0 + r + 1, n_tokens)).  Paged: row r is sequence r
 *            (n_q == keys->batch) and its candidates are s in [0, seq_lens[r]).
 *   scores   [n_q, ld_scores] fp32; entries [0, len_r) of row r are written, the rest of
 *            the row is left untouched.  ld_scores >= the longest row, multiple of 4.
 */
dsa_status dsa_indexer_score(const void* q, int32_t q_dtype, const float* q_scale, const float* w, int32_t n_q,
                             int32_t q_pos0, const dsa_cache_view* keys, float* scores, int64_t ld_scores,
                             void* stream);

/* ---------------------------------------------------------------------------------------
 * Step a4: per-row Top-k (ailearn "一枚 Token，怎样穿过 78 层": core attention reads only the
 * Top-2,048).  Row r holds len_r candidates scores[r, 0 .. len_r): len_r = row_len[r]
 * (device array) when row_len != NULL, else min(causal_len0 + r, ld).  Writes
 * idx_out [n_rows, k]: the positions of the k largest scores (ties: lower position wins),
 * in unspecified order, padded with -1 when len_r < k.  1 <= k <= 2048.
 * workspace: device scratch of at least dsa_topk_workspace_bytes(n_rows, max_len, k)
 * bytes (may be 0 bytes, then workspace may be NULL).
 */
size_t dsa_topk_workspace_bytes(int32_t n_rows, int64_t max_len, int32_t k);
dsa_status dsa_topk(const float* scores, int64_t ld, int32_t n_rows, const int32_t* row_len, int64_t causal_len0,
                    int64_t max_len, int32_t k, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                    void* stream);

/* ---------------------------------------------------------------------------------------
 * Step a6: sparse MLA attention over the selected latent rows (ailearn architecture card:
 * 64 heads, KV rank 512; absorbed form with a 576-wide key = 512 latent + 64 RoPE dims and
 * the first 512 dims as value):
 *   z[h,j] = softmax_scale * q[r,h,:] . kv[idx_j, :576];  p = softmax_j(z);
 *   out[r,h,:] = sum_j p[h,j] kv[idx_j, :512];  lse[r,h] = log sum_j exp(z[h,j]).
 *   q    [n_q, 64, 576] bf16;  out [n_q, 64, 512] bf16;  lse [n_q, 64] fp32 or NULL.
 *   idx  [n_q / q_rows_per_idx_row, k] int32; query row r uses idx row r / q_rows_per_idx_row
 *        (MTP rows sharing row 0's selection).  -1 entries are skipped.
 *   kv   dim 576.  Dense bf16: idx values are token rows of kv.  Paged e4m3: idx row i is
 *        sequence i and its values are token positions s < seq_lens[i].
 *   A row with no valid index gets out = 0 and lse = -inf.
 *   Paged e4m3 caches: the products run on f16 operands (e4m3 values are exact in f16), so q is
 *   converted from bf16 to f16 and must lie within the f16 range, |q| < 65520; a larger value
 *   would become infinite and is reported as DSA_ERR_RANGE by dsa_sync_status (that row's output
 *   is then undefined).  Values below 2^-14 keep f16's subnormal precision (absolute error at most
 *   2^-25).  Dense bf16 caches take any finite bf16 q.
 * workspace: dsa_sparse_mla_workspace_bytes(...) bytes (split-KV partials for few rows).
 */
size_t dsa_sparse_mla_workspace_bytes(int32_t n_q, int32_t k, const dsa_cache_view* kv);
dsa_status dsa_sparse_mla_attn(const void* q, const dsa_cache_view* kv, const int32_t* idx, int32_t n_q,
                               int32_t q_rows_per_idx_row, int32_t k, float softmax_scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * One IndexShare group: a Full layer followed by up to 3 Shared layers (ailearn
 * "IndexShare：四层共用一次搜索结果").  Unless reuse_only, the Full layer runs a1 (when
 * indexer_dtype is e4m3 and the inputs are bf16), a2-a4 into h->idx and bumps the handle;
 * then every layer l < n_layers runs a6 with its own q[l]/kv[l] and the handle's indices.
 * reuse_only = 1 skips a1-a4 and requires a filled handle of matching rows and k
 * (DSA_ERR_STALE_HANDLE otherwise): Shared layers of a later call, MTP draft steps >= 2.
 *   q_idx  [n_idx_rows, 32, 128] bf16 (row i = prefill query row i, or decode sequence i)
 *   w      [n_idx_rows, 32] fp32
 *   idx_keys: dim 128 cache (bf16 dense; or e4m3 dense/paged with scales)
 *   indexer_dtype: DSA_BF16 (requires bf16 keys) or DSA_E4M3 (bf16 q is quantised; bf16
 *                  dense keys are quantised too)
 *   q_pos0: position of prefill query row 0 (ignored for paged caches)
 *   q_rows_per_idx_row: 1 in prefill, 1 + d in decode with d MTP draft rows
 *   q[l] [n_idx_rows * q_rows_per_idx_row, 64, 576] bf16, kv[l] dim 576, out[l], lse[l]
 *   workspace: at least dsa_group_workspace_bytes(a) bytes of device memory: e4m3 copies of
 *              the indexer inputs (when quantised here), the scores of one chunk of query rows
 *              (rows x causal length <= max(64 MB, 2,048 x longest row x 4 B), at most 1 GB),
 *              the Top-k scratch, the split-KV partials of the attention and, when paged
 *              layers cut every query row over many CTAs (few rows), the f16 copies of those
 *              layers' q (converted once per call instead of once per CTA).
 * The call allocates nothing and only enqueues kernels and memsets on `stream`, so once a
 * first call has set the device up it may be captured into a CUDA graph and replayed.
 */
#define DSA_GROUP_MAX_LAYERS 4
typedef struct {
  const void* q_idx;
  const float* w;
  dsa_cache_view idx_keys;
  int32_t indexer_dtype;
  int32_t n_idx_rows;
  int32_t q_pos0;
  int32_t k;
  int32_t q_rows_per_idx_row;
  int32_t n_layers;
  int32_t first_layer;
  float softmax_scale;
  const void* q[DSA_GROUP_MAX_LAYERS];
  dsa_cache_view kv[DSA_GROUP_MAX_LAYERS];
  void* out[DSA_GROUP_MAX_LAYERS];
  float* lse[DSA_GROUP_MAX_LAYERS];
  void* workspace;
  size_t workspace_bytes;
  /* Optional tracing: NULL, or an array of 2 + 2 * n_layers cudaEvent_t created by the
   * caller.  Recorded on `stream` around the Full layer's a1-a4 phase (events 0, 1) and
   * around layer l's a6 launch (events 2 + 2l, 3 + 2l). */
  void** trace_events;
} dsa_group_args;

size_t dsa_group_workspace_bytes(const dsa_group_args* a);
dsa_status indexshare_group_forward(const dsa_group_args* a, dsa_index_handle* h, int32_t reuse_only,
                                    void* stream);

/* ---------------------------------------------------------------------------------------
 * Top-k for callers that cannot allocate device memory.  (The pages have no counterpart:
 * this is a deployment convenience of this library, not a step of the method.)
 *
 * Same selection and output as dsa_topk (same arguments minus the workspace), computed by
 * the multi-CTA segmented variant with its scratch in a fixed array inside the library
 * (DSA_TOPK_NO_ALLOC_SCRATCH_BYTES of device memory, held by every GPU that loads the
 * library until the process exits).  For callers whose device memory is wholly owned by
 * another allocator (e.g. an engine that reserves the whole KV pool up front) or that must
 * not call cudaMalloc / cudaFree, whose implicit device-wide synchronisation would stall
 * other streams.  Nothing is allocated on any call.
 *   - n_rows <= DSA_TOPK_NO_ALLOC_MAX_ROWS, else DSA_ERR_INVALID_ARG (no launch).
 *   - The first call on each device looks up the array's device address; make that first
 *     call before any stream capture.
 *   - All calls share the one array: calls that can overlap on the GPU (different streams,
 *     or different threads without ordering) race and must be serialised by the caller.
 *     Each call clears the parts that must start at zero.
 *   - Rows whose threshold bin holds more than 16,384 candidates take a slower path that
 *     re-reads the row; the result is the same.
 */
#define DSA_TOPK_NO_ALLOC_MAX_ROWS 32
#define DSA_TOPK_NO_ALLOC_SCRATCH_BYTES (32u * (4096u * 4u + 16u + 16384u * 8u))
dsa_status dsa_topk_no_alloc(const float* scores, int64_t ld, int32_t n_rows, const int32_t* row_len,
                             int64_t causal_len0, int64_t max_len, int32_t k, int32_t* idx_out, void* stream);

/* ---------------------------------------------------------------------------------------
 * The inputs of the indexer (the step before a2): its query from the query latent, its key and
 * per-head weights from the hidden state (ailearn "一枚 Token，怎样穿过 78 层": hidden size 6,144,
 * 32 indexer heads of 128; "IndexShare：四层共用一次搜索结果": 9,371,904 parameters per indexer,
 * which the shapes below reproduce with q_rank = 2,048 and hidden = 6,144; the LayerNorm on the
 * key and the rank of the query latent are this library's reading):
 *   q_out[t]  = cq[t] . Wq^T                             [T, 4096] = [T, 32, 128] bf16
 *   k_out[t]  = LayerNorm(x[t] . Wk^T) * gamma + beta    [T, 128] bf16 (eps 1e-6, biased variance)
 *   w_out[t]  = x[t] . Ww^T                              [T, 32] fp32
 *   cq   [T, q_rank] bf16;  x [T, hidden] bf16;  Wq [4096, q_rank] bf16 (row = output);
 *   Wkw  [160, hidden] bf16: rows 0..127 = Wk, rows 128..159 = Ww;  gamma, beta [128] fp32.
 *   q_rank and hidden: positive multiples of 64.  Products on the tensor cores (bf16 in, fp32
 *   accumulate).  workspace: dsa_indexer_project_workspace_bytes(T) bytes of device memory.
 */
size_t dsa_indexer_project_workspace_bytes(int32_t n_tokens);
dsa_status dsa_indexer_project(const void* cq, const void* x, const void* Wq, const void* Wkw, const float* gamma,
                               const float* beta, int32_t n_tokens, int32_t q_rank, int32_t hidden, void* q_out,
                               void* k_out, float* w_out, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * The latent KV rows that sparse MLA reads (ailearn architecture card: KV joint compression of
 * rank 512, RoPE with theta = 8,000,000 over 2^20 positions; the RMSNorm, the 64 RoPE dims and
 * the pairing of the rotation are this library's reading):
 *   latent_out[t] = [ RMSNorm(x[t] . W_dkv^T) * gamma  ||  RoPE(x[t] . W_kr^T, pos[t]) ]   [T, 576] bf16
 *   RMSNorm: v / sqrt(mean(v^2) + 1e-6).  RoPE: pair (2i, 2i + 1) of the 64 dims turned by the
 *   angle pos * theta^(-2i/64) (the angle is reduced in double precision).
 *   x [T, hidden] bf16;  Wkv [576, hidden] bf16: rows 0..511 = W_dkv, rows 512..575 = W_kr;
 *   gamma [512] fp32;  pos [T] int32 (>= 0).  workspace: dsa_mla_latent_workspace_bytes(T).
 * dsa_rope_query turns dims 512..575 of every head of q [T, 64, 576] bf16 in place, the same way,
 * to position pos[t], so that the RoPE part of a logit depends on the distance of the two tokens.
 */
size_t dsa_mla_latent_workspace_bytes(int32_t n_tokens);
dsa_status dsa_mla_latent(const void* x, const void* Wkv, const float* gamma, const int32_t* pos, int32_t n_tokens,
                          int32_t hidden, float theta, void* latent_out, void* workspace, size_t workspace_bytes,
                          void* stream);
dsa_status dsa_rope_query(void* q, const int32_t* pos, int32_t n_q, float theta, void* stream);

/* ---------------------------------------------------------------------------------------
 * Split-N decode of one long sequence over G GPUs (the pages' full 1M context starts at 8 B200s
 * with an FP8 KV cache, ailearn deployment section "CP · EP · P/D · HiCache"; the split itself is
 * this library's design).  Rank r holds the contiguous cache slice of positions [lo_r, hi_r) and
 * runs a2-a4 on it (dsa_indexer_score / dsa_topk over the slice, local positions); then:
 *   dsa_split_candidates: local Top-k idx_local [n_rows, k] of the slice's scores
 *     [n_rows, ld] -> cand_score / cand_idx [n_rows, k]: (score, lo_r + position) ordered by
 *     position, padding (-inf, -1) last.  Positions >= n_local are skipped (DSA_ERR_BOUNDS).
 *   (the caller gathers every rank's candidates, in rank order, into [n_rows, G * k])
 *   dsa_split_merge: the k best of the n_cand = G * k candidates of each row -> idx_global
 *     [n_rows, k] (the same on every rank, equal to the Top-k of the unsplit row: equal scores go
 *     to the lower position) and idx_local [n_rows, k] = idx_global - lo for positions in
 *     [lo, hi), else -1, for dsa_sparse_mla_attn over this rank's slice (with lse).
 *     n_cand a multiple of 4; workspace: dsa_split_merge_workspace_bytes(...).
 *   (the caller gathers every rank's out / lse into o_parts [G, n_q, 64, 512] bf16 and
 *   lse_parts [G, n_q, 64] fp32)
 *   dsa_combine_partials: lse = log sum_r exp(lse_r), out = sum_r exp(lse_r - lse) out_r
 *     [n_q, 64, 512] bf16; lse may be NULL.  A part with lse_r = -inf contributes nothing.
 */
dsa_status dsa_split_candidates(const float* scores, int64_t ld, int32_t n_rows, const int32_t* idx_local, int32_t k,
                                int32_t n_local, int32_t offset, float* cand_score, int32_t* cand_idx, void* stream);
size_t dsa_split_merge_workspace_bytes(int32_t n_rows, int32_t n_cand, int32_t k);
dsa_status dsa_split_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_rows, int32_t n_cand, int32_t k,
                           int32_t lo, int32_t hi, int32_t* idx_global, int32_t* idx_local, void* workspace,
                           size_t workspace_bytes, void* stream);
dsa_status dsa_combine_partials(const void* o_parts, const float* lse_parts, int32_t n_parts, int32_t n_q, void* out,
                                float* lse, void* stream);

/* ---------------------------------------------------------------------------------------
 * 78-layer schedule (ailearn "IndexShare：四层共用一次搜索结果"): Full at 0-based layers 0, 1
 * and 2 + 4g; every other layer reuses the closest preceding Full layer.
 */
int32_t dsa_layer_is_full(int32_t layer);
int32_t dsa_layer_producer(int32_t layer);

/* ---------------------------------------------------------------------------------------
 * Status / diagnostics.
 */
const char* dsa_status_str(dsa_status s);
const char* dsa_last_error(void);       /* thread-local text of the last failure; never NULL */
int32_t dsa_abi_version(void);
/* sizeof of the ABI structs as compiled into the library (0: dsa_cache_view,
 * 1: dsa_index_handle, 2: dsa_group_args), so bindings can check their own layout. */
size_t dsa_abi_sizeof(int32_t which);
/* Synchronise the stream, then read and clear the device status word of the current
 * device: DSA_ERR_TIMEOUT if a bounded wait ran out, DSA_ERR_BOUNDS if a kernel skipped an
 * out-of-range index/page, DSA_ERR_RANGE if an attention over an e4m3 cache met a query value
 * outside the f16 range, DSA_ERR_CUDA on a CUDA error, else DSA_OK. */
dsa_status dsa_sync_status(void* stream);
/* Test hook: launch one CTA that waits on an mbarrier nothing will complete, bounded by
 * timeout_ns; the kernel then records DSA_ERR_TIMEOUT in the status word and exits. */
dsa_status dsa_debug_bounded_wait(int64_t timeout_ns, void* stream);
/* Number of kernels this library has launched in this process (all devices). */
int64_t dsa_launch_count(void);
/* Device-side wait limit used by all kernels (default 2 s); returns the previous value. */
int64_t dsa_set_wait_limit_ns(int64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */

"""fp64 oracle of one DSA + IndexShare step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or call this module; the CUDA library never does.

Sources, cited by page title and section:

* [wiki]    "GLM-5.2 — 1M上下文开放权重的长程任务旗舰" (wiki-for-amaranth.pages.dev),
            sections "注意力机制：DSA + IndexShare" and "推理优化".
* [ailearn] "Z.ai / 智谱 GLM-5.2 怎样让百万上下文真正跑起来" (ailearn.mscapital.top),
            sections "一枚 Token，怎样穿过 78 层" (architecture card),
            "IndexShare：四层共用一次搜索结果" and "MTP：同一位速记员，多猜几枚未来 Token".
* [forum]   forum.sourcefind.cn thread on GLM-5.2 (DCU deployment), sub-headings
            "IndexShare：省掉3/4的索引计算", "MTP推测解码改进", "vLLM推理启动".
* [context] "GLM-5.2 权重落地：开放阵营把前沿压成了按季度刷新的常态" (the-context.pages.dev),
            section "技术要点".

The pages print no formula.  Where they are silent this file takes the plainest
reading, listed once here and used consistently:

R1  Indexer score: I[t,s] = sum_h w[t,h] * max(0, q[t,h,:] . k[s,:]) over 32 heads of 128
    dims (a lightweight indexer that scores each history token per query, [forum]
    "IndexShare：省掉3/4的索引计算"; 32 indexer heads, [ailearn] architecture card).  No
    global constant: a positive constant leaves the Top-k unchanged.  The pages print no
    formula and no value for it, so indexer_scores is parity unpinned by the pages: its
    tests pin it to this definition (closed forms on unit vectors, invariances), not to a
    printed number.
R2  Causal candidates include the query itself: s <= t (prefill); s < N_b in decode,
    where N_b counts the current token.
R3  Top-k keeps the k largest scores; equal scores go to the lower index; with fewer than
    k candidates all are kept and the row is padded with -1.
R4  Sparse MLA in the absorbed form: one 576-wide latent key (512 latent + 64 RoPE dims)
    shared by the 64 heads; the value is the first 512 dims; logits scaled by
    softmax_scale (1/sqrt(576)); LSE is the natural-log log-sum-exp.
R5  FP8: e4m3 (OCP e4m3fn, max 448).  Scales: one fp32 per 128-wide indexer query head
    vector and one per key / latent token; scale = amax/448 (amax = 0 -> 1); code =
    round-to-nearest-even(x / scale) with saturation, decided in fp32.
R6  IndexShare: the Full layer's indices are passed unchanged to the next 3 Shared
    layers ([wiki] "注意力机制：DSA + IndexShare"; [ailearn] "IndexShare：四层共用一次搜索结果").
R7  MTP: the first draft step's Top-k is reused by later steps and drafts add no KV
    (KV Share) ([ailearn] MTP section; [forum] "MTP推测解码改进").  In one decode step
    the 1+d query rows of a sequence all use row 0's indices and the same cache.
V1  MTP verification, the alternative to R7: each of the 1+d query rows of a sequence has its
    own indexer query and head weights, scores the same N_b cached keys (drafts still add
    no KV) and keeps its own Top-k, which that row's sparse MLA uses in every layer of the
    group.  The pages describe only the reuse of R7 ([ailearn] MTP section); this policy
    is what that reuse saves, so it is built to be compared against it.
R8  78-layer schedule: Full at 0-based layers 0, 1 and 2 + 4g; the rest Shared, each
    reusing the preceding Full layer ([ailearn] "IndexShare：四层共用一次搜索结果").
R10 The paged FP8 latent cache holds all 576 dims as e4m3 with one fp32 scale per token
    (the pages name an FP8 KV cache, [forum] "vLLM推理启动", but not its layout).
R11 Paged caches: token s of sequence b sits in page block_table[b][s // 64], slot s % 64
    (the pages give no block size).
R12 Indexer inputs (what feeds R1): q_idx[t] = cq[t] Wq^T split into 32 heads of 128, from the
    query latent cq of rank 2,048; k[t] = LayerNorm(x[t] Wk^T) * gamma + beta over the 128 key
    dims (eps 1e-6, biased variance), and w[t] = x[t] Ww^T, from the hidden state x of width
    6,144 ([ailearn] "一枚 Token，怎样穿过 78 层": hidden 6,144, 32 indexer heads; "IndexShare：
    四层共用一次搜索结果": 9,371,904 parameters per indexer, which these shapes reproduce).  No
    rotary embedding inside the indexer (the pages give none).
R13 Latent KV rows (what feeds R4): row[t] = [RMSNorm(x[t] W_dkv^T) * gamma (512 dims, eps 1e-6) ||
    RoPE(x[t] W_kr^T, t) (64 dims)]; the query's 64 RoPE dims are rotated the same way at their
    own position ([ailearn] architecture card: KV joint compression of rank 512, RoPE theta
    8,000,000 over 2^20 positions).  RoPE turns pair (2i, 2i+1) by the angle pos * theta^(-2i/64).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64", "e4m3_to_f64", "quantize_e4m3_rows", "cache_write_e4m3", "indexer_scores",
    "topk_row", "sparse_mla_row", "dense_causal_attention_row", "prefill_tables",
    "group_prefill", "paged_rows", "group_decode", "group_decode_per_row", "layer_schedule", "indexer_param_count",
    "E4M3_MAX", "IDX_HEADS", "IDX_DIM", "MLA_HEADS", "D_QK", "D_V", "PAGE", "ROPE_THETA", "NORM_EPS",
    "layer_norm", "rms_norm", "rope_pairs", "indexer_projections", "mla_latent_rows", "rope_query",
]

E4M3_MAX = 448.0
IDX_HEADS, IDX_DIM = 32, 128        # [ailearn] architecture card: 32 indexer heads
MLA_HEADS, D_QK, D_V = 64, 576, 512  # [ailearn] architecture card: 64 heads, KV rank 512 (+64 RoPE, R4)
PAGE = 64
ROPE_THETA = 8.0e6                    # [ailearn] architecture card
NORM_EPS = 1e-6                       # R12, R13


# ----------------------------------------------------------------------------- number formats


def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: sign, 8 exponent bits (bias 127), 7 fraction bits."""
    b = np.asarray(bits).astype(np.int64) & 0xFFFF
    sign = np.where(b >> 15, -1.0, 1.0)
    e = (b >> 7) & 0xFF
    f = (b & 0x7F).astype(np.float64)
    val = np.where(e == 0, np.ldexp(f, -133),                      # subnormal: f * 2^-126 / 128
                   np.ldexp(1.0 + f / 128.0, (e - 127).astype(np.int64)))
    val = np.where(e == 0xFF, np.where(f == 0, np.inf, np.nan), val)
    return sign * val


def e4m3_to_f64(codes) -> np.ndarray:
    """Exact value of OCP e4m3fn codes: sign, 4 exponent bits (bias 7), 3 fraction bits.

    Exponent 0 is subnormal (m * 2^-9); code magnitude 0x7F is NaN; there is no infinity."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, np.ldexp(m, -9), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def _encode_e4m3_rne_sat(v32: np.ndarray) -> np.ndarray:
    """Nearest-even e4m3 code of fp32 values, saturating to +-448 (R5)."""
    v = v32.astype(np.float64)
    sign = (np.signbit(v)).astype(np.int64)
    a = np.abs(v)
    # exponent of the quantum: normals have 3 fraction bits above 2^-6, subnormals step 2^-9
    ex = np.frexp(np.where(a > 0, a, 1.0))[1].astype(np.int64) - 1   # floor(log2 a), exact
    ex = np.maximum(ex, -6)
    q = np.ldexp(1.0, ex - 3)
    n = np.rint(a / q)                      # numpy rint: ties to even
    r = np.minimum(n * q, E4M3_MAX)          # saturate
    # encode r exactly
    code = np.zeros(a.shape, dtype=np.int64)
    sub = r < 2.0 ** -6
    code = np.where(sub, np.rint(r / 2.0 ** -9).astype(np.int64), code)
    rn = np.where(sub, 1.0, r)
    e = np.frexp(rn)[1].astype(np.int64) - 1
    m = np.rint((rn / np.ldexp(1.0, e) - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, code, ((e + 7) << 3) | m)
    return ((sign << 7) | code).astype(np.uint8)


def quantize_e4m3_rows(x_bf16_bits, vec_len: int):
    """Per-vector e4m3 quantisation (R5), with the rounding decisions taken in fp32.

    x_bf16_bits: uint16 array whose last axes flatten to [n_vec, vec_len].
    Returns (codes uint8 same shape, scale fp32 [n_vec])."""
    x = bf16_to_f64(x_bf16_bits).astype(np.float32).reshape(-1, vec_len)
    amax = np.max(np.abs(x), axis=1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v = (x / scale[:, None]).astype(np.float32)          # IEEE fp32 division
    codes = _encode_e4m3_rne_sat(v).reshape(np.asarray(x_bf16_bits).shape)
    return codes, scale


def cache_write_e4m3(pool, scale, block_table, x_bf16_bits, seq, pos):
    """Decode-side FP8 cache write (R5, R10, R11): new row r is quantised with one scale over its whole
    row and stored at entry pos[r] % 64 of page block_table[seq[r]][pos[r] // 64].  Returns
    written copies of pool [n_pages,64,dim] and scale [n_pages,64]."""
    pool, scale = np.array(pool, copy=True), np.array(scale, copy=True)
    codes, sc = quantize_e4m3_rows(x_bf16_bits, pool.shape[2])
    for r in range(len(pos)):
        b, t = int(seq[r]), int(pos[r])
        page = int(block_table[b][t // PAGE])
        pool[page, t % PAGE] = codes[r]
        scale[page, t % PAGE] = sc[r]
    return pool, scale


# ----------------------------------------------------------------------------- indexer


def indexer_scores(q, w, k, row_len) -> np.ndarray:
    """Lightweight-indexer scores (R1, R2) for T queries against N keys, fp64.

    q [T,32,128], w [T,32], k [N,128] (values, already dequantised); row_len [T] = number
    of candidate keys per query.  Entries at s >= row_len[t] are -inf."""
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    T, N = q.shape[0], k.shape[0]
    out = np.full((T, N), -np.inf)
    for t in range(T):
        n = int(row_len[t])
        if n <= 0:
            continue
        x = q[t] @ k[:n].T                        # [32, n] per-head dot products
        out[t, :n] = w[t] @ np.maximum(x, 0.0)    # ReLU, per-head weight, sum over heads
    return out


def topk_row(scores_row, n: int, k: int) -> np.ndarray:
    """Indices of the k largest of scores_row[:n] (R3), padded with -1."""
    s = np.asarray(scores_row, dtype=np.float64)[:n]
    order = np.lexsort((np.arange(n), -s))        # primary: score desc; secondary: index asc
    sel = order[:min(k, n)]
    out = np.full(k, -1, dtype=np.int32)
    out[:len(sel)] = sel
    return out


# ----------------------------------------------------------------------------- attention


def sparse_mla_row(Q, KV, idx, softmax_scale: float):
    """One query row of sparse MLA (R4) over the selected rows of KV.

    Q [64,576], KV [*,576] values; idx [k] row numbers into KV, -1 = padding.
    Returns O [64,512], lse [64].  With no valid index: O = 0, lse = -inf."""
    Q = np.asarray(Q, dtype=np.float64)
    sel = np.asarray(idx)
    sel = sel[sel >= 0]
    H = Q.shape[0]
    if sel.size == 0:
        return np.zeros((H, D_V)), np.full(H, -np.inf)
    kv = np.asarray(KV, dtype=np.float64)[sel]    # gathered rows [n, 576]
    z = softmax_scale * (Q @ kv.T)                # [64, n]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    O = (p @ kv[:, :D_V]) / l
    return O, (m + np.log(l))[:, 0]


def dense_causal_attention_row(Q, KV_prefix, softmax_scale: float):
    """Full softmax attention of one query over every row of KV_prefix (no selection).

    Written separately from :func:`sparse_mla_row` as the reference for the k >= L case."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(KV_prefix, dtype=np.float64)
    logits = softmax_scale * np.einsum("hd,nd->hn", Q, K)
    out = np.zeros((Q.shape[0], D_V))
    lse = np.zeros(Q.shape[0])
    for h in range(Q.shape[0]):
        zmax = max(logits[h])
        e = [math.exp(z - zmax) for z in logits[h]]
        tot = math.fsum(e)
        out[h] = np.sum([e[j] * K[j, :D_V] for j in range(K.shape[0])], axis=0) / tot
        lse[h] = zmax + math.log(tot)
    return out, lse


# ----------------------------------------------------------------------------- group / schedule


def prefill_tables(inp: dict, fp8_indexer: bool = False) -> dict:
    """The whole-sequence tables of a prefill group as fp64 values: the indexer keys (bf16, or
    quantised per token to e4m3 and dequantised, R5) and each layer's latent KV rows.

    Computed once per input set; :func:`group_prefill` takes them so that a call over a few
    query rows does only those rows' work."""
    if fp8_indexer:
        k8, sk = quantize_e4m3_rows(inp["k_idx"], IDX_DIM)
        keys = e4m3_to_f64(k8) * sk.reshape(-1, 1)
    else:
        keys = bf16_to_f64(inp["k_idx"])
    return {"fp8_indexer": fp8_indexer, "keys": keys, "KV": [bf16_to_f64(x) for x in inp["KV"]]}


def group_prefill(inp: dict, rows, fp8_indexer: bool = False, idx_override=None, tables=None):
    """One IndexShare group in causal prefill for the listed query rows (R1-R6).

    inp holds numpy arrays as built by the input generator (bf16 as uint16 bits):
    q_idx [L,32,128], w [L,32], k_idx [L,128], Q[l] [L,64,576], KV[l] [L,576].
    Layer 0 is Full: scores + Top-k; layers 1.. reuse its indices.  ``tables`` (from
    :func:`prefill_tables` with the same ``fp8_indexer``) skips the whole-table conversions.
    Returns {"idx": {t: [k]}, "O": [ {t: [64,512]} per layer ], "lse": [...]}."""
    L, k = inp["L"], inp["k"]
    rows = list(rows)
    if tables is None:
        tables = prefill_tables(inp, fp8_indexer)
    assert tables["fp8_indexer"] == fp8_indexer
    kv = tables["keys"]

    def query(t):  # indexer query of row t (only the rows asked for are converted)
        if fp8_indexer:
            q8, sq = quantize_e4m3_rows(np.asarray(inp["q_idx"][t])[None], IDX_DIM)
            return e4m3_to_f64(q8) * sq.reshape(1, IDX_HEADS, 1)
        return bf16_to_f64(np.asarray(inp["q_idx"][t])[None])

    idx = {}
    if idx_override is None:
        for t in rows:
            wt = np.asarray(inp["w"][t], dtype=np.float64)[None]
            sc = indexer_scores(query(t), wt, kv, [t + 1])[0]
            idx[t] = topk_row(sc, t + 1, k)
    else:
        idx = {t: np.asarray(idx_override[t]) for t in rows}
    outO, outL = [], []
    for l in range(len(inp["Q"])):
        Q = inp["Q"][l]
        KVl = tables["KV"][l]
        O, Ls = {}, {}
        for t in rows:
            O[t], Ls[t] = sparse_mla_row(bf16_to_f64(Q[t]), KVl, idx[t], inp["softmax_scale"])
        outO.append(O)
        outL.append(Ls)
    return {"idx": idx, "O": outO, "lse": outL}


def paged_rows(pool, scale, block_table_row, n: int) -> np.ndarray:
    """Dequantised cache rows 0..n-1 of one sequence (R10, R11): row s lives in page bt[s // 64], slot s % 64."""
    s = np.arange(n)
    pages = np.asarray(block_table_row)[s // PAGE]
    slots = s % PAGE
    return e4m3_to_f64(pool[pages, slots]) * np.asarray(scale, dtype=np.float64)[pages, slots][:, None]


def group_decode(inp: dict, seqs=None, idx_override=None, layers=None):
    """One IndexShare group in batched decode with MTP rows (R1-R7), paged FP8 caches.

    Row 0 of each sequence scores its N_b cached keys with an e4m3-quantised query; the
    Top-k is used by all 1+d rows of that sequence and by every layer of the group."""
    ctx, bt, k, R = inp["ctx"], inp["block_table"], inp["k"], inp["rows_per_seq"]
    seqs = range(len(ctx)) if seqs is None else seqs
    q8, sq = quantize_e4m3_rows(inp["q_idx"], IDX_DIM)
    qv = e4m3_to_f64(q8) * sq.reshape(-1, IDX_HEADS, 1)
    w = np.asarray(inp["w"], dtype=np.float64)
    idx = {}
    for b in seqs:
        n = int(ctx[b])
        if idx_override is not None:
            idx[b] = np.asarray(idx_override[b])
            continue
        keys = paged_rows(inp["idx_keys"], inp["idx_key_scale"], bt[b], n)
        sc = indexer_scores(qv[b:b + 1], w[b:b + 1], keys, [n])[0]
        idx[b] = topk_row(sc, n, k)
    layers = range(len(inp["Q"])) if layers is None else layers
    outO, outL = [], []
    for l in layers:
        O, Ls = {}, {}
        for b in seqs:
            n = int(ctx[b])
            kvrows = paged_rows(inp["KV"][l], inp["KV_scale"][l], bt[b], n)
            for r in range(R):
                row = b * R + r
                O[row], Ls[row] = sparse_mla_row(bf16_to_f64(inp["Q"][l][row]), kvrows, idx[b],
                                                 inp["softmax_scale"])
        outO.append(O)
        outL.append(Ls)
    return {"idx": idx, "O": outO, "lse": outL}


def group_decode_per_row(inp: dict, seqs=None, layers=None):
    """One IndexShare group in batched decode where every query row takes its own Top-k (V1).

    inp holds q_idx [B*R,32,128] and w [B*R,32]: query row b*R + r scores sequence b's N_b
    cached keys with its own e4m3-quantised indexer query, keeps its own Top-k, and attends
    over those rows in every layer of the group."""
    ctx, bt, k, R = inp["ctx"], inp["block_table"], inp["k"], inp["rows_per_seq"]
    seqs = range(len(ctx)) if seqs is None else seqs
    q8, sq = quantize_e4m3_rows(inp["q_idx"], IDX_DIM)
    qv = e4m3_to_f64(q8) * sq.reshape(-1, IDX_HEADS, 1)
    w = np.asarray(inp["w"], dtype=np.float64)
    idx = {}
    for b in seqs:
        n = int(ctx[b])
        keys = paged_rows(inp["idx_keys"], inp["idx_key_scale"], bt[b], n)
        for r in range(R):
            row = b * R + r
            sc = indexer_scores(qv[row:row + 1], w[row:row + 1], keys, [n])[0]
            idx[row] = topk_row(sc, n, k)
    layers = range(len(inp["Q"])) if layers is None else layers
    outO, outL = [], []
    for l in layers:
        O, Ls = {}, {}
        for b in seqs:
            kvrows = paged_rows(inp["KV"][l], inp["KV_scale"][l], bt[b], int(ctx[b]))
            for r in range(R):
                row = b * R + r
                O[row], Ls[row] = sparse_mla_row(bf16_to_f64(inp["Q"][l][row]), kvrows, idx[row],
                                                 inp["softmax_scale"])
        outO.append(O)
        outL.append(Ls)
    return {"idx": idx, "O": outO, "lse": outL}


def layer_schedule(n_layers: int = 78):
    """(layer, is_full, producer) for each 0-based layer (R8)."""
    out = []
    for l in range(n_layers):
        full = l < 2 or (l - 2) % 4 == 0
        out.append((l, full, l if full else 2 + 4 * ((l - 2) // 4)))
    return out


def indexer_param_count(q_rank: int = 2048, hidden: int = 6144, heads: int = IDX_HEADS,
                        dim: int = IDX_DIM) -> int:
    """Parameters of one indexer under one reconstruction of the 'public dims'.

    q projection from the query latent (q_rank -> heads*dim), k projection (hidden -> dim),
    head-weight projection (hidden -> heads), and a key LayerNorm (weight + bias).  The
    hidden size 6,144 and the 32 heads are on [ailearn] ("一枚 Token，怎样穿过 78 层");
    the 2,048 query rank and the LayerNorm are this file's reading.  Check only."""
    return q_rank * heads * dim + hidden * dim + hidden * heads + 2 * dim


# ----------------------------------------------------------------------------- inputs of the path


def layer_norm(x, gamma, beta, eps: float = NORM_EPS) -> np.ndarray:
    """Per-row LayerNorm over the last axis (R12): (x - mean) / sqrt(var + eps) * gamma + beta,
    var the biased (1/n) variance."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, dtype=np.float64) + np.asarray(beta, dtype=np.float64)


def rms_norm(x, gamma, eps: float = NORM_EPS) -> np.ndarray:
    """Per-row RMSNorm over the last axis (R13): x / sqrt(mean(x^2) + eps) * gamma."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x ** 2).mean(axis=-1, keepdims=True) + eps) * np.asarray(gamma, dtype=np.float64)


def rope_pairs(x, pos, theta: float = ROPE_THETA) -> np.ndarray:
    """Rotary embedding of the last axis (64 dims, R13): pair (2i, 2i+1) of a vector at position
    pos turns by the angle pos * theta^(-2i/64)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    freq = theta ** (-np.arange(0, d, 2, dtype=np.float64) / d)          # [d/2]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq             # [..., d/2]
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    out[..., 1::2] = x[..., 0::2] * s + x[..., 1::2] * c
    return out


def indexer_projections(cq, x, Wq, Wk, Ww, gamma, beta):
    """Indexer inputs of T tokens (R12): cq [T,2048], x [T,6144] values; Wq [4096,2048],
    Wk [128,6144], Ww [32,6144] (output x input); gamma, beta [128].
    Returns q_idx [T,32,128], k [T,128], w [T,32] in fp64."""
    cq, x = np.asarray(cq, dtype=np.float64), np.asarray(x, dtype=np.float64)
    q = cq @ np.asarray(Wq, dtype=np.float64).T
    k = layer_norm(x @ np.asarray(Wk, dtype=np.float64).T, gamma, beta)
    w = x @ np.asarray(Ww, dtype=np.float64).T
    return q.reshape(len(q), IDX_HEADS, IDX_DIM), k, w


def mla_latent_rows(x, W_dkv, W_kr, gamma, pos):
    """Latent KV rows of T tokens (R13): x [T,6144]; W_dkv [512,6144], W_kr [64,6144]; gamma [512];
    pos [T].  Returns [T,576] = [RMSNorm(x W_dkv^T) * gamma || RoPE(x W_kr^T, pos)] in fp64."""
    x = np.asarray(x, dtype=np.float64)
    c = rms_norm(x @ np.asarray(W_dkv, dtype=np.float64).T, gamma)
    r = rope_pairs(x @ np.asarray(W_kr, dtype=np.float64).T, pos)
    return np.concatenate([c, r], axis=-1)


def rope_query(q, pos) -> np.ndarray:
    """The query side of R13: q [T,64,576] with dims 512..575 of every head turned to position pos[t]."""
    q = np.array(q, dtype=np.float64, copy=True)
    q[:, :, D_V:] = rope_pairs(q[:, :, D_V:], np.asarray(pos)[:, None])
    return q

"""ctypes binding of ``libdsa.so`` (the C ABI in include/dsa.h).

Argument marshalling only: every step of the path runs in the CUDA library.  Tensors are
torch tensors on the current CUDA device; outputs are allocated here with torch and filled
by the library on the current torch stream.  There is no CPU fallback: if the library or a
GPU is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa.so")

DSA_BF16, DSA_E4M3 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "stale index handle", 4: "device wait timed out",
          5: "CUDA error", 6: "workspace too small", 7: "index or page out of range",
          8: "input value outside the supported range"}
DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_STALE_HANDLE, DSA_ERR_TIMEOUT, DSA_ERR_CUDA, \
    DSA_ERR_WORKSPACE, DSA_ERR_BOUNDS, DSA_ERR_RANGE = range(9)

EXPORTS = [
    "dsa_quant_e4m3", "dsa_indexer_score", "dsa_topk_workspace_bytes", "dsa_topk",
    "dsa_sparse_mla_workspace_bytes", "dsa_sparse_mla_attn", "dsa_group_workspace_bytes",
    "indexshare_group_forward", "dsa_layer_is_full", "dsa_layer_producer", "dsa_status_str",
    "dsa_last_error", "dsa_abi_version", "dsa_abi_sizeof", "dsa_sync_status", "dsa_debug_bounded_wait",
    "dsa_set_wait_limit_ns", "dsa_launch_count", "dsa_topk_no_alloc", "dsa_cache_write_e4m3",
    "dsa_indexer_project_workspace_bytes", "dsa_indexer_project", "dsa_mla_latent_workspace_bytes", "dsa_mla_latent",
    "dsa_rope_query", "dsa_split_candidates", "dsa_split_merge_workspace_bytes", "dsa_split_merge",
    "dsa_combine_partials", "dsa_cache_write_e4m3_pools",
]


class CacheView(ctypes.Structure):
    _fields_ = [("data", c_void_p), ("scale", c_void_p), ("block_table", c_void_p), ("seq_lens", c_void_p),
                ("row_stride", c_int64), ("n_tokens", c_int64), ("dim", c_int32), ("dtype", c_int32),
                ("max_pages", c_int32), ("batch", c_int32)]


class IndexHandle(ctypes.Structure):
    _fields_ = [("idx", c_void_p), ("rows", c_int32), ("k", c_int32), ("filled", c_int32),
                ("producer_layer", c_int32), ("generation", c_int64)]


class GroupArgs(ctypes.Structure):
    _fields_ = [("q_idx", c_void_p), ("w", c_void_p), ("idx_keys", CacheView), ("indexer_dtype", c_int32),
                ("n_idx_rows", c_int32), ("q_pos0", c_int32), ("k", c_int32), ("q_rows_per_idx_row", c_int32),
                ("n_layers", c_int32), ("first_layer", c_int32), ("softmax_scale", c_float),
                ("q", c_void_p * 4), ("kv", CacheView * 4), ("out", c_void_p * 4), ("lse", c_void_p * 4),
                ("workspace", c_void_p), ("workspace_bytes", c_size_t), ("trace_events", c_void_p)]


class DsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load libdsa.so (raises if it was not built) and declare the signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with long_context_sparse_11_b200/build.py")
    lib = ctypes.CDLL(path)
    S = c_int32
    sig = {
        "dsa_quant_e4m3": (S, [c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]),
        "dsa_cache_write_e4m3": (S, [c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                     c_int32, c_void_p, c_void_p, c_void_p]),
        "dsa_indexer_score": (S, [c_void_p, c_int32, c_void_p, c_void_p, c_int32, c_int32, POINTER(CacheView),
                                  c_void_p, c_int64, c_void_p]),
        "dsa_topk_workspace_bytes": (c_size_t, [c_int32, c_int64, c_int32]),
        "dsa_topk": (S, [c_void_p, c_int64, c_int32, c_void_p, c_int64, c_int64, c_int32, c_void_p, c_void_p,
                         c_size_t, c_void_p]),
        "dsa_sparse_mla_workspace_bytes": (c_size_t, [c_int32, c_int32, POINTER(CacheView)]),
        "dsa_sparse_mla_attn": (S, [c_void_p, POINTER(CacheView), c_void_p, c_int32, c_int32, c_int32, c_float,
                                    c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "dsa_group_workspace_bytes": (c_size_t, [POINTER(GroupArgs)]),
        "indexshare_group_forward": (S, [POINTER(GroupArgs), POINTER(IndexHandle), c_int32, c_void_p]),
        "dsa_layer_is_full": (c_int32, [c_int32]),
        "dsa_layer_producer": (c_int32, [c_int32]),
        "dsa_status_str": (ctypes.c_char_p, [c_int32]),
        "dsa_last_error": (ctypes.c_char_p, []),
        "dsa_abi_version": (c_int32, []),
        "dsa_abi_sizeof": (c_size_t, [c_int32]),
        "dsa_sync_status": (S, [c_void_p]),
        "dsa_debug_bounded_wait": (S, [c_int64, c_void_p]),
        "dsa_set_wait_limit_ns": (c_int64, [c_int64]),
        "dsa_launch_count": (c_int64, []),
        "dsa_topk_no_alloc": (S, [c_void_p, c_int64, c_int32, c_void_p, c_int64, c_int64, c_int32, c_void_p,
                                  c_void_p]),
        "dsa_indexer_project_workspace_bytes": (c_size_t, [c_int32]),
        "dsa_indexer_project": (S, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                    c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "dsa_mla_latent_workspace_bytes": (c_size_t, [c_int32]),
        "dsa_mla_latent": (S, [c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_float, c_void_p, c_void_p,
                               c_size_t, c_void_p]),
        "dsa_rope_query": (S, [c_void_p, c_void_p, c_int32, c_float, c_void_p]),
        "dsa_split_candidates": (S, [c_void_p, c_int64, c_int32, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                     c_void_p, c_void_p]),
        "dsa_split_merge_workspace_bytes": (c_size_t, [c_int32, c_int32, c_int32]),
        "dsa_split_merge": (S, [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                c_void_p, c_size_t, c_void_p]),
        "dsa_combine_partials": (S, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p]),
        "dsa_cache_write_e4m3_pools": (S, [c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_void_p,
                                           c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def _check(status: int):
    if status != DSA_OK:
        raise DsaError(status, load().dsa_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------------------------ cache views


def dense_view(data, scale=None) -> CacheView:
    """Dense token-major cache: data [n_tokens, row_stride] (bf16 or uint8 e4m3), scale [n_tokens]."""
    import torch
    assert data.dim() == 2 and data.stride(1) == 1
    dt = DSA_BF16 if data.dtype == torch.bfloat16 else DSA_E4M3
    dim = 128 if data.shape[1] < 576 else 576
    v = CacheView(data.data_ptr(), _ptr(scale), None, None, data.stride(0), data.shape[0], dim, dt, 0, 0)
    v._keep = (data, scale)
    return v


def paged_view(pool, scale, block_table, seq_lens, rows_per_seq: int = 1) -> CacheView:
    """Paged e4m3 cache: pool [n_pages,64,dim] uint8, scale [n_pages,64] fp32,
    block_table [B,max_pages] int32, seq_lens [B] int32 (all on the device).

    rows_per_seq > 1 presents each sequence as that many consecutive entries sharing its pages
    and length (the block-table rows and lengths are repeated once, here; the pages are not
    copied): the view through which every MTP verification row is scored, selected and attended
    as its own row, for a per-row Top-k instead of the reuse of row 0's."""
    n_pages, page, dim = pool.shape
    assert page == 64 and rows_per_seq >= 1
    if rows_per_seq > 1:
        block_table = block_table.repeat_interleave(rows_per_seq, dim=0).contiguous()
        seq_lens = seq_lens.repeat_interleave(rows_per_seq).contiguous()
    v = CacheView(pool.data_ptr(), scale.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(), dim,
                  n_pages * 64, dim, DSA_E4M3, block_table.shape[1], block_table.shape[0])
    v._keep = (pool, scale, block_table, seq_lens)
    return v


# ------------------------------------------------------------------------------ entry points


def quant_e4m3(x, codes=None, scale=None):
    """a1: x [..., 128] bf16 -> (codes uint8 same shape, scale fp32 [n_vec])."""
    import torch
    n_vec = x.numel() // 128
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device) if codes is None else codes
    scale = torch.empty(n_vec, dtype=torch.float32, device=x.device) if scale is None else scale
    _check(load().dsa_quant_e4m3(x.data_ptr(), n_vec, 128, codes.data_ptr(), scale.data_ptr(), _stream()))
    return codes, scale


def cache_write_e4m3(x, pos, block_table, pool, pool_scale, seq=None):
    """a1 for decode: rows x [n,dim] bf16 (dim 128 or 576) quantised per token into their slots of
    the paged pool [n_pages,64,dim] uint8 / pool_scale [n_pages,64] fp32; row r goes to sequence
    seq[r] (r when seq is None) at position pos[r] through block_table [B,max_pages] int32."""
    n, dim = x.shape
    _check(load().dsa_cache_write_e4m3(x.data_ptr(), n, dim, _ptr(seq), pos.data_ptr(), block_table.data_ptr(),
                                       block_table.shape[0], block_table.shape[1], pool.shape[0], pool.data_ptr(),
                                       pool_scale.data_ptr(), _stream()))
    return pool, pool_scale


class CacheWriteBatch:
    """The current token's rows of one decode step into several paged e4m3 pools with one launch:
    writes[i] = (x [n,dim] bf16, pool [n_pages,64,dim] uint8, scale [n_pages,64] fp32), all over the
    same block_table [B,max_pages] int32 and positions pos [n] int32 (row r -> sequence seq[r], or r).
    The host-side pointer arrays are built once, here."""

    def __init__(self, writes, pos, block_table, seq=None):
        n = len(writes)
        self.n_rows = writes[0][0].shape[0]
        self.xs = (c_void_p * n)(*[x.data_ptr() for x, _, _ in writes])
        self.dims = (c_int32 * n)(*[x.shape[1] for x, _, _ in writes])
        self.pools = (c_void_p * n)(*[p.data_ptr() for _, p, _ in writes])
        self.scales = (c_void_p * n)(*[s.data_ptr() for _, _, s in writes])
        self.n_pages = writes[0][1].shape[0]
        self.pos, self.block_table, self.seq = pos, block_table, seq
        self._keep = writes

    def __call__(self):
        _check(load().dsa_cache_write_e4m3_pools(len(self._keep), self.xs, self.dims, self.pools, self.scales,
                                                 self.n_rows, _ptr(self.seq), self.pos.data_ptr(),
                                                 self.block_table.data_ptr(), self.block_table.shape[0],
                                                 self.block_table.shape[1], self.n_pages, _stream()))


def indexer_score(q, w, keys: CacheView, scores, q_scale=None, q_pos0: int = 0):
    """a2+a3: scores[r, :len_r] for q [n_q,32,128] (bf16 or uint8 e4m3) against `keys`."""
    import torch
    dt = DSA_BF16 if q.dtype == torch.bfloat16 else DSA_E4M3
    _check(load().dsa_indexer_score(q.data_ptr(), dt, _ptr(q_scale), w.data_ptr(), q.shape[0], q_pos0,
                                    ctypes.byref(keys), scores.data_ptr(), scores.stride(0), _stream()))
    return scores


def topk(scores, k: int, row_len=None, causal_len0: int = 0, max_len=None, out=None, workspace=None):
    """a4: exact per-row Top-k positions [n_rows, k] int32 (-1 padded)."""
    import torch
    n = scores.shape[0]
    max_len = scores.shape[1] if max_len is None else max_len
    out = torch.empty(n, k, dtype=torch.int32, device=scores.device) if out is None else out
    lib = load()
    need = lib.dsa_topk_workspace_bytes(n, max_len, k)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=scores.device)
    _check(lib.dsa_topk(scores.data_ptr(), scores.stride(0), n, _ptr(row_len), causal_len0, max_len, k,
                        out.data_ptr(), _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream()))
    return out


def topk_no_alloc(scores, k: int, out, row_len=None, causal_len0: int = 0, max_len=None):
    """a4 for callers that cannot allocate device memory: same result as :func:`topk`, scratch
    inside the library; `out` [n_rows, k] int32 must be provided (nothing is allocated here)."""
    n = scores.shape[0]
    max_len = scores.shape[1] if max_len is None else max_len
    _check(load().dsa_topk_no_alloc(scores.data_ptr(), scores.stride(0), n, _ptr(row_len), causal_len0, max_len, k,
                                    out.data_ptr(), _stream()))
    return out


def sparse_mla_attn(q, kv: CacheView, idx, k: int, softmax_scale: float, q_rows_per_idx_row: int = 1,
                    out=None, lse=None, workspace=None):
    """a6: out [n_q,64,512] bf16 and lse [n_q,64] fp32 of sparse MLA over idx."""
    import torch
    n_q = q.shape[0]
    out = torch.empty(n_q, 64, 512, dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(n_q, 64, dtype=torch.float32, device=q.device) if lse is None else lse
    lib = load()
    need = lib.dsa_sparse_mla_workspace_bytes(n_q, k, ctypes.byref(kv))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.dsa_sparse_mla_attn(q.data_ptr(), ctypes.byref(kv), idx.data_ptr(), n_q, q_rows_per_idx_row, k,
                                   softmax_scale, out.data_ptr(), lse.data_ptr(), _ptr(workspace),
                                   0 if workspace is None else workspace.numel(), _stream()))
    return out, lse


ROPE_THETA = 8.0e6


def indexer_project(cq, x, Wq, Wkw, gamma, beta, q_out=None, k_out=None, w_out=None, workspace=None):
    """The indexer's inputs: q [T,32,128] bf16 from the query latent cq [T,q_rank], the key
    [T,128] bf16 (LayerNorm) and head weights [T,32] fp32 from the hidden state x [T,hidden];
    Wq [4096,q_rank], Wkw [160,hidden] (Wk rows then Ww rows) bf16, gamma / beta [128] fp32."""
    import torch
    T = cq.shape[0]
    dev = cq.device
    q_out = torch.empty(T, 32, 128, dtype=torch.bfloat16, device=dev) if q_out is None else q_out
    k_out = torch.empty(T, 128, dtype=torch.bfloat16, device=dev) if k_out is None else k_out
    w_out = torch.empty(T, 32, dtype=torch.float32, device=dev) if w_out is None else w_out
    lib = load()
    need = lib.dsa_indexer_project_workspace_bytes(T)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib.dsa_indexer_project(cq.data_ptr(), x.data_ptr(), Wq.data_ptr(), Wkw.data_ptr(), gamma.data_ptr(),
                                   beta.data_ptr(), T, cq.shape[1], x.shape[1], q_out.data_ptr(), k_out.data_ptr(),
                                   w_out.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream()))
    return q_out, k_out, w_out


def mla_latent(x, Wkv, gamma, pos, theta: float = ROPE_THETA, out=None, workspace=None):
    """Latent KV rows [T,576] bf16 from the hidden state x [T,hidden]: RMSNorm of x W_dkv^T (512 dims)
    and RoPE of x W_kr^T (64 dims) at positions pos [T] int32; Wkv [576,hidden] bf16, gamma [512] fp32."""
    import torch
    T = x.shape[0]
    out = torch.empty(T, 576, dtype=torch.bfloat16, device=x.device) if out is None else out
    lib = load()
    if workspace is None:
        workspace = torch.empty(max(lib.dsa_mla_latent_workspace_bytes(T), 16), dtype=torch.uint8, device=x.device)
    _check(lib.dsa_mla_latent(x.data_ptr(), Wkv.data_ptr(), gamma.data_ptr(), pos.data_ptr(), T, x.shape[1], theta,
                              out.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream()))
    return out


def rope_query(q, pos, theta: float = ROPE_THETA):
    """Turn dims 512..575 of every head of q [T,64,576] bf16 in place to positions pos [T] int32."""
    _check(load().dsa_rope_query(q.data_ptr(), pos.data_ptr(), q.shape[0], theta, _stream()))
    return q


def split_candidates(scores, idx_local, n_local: int, offset: int):
    """A rank's local Top-k [rows, k] over its slice's scores [rows, ld] -> (cand_score [rows, k] fp32,
    cand_idx [rows, k] int32): (score, offset + position) ordered by position, padding last."""
    import torch
    rows, k = idx_local.shape
    cs = torch.empty(rows, k, dtype=torch.float32, device=scores.device)
    ci = torch.empty(rows, k, dtype=torch.int32, device=scores.device)
    _check(load().dsa_split_candidates(scores.data_ptr(), scores.stride(0), rows, idx_local.data_ptr(), k, n_local,
                                       offset, cs.data_ptr(), ci.data_ptr(), _stream()))
    return cs, ci


def split_merge(cand_score, cand_idx, k: int, lo: int, hi: int, workspace=None):
    """All ranks' candidates [rows, G*k] (rank order) -> (idx_global [rows, k], idx_local [rows, k])."""
    import torch
    rows, n_cand = cand_score.shape
    ig = torch.empty(rows, k, dtype=torch.int32, device=cand_score.device)
    il = torch.empty(rows, k, dtype=torch.int32, device=cand_score.device)
    lib = load()
    need = lib.dsa_split_merge_workspace_bytes(rows, n_cand, k)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=cand_score.device)
    _check(lib.dsa_split_merge(cand_score.data_ptr(), cand_idx.data_ptr(), rows, n_cand, k, lo, hi, ig.data_ptr(),
                               il.data_ptr(), _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream()))
    return ig, il


def combine_partials(o_parts, lse_parts, out=None, lse=None):
    """Partial attention of G ranks, o_parts [G,n_q,64,512] bf16 and lse_parts [G,n_q,64] fp32 -> out, lse."""
    import torch
    G, n_q = lse_parts.shape[0], lse_parts.shape[1]
    out = torch.empty(n_q, 64, 512, dtype=torch.bfloat16, device=o_parts.device) if out is None else out
    lse = torch.empty(n_q, 64, dtype=torch.float32, device=o_parts.device) if lse is None else lse
    _check(load().dsa_combine_partials(o_parts.data_ptr(), lse_parts.data_ptr(), G, n_q, out.data_ptr(),
                                       _ptr(lse), _stream()))
    return out, lse


class IndexShareGroup:
    """One IndexShare group call: a Full layer's indexer + Top-k into a reuse handle, then
    sparse MLA for every layer of the group with the handle's indices."""

    def __init__(self, q_idx, w, idx_keys: CacheView, k: int, q: list, kv: list, softmax_scale: float,
                 indexer_dtype: int = DSA_BF16, q_pos0: int = 0, q_rows_per_idx_row: int = 1,
                 first_layer: int = 0, handle_idx=None):
        import torch
        dev = q_idx.device
        n = q_idx.shape[0]
        nq = n * q_rows_per_idx_row
        self.out = [torch.empty(nq, 64, 512, dtype=torch.bfloat16, device=dev) for _ in q]
        self.lse = [torch.empty(nq, 64, dtype=torch.float32, device=dev) for _ in q]
        self.idx = torch.empty(n, k, dtype=torch.int32, device=dev) if handle_idx is None else handle_idx
        a = GroupArgs()
        a.q_idx, a.w, a.idx_keys = q_idx.data_ptr(), w.data_ptr(), idx_keys
        a.indexer_dtype, a.n_idx_rows, a.q_pos0, a.k = indexer_dtype, n, q_pos0, k
        a.q_rows_per_idx_row, a.n_layers, a.first_layer, a.softmax_scale = q_rows_per_idx_row, len(q), first_layer, \
            softmax_scale
        for i, (qq, vv) in enumerate(zip(q, kv)):
            a.q[i], a.kv[i], a.out[i], a.lse[i] = qq.data_ptr(), vv, self.out[i].data_ptr(), self.lse[i].data_ptr()
        lib = load()
        # 0 when the arguments are invalid: forward() then returns the validation error itself
        need = lib.dsa_group_workspace_bytes(ctypes.byref(a))
        self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        a.workspace, a.workspace_bytes = self.workspace.data_ptr(), self.workspace.numel()
        self.args = a
        self.handle = IndexHandle(self.idx.data_ptr(), n, k, 0, -1, 0)
        self._keep = (q_idx, w, idx_keys, q, kv)

    def forward(self, reuse_only: bool = False):
        _check(load().indexshare_group_forward(ctypes.byref(self.args), ctypes.byref(self.handle),
                                               1 if reuse_only else 0, _stream()))
        return self.out, self.lse


def sync_status():
    """Synchronise the current stream and raise if a kernel recorded a device-side error."""
    _check(load().dsa_sync_status(_stream()))


def layer_is_full(layer: int) -> bool:
    return bool(load().dsa_layer_is_full(layer))


def layer_producer(layer: int) -> int:
    return int(load().dsa_layer_producer(layer))

"""Input recipes for the workloads (seeded, synthetic; no method arithmetic here).

Workloads, named by what they are:

* ``tiny_prefill``    causal prefill L=512, Top-128, bf16, one IndexShare group of 4 layers;
                      indexer q/k ~N(0,1)/sqrt(128), head weights ~N(0,1), MLA q/KV ~N(0,1).
* ``prefill_32k``     causal prefill L=32,768, Top-2048, bf16; indexer keys drift along
                      positions as AR(1) with rho=0.99 so the selected sets are local.
* ``prefill_128k_fp8`` causal prefill L=131,072, Top-2048; indexer q/k are bf16 ~N(0,1)
                      quantised to e4m3 on the path; MLA latent KV bf16.
* ``decode_b32_mtp4`` 32 sequences, context ~U[65,536, 262,144], 1 + 4 draft rows per
                      sequence, FP8 paged caches (64-token pages, physically permuted).
* ``decode_b32_d0``   the same batch and caches as ``decode_b32_mtp4`` with one query row per
                      sequence (no draft rows): sparse MLA reads 580 B per selected key for 139,264
                      flops, so it is bound by memory rather than by the tensor cores.
* ``decode_b32_mtp4_verify`` the batch, caches and MLA rows of ``decode_b32_mtp4``, but each of
                      the 5 rows of a sequence has its own indexer query and head weights (row 0
                      keeps the ``decode_b32_mtp4`` ones) and takes its own Top-k: the per-token
                      selection for MTP verification rows, against the reuse of row 0's.
* ``decode_1m_mtp5``  1 sequence of 1,048,576 tokens, 1 + 5 rows, 78-layer schedule.

Stream ids keep every tensor independent: ``sub_seed(seed, layer, TENSOR_ID)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .generators import (
    normal_np, normal_torch, bf16_bits_np, bf16_bits_torch, sub_seed, ar1_keys_np,
    uniform_np, e4m3_codes_torch, splitmix64_np, normal_bf16_torch,
)

__all__ = ["PrefillSpec", "DecodeSpec", "WORKLOADS", "make_prefill", "make_decode",
           "decode_context_lengths", "page_table", "make_decode_indexer", "make_decode_new_tokens",
           "IDX_HEADS", "IDX_DIM", "MLA_HEADS", "D_QK", "D_V", "PAGE"]

IDX_HEADS, IDX_DIM = 32, 128
MLA_HEADS, D_QK, D_V = 64, 576, 512
PAGE = 64

T_QIDX, T_W, T_KIDX, T_Q, T_KV, T_PERM, T_CTX, T_KSCALE, T_KVSCALE = range(1, 10)
T_QIDX_DRAFT, T_W_DRAFT = 10, 11   # indexer query and weights of draft rows (per-row Top-k only)
T_NEW_KV, T_NEW_KEY = 12, 13         # a decode step's new token rows (latent row, indexer key)


@dataclass
class PrefillSpec:
    name: str
    L: int
    k: int
    indexer_fp8: bool = False
    n_layers: int = 4
    seed: int = 0
    idx_std: float = 1.0          # std of indexer q and k
    ar1_rho: float | None = None  # AR(1) drift of indexer keys along positions
    softmax_scale: float = 1.0 / math.sqrt(D_QK)


@dataclass
class DecodeSpec:
    name: str
    batch: int
    ctx_lo: int
    ctx_hi: int
    rows_per_seq: int
    k: int = 2048
    n_layers: int = 4
    seed: int = 0
    fixed_ctx: int | None = None
    softmax_scale: float = 1.0 / math.sqrt(D_QK)
    full_layers: list = field(default_factory=lambda: [0])
    topk_per_row: bool = False    # every query row has its own indexer query and Top-k


WORKLOADS = {
    "tiny_prefill": PrefillSpec("tiny_prefill", L=512, k=128, seed=0, idx_std=1.0 / math.sqrt(IDX_DIM)),
    "prefill_32k": PrefillSpec("prefill_32k", L=32768, k=2048, seed=2, ar1_rho=0.99),
    "prefill_128k_fp8": PrefillSpec("prefill_128k_fp8", L=131072, k=2048, seed=3, indexer_fp8=True),
    "decode_b32_mtp4": DecodeSpec("decode_b32_mtp4", batch=32, ctx_lo=65536, ctx_hi=262144,
                                  rows_per_seq=5, seed=4),
    "decode_b32_d0": DecodeSpec("decode_b32_d0", batch=32, ctx_lo=65536, ctx_hi=262144, rows_per_seq=1, seed=4),
    "decode_b32_mtp4_verify": DecodeSpec("decode_b32_mtp4_verify", batch=32, ctx_lo=65536, ctx_hi=262144,
                                         rows_per_seq=5, seed=4, topk_per_row=True),
    "decode_1m_mtp5": DecodeSpec("decode_1m_mtp5", batch=1, ctx_lo=1 << 20, ctx_hi=1 << 20,
                                 rows_per_seq=6, seed=5, n_layers=78, fixed_ctx=1 << 20),
}


def _normal(seed, n, device):
    if device is None:
        return normal_np(seed, 0, n)
    return normal_torch(seed, 0, n, device=device)


def _bf16(x, device):
    if device is None:
        return bf16_bits_np(x)
    return bf16_bits_torch(x)


def _f32(x, device):
    if device is None:
        return np.asarray(x, dtype=np.float32)
    import torch
    return x.to(torch.float32)


def _cat_rows(first, rest, shape):
    """Row 0 of each sequence from `first` [B,...], rows 1.. from `rest` [B,R-1,...], flattened."""
    if isinstance(first, np.ndarray):
        return np.concatenate([first[:, None], rest], axis=1).reshape(shape)
    import torch
    return torch.cat([first[:, None], rest], dim=1).reshape(shape)


def make_prefill(spec: PrefillSpec, L: int | None = None, device=None, layers=None) -> dict:
    """Inputs of one IndexShare group for causal prefill of length ``L`` (default: the spec's).

    ``device=None`` returns numpy arrays (bf16 as uint16 bit patterns); otherwise torch
    tensors on that device (bf16 as torch.bfloat16).  Layouts:
      q_idx [L,32,128] bf16, w [L,32] fp32, k_idx [L,128] bf16,
      Q[l] [L,64,576] bf16, KV[l] [L,576] bf16 for l in range(n_layers).
    """
    L = spec.L if L is None else L
    s = spec.seed
    out = {"L": L, "k": spec.k, "softmax_scale": spec.softmax_scale}
    q = _normal(sub_seed(s, 0, T_QIDX), L * IDX_HEADS * IDX_DIM, device) * spec.idx_std
    out["q_idx"] = _bf16(q, device).reshape(L, IDX_HEADS, IDX_DIM)
    out["w"] = _f32(_normal(sub_seed(s, 0, T_W), L * IDX_HEADS, device), device).reshape(L, IDX_HEADS)
    if spec.ar1_rho is not None:
        kk = ar1_keys_np(sub_seed(s, 0, T_KIDX), L, IDX_DIM, spec.ar1_rho) * spec.idx_std
        kb = bf16_bits_np(kk)
        if device is not None:
            import torch
            kb = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).to(device)
        out["k_idx"] = kb
    else:
        kk = _normal(sub_seed(s, 0, T_KIDX), L * IDX_DIM, device) * spec.idx_std
        out["k_idx"] = _bf16(kk, device).reshape(L, IDX_DIM)
    layers = range(spec.n_layers) if layers is None else layers
    out["Q"], out["KV"] = [], []
    for l in layers:
        out["Q"].append(_bf16_normal(sub_seed(s, l, T_Q), L * MLA_HEADS * D_QK, device).reshape(L, MLA_HEADS, D_QK))
        out["KV"].append(_bf16_normal(sub_seed(s, l, T_KV), L * D_QK, device).reshape(L, D_QK))
    return out


def _bf16_normal(seed, n, device):
    if device is None:
        return bf16_bits_np(normal_np(seed, 0, n))
    return normal_bf16_torch(seed, n, device)


def decode_context_lengths(spec: DecodeSpec) -> np.ndarray:
    """Per-sequence context lengths N_b (the current token is included)."""
    if spec.fixed_ctx is not None:
        return np.full(spec.batch, spec.fixed_ctx, dtype=np.int64)
    u = uniform_np(sub_seed(spec.seed, 0, T_CTX), 0, spec.batch)
    span = spec.ctx_hi - spec.ctx_lo + 1
    return (spec.ctx_lo + np.floor(u * span)).astype(np.int64)


def page_table(spec: DecodeSpec, ctx: np.ndarray):
    """Block table [B, max_pages] int32 over a physically permuted page pool (-1 = unused)."""
    pages = (ctx + PAGE - 1) // PAGE
    total = int(pages.sum())
    keys = splitmix64_np(sub_seed(spec.seed, 0, T_PERM), np.arange(total, dtype=np.uint64))
    perm = np.argsort(keys, kind="stable").astype(np.int32)
    maxp = int(pages.max())
    bt = np.full((len(ctx), maxp), -1, dtype=np.int32)
    off = 0
    for b, p in enumerate(pages):
        bt[b, :p] = perm[off:off + p]
        off += int(p)
    return bt, total


def _fp8_pool(seed, n_pages, dim, device):
    """Synthetic FP8 cache: ~N(0,1) values stored as e4m3 codes with a per-token fp32 scale.

    The per-token scale is drawn uniformly in [1/128, 1/96] (a storage recipe of the
    generator, independent of the path's own quantisation rule)."""
    import torch
    n_tok = n_pages * PAGE
    sc = (1.0 / 128.0 + (1.0 / 96.0 - 1.0 / 128.0) *
          torch.from_numpy(uniform_np(seed ^ 0x5A5A, 0, n_tok))).to(torch.float32)
    dev = "cpu" if device is None else device
    sc = sc.to(dev)
    codes = torch.empty(n_tok, dim, dtype=torch.uint8, device=dev)
    step = max(1, (1 << 24) // dim)
    for a in range(0, n_tok, step):
        b = min(n_tok, a + step)
        x = normal_torch(seed, a * dim, (b - a) * dim, device=dev).view(b - a, dim)
        codes[a:b] = e4m3_codes_torch(x / sc[a:b, None].to(torch.float64))
    codes = codes.view(n_pages, PAGE, dim)
    sc = sc.view(n_pages, PAGE)
    if device is None:
        return codes.numpy(), sc.numpy()
    return codes, sc


def make_decode_indexer(spec: DecodeSpec, layer: int, n_pages: int, batch: int, device=None) -> dict:
    """Indexer inputs of one Full layer of a decode step: q_idx [B,32,128] bf16, w [B,32] fp32,
    idx_keys [P,64,128] e4m3 + idx_key_scale [P,64] (streams keyed by the layer number)."""
    s = spec.seed
    q = _normal(sub_seed(s, layer, T_QIDX), batch * IDX_HEADS * IDX_DIM, device)
    w = _f32(_normal(sub_seed(s, layer, T_W), batch * IDX_HEADS, device), device).reshape(batch, IDX_HEADS)
    keys, sc = _fp8_pool(sub_seed(s, layer, T_KIDX), n_pages, IDX_DIM, device)
    return {"q_idx": _bf16(q, device).reshape(batch, IDX_HEADS, IDX_DIM), "w": w, "idx_keys": keys,
            "idx_key_scale": sc}


def make_decode_new_tokens(spec: DecodeSpec, batch: int, layers, full_layers, device=None) -> dict:
    """The rows a decode step appends for its current token (position N_b - 1 of each sequence):
    a latent row [B,576] bf16 ~N(0,1) for every layer in ``layers`` and an indexer key row
    [B,128] bf16 ~N(0,1) for every Full layer in ``full_layers`` (streams keyed by the layer)."""
    s = spec.seed
    kv = {l: _bf16(_normal(sub_seed(s, l, T_NEW_KV), batch * D_QK, device), device).reshape(batch, D_QK)
          for l in layers}
    key = {l: _bf16(_normal(sub_seed(s, l, T_NEW_KEY), batch * IDX_DIM, device), device).reshape(batch, IDX_DIM)
           for l in full_layers}
    return {"kv": kv, "key": key}


def make_decode(spec: DecodeSpec, device=None, ctx=None, layers=None) -> dict:
    """Inputs of one decode step (batch of sequences with paged FP8 caches).

    Layouts: q_idx [B,32,128] bf16 (row 0 of each sequence), w [B,32] fp32; with
    ``topk_per_row`` q_idx [B*R,32,128] and w [B*R,32], row b*R the same as above and rows
    b*R+1..b*R+R-1 from their own streams;
    idx_keys [P,64,128] e4m3 + idx_key_scale [P,64] fp32 (one pool per Full layer),
    Q[l] [B*R,64,576] bf16, KV[l] [P,64,576] e4m3 + KV_scale[l] [P,64] fp32,
    block_table [B,max_pages] int32, seq_lens [B] int32.
    """
    ctx = decode_context_lengths(spec) if ctx is None else np.asarray(ctx, dtype=np.int64)
    bt, total = page_table(spec, ctx)
    B, R, s = len(ctx), spec.rows_per_seq, spec.seed
    out = {"ctx": ctx, "block_table": bt, "n_pages": total, "k": spec.k, "rows_per_seq": R,
           "softmax_scale": spec.softmax_scale}
    q = _normal(sub_seed(s, 0, T_QIDX), B * IDX_HEADS * IDX_DIM, device)
    out["q_idx"] = _bf16(q, device).reshape(B, IDX_HEADS, IDX_DIM)
    out["w"] = _f32(_normal(sub_seed(s, 0, T_W), B * IDX_HEADS, device), device).reshape(B, IDX_HEADS)
    out["topk_per_row"] = bool(spec.topk_per_row)
    if spec.topk_per_row and R > 1:
        if spec.n_layers > 4:
            raise ValueError("per-row Top-k inputs are drawn for one IndexShare group only")
        qd = _bf16(_normal(sub_seed(s, 0, T_QIDX_DRAFT), B * (R - 1) * IDX_HEADS * IDX_DIM, device), device)
        wd = _f32(_normal(sub_seed(s, 0, T_W_DRAFT), B * (R - 1) * IDX_HEADS, device), device)
        out["q_idx"] = _cat_rows(out["q_idx"], qd.reshape(B, R - 1, IDX_HEADS, IDX_DIM), (B * R, IDX_HEADS, IDX_DIM))
        out["w"] = _cat_rows(out["w"], wd.reshape(B, R - 1, IDX_HEADS), (B * R, IDX_HEADS))
    out["idx_keys"], out["idx_key_scale"] = _fp8_pool(sub_seed(s, 0, T_KIDX), total, IDX_DIM, device)
    layers = range(spec.n_layers) if layers is None else layers
    out["Q"], out["KV"], out["KV_scale"] = [], [], []
    for l in layers:
        out["Q"].append(_bf16(_normal(sub_seed(s, l, T_Q), B * R * MLA_HEADS * D_QK, device), device)
                        .reshape(B * R, MLA_HEADS, D_QK))
        c, sc = _fp8_pool(sub_seed(s, l, T_KV), total, D_QK, device)
        out["KV"].append(c)
        out["KV_scale"].append(sc)
    return out

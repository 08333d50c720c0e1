"""Full-size workloads in the launch configuration the benchmark times, checked on sampled
rows that the fp64 oracle computes one by one (needs a B200).

* prefill_32k       L=32,768, Top-2048, bf16 indexer with AR(1) keys, 4 layers
* prefill_128k_fp8  L=131,072, Top-2048, FP8 indexer quantised on the path, 4 layers
* decode_b32_mtp4   32 sequences of 65K..262K tokens, 5 rows each, paged FP8 caches
* decode_1m_mtp5    1 sequence of 1,048,576 tokens, 6 rows, the 78-layer schedule (21 groups)
Tolerances as in test_gpu_kernels.py / test_gpu_group.py.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_sparse_11_b200 as dsa  # noqa: E402
import oracle.dsa_oracle as O  # noqa: E402
from synth import make_prefill, make_decode, WORKLOADS  # noqa: E402
from test_gpu_kernels import check_topk_sets, attn_errors  # noqa: E402


def host_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


def _prefill(name):
    spec = WORKLOADS[name]
    inp = make_prefill(spec, device="cuda")
    g = dsa.IndexShareGroup(inp["q_idx"], inp["w"], dsa.dense_view(inp["k_idx"]), spec.k, inp["Q"],
                            [dsa.dense_view(x) for x in inp["KV"]], inp["softmax_scale"],
                            indexer_dtype=dsa.DSA_E4M3 if spec.indexer_fp8 else dsa.DSA_BF16)
    out, lse = g.forward()
    dsa.sync_status()
    return spec, inp, g, out


def _sample_rows(L, k, n_random, seed):
    fixed = [0, 1, k - 1, k, k + 1, L // 2, L - 2, L - 1]
    rnd = np.random.default_rng(seed).integers(0, L, size=n_random)
    return sorted(set(fixed + [int(r) for r in rnd]))


@pytest.mark.parametrize("name", ["prefill_32k", "prefill_128k_fp8"])
def test_fullsize_prefill_sampled_rows(name):
    spec, inp, g, out = _prefill(name)
    L, k = spec.L, spec.k
    rows = _sample_rows(L, k, 6 if spec.indexer_fp8 else 10, 17)
    idx = g.idx.cpu().numpy()
    host = {"L": L, "k": k, "softmax_scale": spec.softmax_scale, "k_idx": host_bits(inp["k_idx"]),
            "q_idx": {t: host_bits(inp["q_idx"][t]) for t in rows},
            "w": {t: inp["w"][t].cpu().numpy() for t in rows},
            "Q": [{t: host_bits(q[t]) for t in rows} for q in inp["Q"]],
            "KV": [host_bits(x) for x in inp["KV"]]}
    # Top-k: exact up to swaps within the tolerance band, against the oracle on the path's inputs
    if spec.indexer_fp8:
        k8, sk = O.quantize_e4m3_rows(host["k_idx"], 128)
        kv = O.e4m3_to_f64(k8) * sk.reshape(-1, 1)
    else:
        kv = O.bf16_to_f64(host["k_idx"])
    for t in rows:
        if spec.indexer_fp8:
            q8, sq = O.quantize_e4m3_rows(host["q_idx"][t][None], 128)
            qv = O.e4m3_to_f64(q8) * sq.reshape(1, 32, 1)
        else:
            qv = O.bf16_to_f64(host["q_idx"][t][None])
        sc = O.indexer_scores(qv, host["w"][t][None].astype(np.float64), kv, [t + 1])[0]
        check_topk_sets(idx[t], sc, t + 1, k)
    # attention on the GPU's own indices, every layer
    tables = O.prefill_tables(host, spec.indexer_fp8)
    ref = O.group_prefill(host, rows, fp8_indexer=spec.indexer_fp8, idx_override={t: idx[t] for t in rows},
                          tables=tables)
    for l in range(4):
        o = {t: O.bf16_to_f64(host_bits(out[l][t])) for t in rows}
        for t in rows:
            ma, rl = attn_errors(o[t], ref["O"][l][t])
            assert ma <= 2e-2 and rl <= 5e-3, (name, l, t, ma, rl)
    if spec.indexer_fp8:   # end to end against the oracle's own selection on the same inputs
        own = O.group_prefill(host, rows, fp8_indexer=True, tables=tables)
        num = den = 0.0
        for l in range(4):
            for t in rows:
                o = O.bf16_to_f64(host_bits(out[l][t]))
                num += np.sum((o - own["O"][l][t]) ** 2)
                den += np.sum(own["O"][l][t] ** 2)
        assert math.sqrt(num / den) <= 3e-2


def test_fullsize_decode_b32_mtp4():
    spec = WORKLOADS["decode_b32_mtp4"]
    inp = make_decode(spec, device="cuda")
    ctx_d = torch.from_numpy(inp["ctx"].astype(np.int32)).cuda()
    bt_d = torch.from_numpy(inp["block_table"]).cuda()
    keys = dsa.paged_view(inp["idx_keys"], inp["idx_key_scale"], bt_d, ctx_d)
    kvs = [dsa.paged_view(inp["KV"][l], inp["KV_scale"][l], bt_d, ctx_d) for l in range(4)]
    g = dsa.IndexShareGroup(inp["q_idx"], inp["w"], keys, spec.k, inp["Q"], kvs, inp["softmax_scale"],
                            indexer_dtype=dsa.DSA_E4M3, q_rows_per_idx_row=spec.rows_per_seq)
    out, _ = g.forward()
    dsa.sync_status()
    idx = g.idx.cpu().numpy()
    seqs = [0, 7, 19, 31]
    bt = inp["block_table"]
    qidx = host_bits(inp["q_idx"])
    q8, sq = O.quantize_e4m3_rows(qidx, 128)
    qv = O.e4m3_to_f64(q8) * sq.reshape(-1, 32, 1)
    pool, pscale = inp["idx_keys"].cpu().numpy(), inp["idx_key_scale"].cpu().numpy()
    w = inp["w"].cpu().numpy()
    for b in seqs:
        n = int(inp["ctx"][b])
        kk = O.paged_rows(pool, pscale, bt[b], n)
        sc = O.indexer_scores(qv[b:b + 1], w[b:b + 1], kk, [n])[0]
        check_topk_sets(idx[b], sc, n, spec.k)
    R = spec.rows_per_seq
    for l in (0, 3):
        kvp, kvs_ = inp["KV"][l].cpu().numpy(), inp["KV_scale"][l].cpu().numpy()
        o = O.bf16_to_f64(host_bits(out[l]))
        Q = host_bits(inp["Q"][l])
        for b in seqs:
            sel = idx[b][idx[b] >= 0]
            pages, slots = bt[b][sel // 64], sel % 64      # only the selected rows are dequantised
            rows_kv = O.e4m3_to_f64(kvp[pages, slots]) * kvs_[pages, slots].astype(np.float64)[:, None]
            for r in range(R):
                row = b * R + r
                ref, _ = O.sparse_mla_row(O.bf16_to_f64(Q[row]), rows_kv, np.arange(len(sel)), spec.softmax_scale)
                ma, rl = attn_errors(o[row], ref)
                assert ma <= 2e-2 and rl <= 5e-3, (l, row, ma, rl)


def test_fullsize_decode_1m_mtp5_78_layer_schedule():
    """decode_1m_mtp5: one sequence of 1,048,576 tokens, 1 + 5 rows, the 78-layer schedule run as
    21 IndexShare groups exactly as the benchmark runs them.  Checked: each group's handle comes
    from its own Full layer; the Top-k sets of Full layers 0, 2 and 74 against the oracle on the
    path's e4m3 keys; and all 6 rows of layers 0, 1, 5 and 77 (Full, Full, Shared of 2, Shared of
    74) against the oracle on the GPU's indices."""
    from synth import make_decode_indexer
    spec = WORKLOADS["decode_1m_mtp5"]
    inp = make_decode(spec, device="cuda")
    n, R = int(inp["ctx"][0]), spec.rows_per_seq
    ctx_d = torch.from_numpy(inp["ctx"].astype(np.int32)).cuda()
    bt_d = torch.from_numpy(inp["block_table"]).cuda()
    kvs = [dsa.paged_view(inp["KV"][l], inp["KV_scale"][l], bt_d, ctx_d) for l in range(spec.n_layers)]
    fulls = [l for l in range(spec.n_layers) if dsa.layer_is_full(l)]
    assert len(fulls) == 21
    groups, indexers = {}, {}
    for f, e in zip(fulls, fulls[1:] + [spec.n_layers]):
        ind = inp if f == 0 else make_decode_indexer(spec, f, inp["n_pages"], 1, "cuda")
        keys = dsa.paged_view(ind["idx_keys"], ind["idx_key_scale"], bt_d, ctx_d)
        g = dsa.IndexShareGroup(ind["q_idx"], ind["w"], keys, spec.k, inp["Q"][f:e], kvs[f:e], inp["softmax_scale"],
                                indexer_dtype=dsa.DSA_E4M3, q_rows_per_idx_row=R, first_layer=f)
        g.forward()
        groups[f] = g
        if f in (0, 2, 74):
            indexers[f] = ind
    dsa.sync_status()
    for f, g in groups.items():
        assert g.handle.filled == 1 and g.handle.producer_layer == f and g.handle.generation == 1
    bt = inp["block_table"]
    for f, ind in indexers.items():
        q8, sq = O.quantize_e4m3_rows(host_bits(ind["q_idx"]), 128)
        qv = O.e4m3_to_f64(q8) * sq.reshape(-1, 32, 1)
        kk = O.paged_rows(ind["idx_keys"].cpu().numpy(), ind["idx_key_scale"].cpu().numpy(), bt[0], n)
        sc = O.indexer_scores(qv, ind["w"].cpu().numpy().astype(np.float64), kk, [n])[0]
        check_topk_sets(groups[f].idx[0].cpu().numpy(), sc, n, spec.k)
        del kk, sc
    for l in (0, 1, 5, 77):
        f = dsa.layer_producer(l)
        idx = groups[f].idx[0].cpu().numpy()
        sel = idx[idx >= 0]
        pages, slots = bt[0][sel // 64], sel % 64
        kvp = inp["KV"][l][torch.from_numpy(pages.astype(np.int64)).cuda(),
                           torch.from_numpy(slots.astype(np.int64)).cuda()].cpu().numpy()
        kvs_ = inp["KV_scale"][l][torch.from_numpy(pages.astype(np.int64)).cuda(),
                                  torch.from_numpy(slots.astype(np.int64)).cuda()].cpu().numpy()
        rows_kv = O.e4m3_to_f64(kvp) * kvs_.astype(np.float64)[:, None]
        o = O.bf16_to_f64(host_bits(groups[f].out[l - f]))
        Q = host_bits(inp["Q"][l])
        for r in range(R):
            ref, _ = O.sparse_mla_row(O.bf16_to_f64(Q[r]), rows_kv, np.arange(len(sel)), spec.softmax_scale)
            ma, rl = attn_errors(o[r], ref)
            assert ma <= 2e-2 and rl <= 5e-3, (l, r, ma, rl)
    del groups, inp, kvs
    torch.cuda.empty_cache()

"""Context-parallel prefill on one GPU with 3 ranks emulated in one process (needs a B200): each
rank's two zigzag chunks run as IndexShare group calls over the gathered caches; every row's
selection must equal the single-call selection exactly (the scores of a row do not depend on the
chunking), and its attention must match the single call and the fp64 oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_sparse_11_b200 as dsa  # noqa: E402
import oracle.dsa_oracle as O  # noqa: E402
from long_context_sparse_11_b200 import cp  # noqa: E402
from long_context_sparse_11_b200.splitn import run_emulated  # noqa: E402
from synth import make_prefill, PrefillSpec  # noqa: E402
from test_gpu_kernels import bf16_dev, f32_dev, bf16_host, attn_errors  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


@pytest.mark.parametrize("fp8", [False, True])
def test_context_parallel_prefill_over_three_emulated_ranks(fp8):
    spec = PrefillSpec("cp", L=3001, k=256, n_layers=2, seed=43, indexer_fp8=fp8)
    inp = make_prefill(spec)
    L, G = spec.L, 3
    dt = dsa.DSA_E4M3 if fp8 else dsa.DSA_BF16
    dev = {"q_idx": bf16_dev(inp["q_idx"]), "w": f32_dev(inp["w"]), "k_idx": bf16_dev(inp["k_idx"]),
           "Q": [bf16_dev(q) for q in inp["Q"]], "KV": [bf16_dev(x) for x in inp["KV"]]}
    c = -(-L // (2 * G))
    rows = []
    for r in range(G):
        sel = torch.zeros(2 * c, dtype=torch.long)
        for slot, (lo, n) in enumerate(cp.zigzag_chunks(L, G, r)):
            sel[slot * c:slot * c + n] = torch.arange(lo, lo + n)
        sel = sel.cuda()

        def take(x):
            return x[sel].contiguous()
        rows.append(cp.RankRows(L=L, G=G, rank=r, q_idx=take(dev["q_idx"]), w=take(dev["w"]), k_idx=take(dev["k_idx"]),
                                q=[take(q) for q in dev["Q"]], kv=[take(x) for x in dev["KV"]], k=spec.k,
                                softmax_scale=inp["softmax_scale"], indexer_dtype=dt))
    res = run_emulated(cp.DeviceOps(), rows, lambda parts: torch.stack(parts), step=cp.group_step)
    dsa.sync_status()
    full = dsa.IndexShareGroup(dev["q_idx"], dev["w"], dsa.dense_view(dev["k_idx"]), spec.k, dev["Q"],
                               [dsa.dense_view(x) for x in dev["KV"]], inp["softmax_scale"], indexer_dtype=dt)
    out_full, _ = full.forward()
    dsa.sync_status()
    idx_full = full.idx.cpu().numpy()
    o_full = [O.bf16_to_f64(bf16_host(o)) for o in out_full]
    covered = 0
    for rank_res in res:
        for pos0, idx, layers in rank_res:
            idx = idx.cpu().numpy()
            n = idx.shape[0]
            covered += n
            for i in range(n):
                assert sorted(idx[i]) == sorted(idx_full[pos0 + i]), pos0 + i
            for l, (o, _) in enumerate(layers):
                o = O.bf16_to_f64(bf16_host(o))
                ma, rel = attn_errors(o, o_full[l][pos0:pos0 + n])
                assert ma <= 2e-2 and rel <= 5e-3, (pos0, l, ma, rel)
                for i in (0, n // 2, n - 1):                      # and the oracle on sampled rows
                    ref, _ = O.sparse_mla_row(O.bf16_to_f64(inp["Q"][l][pos0 + i]), O.bf16_to_f64(inp["KV"][l]),
                                              idx[i], inp["softmax_scale"])
                    ma, rel = attn_errors(o[i], ref)
                    assert ma <= 2e-2 and rel <= 5e-3, (pos0 + i, l, ma, rel)
    assert covered == L

"""Split-N decode on one GPU with the ranks emulated in one process (needs a B200): each of 4
slices of a 50,000-token sequence is scored, selected and attended by the CUDA library, and the
candidates and partial results are merged by its split-N kernels.  The merged Top-k must be the
unsplit GPU Top-k exactly (the scores of a key do not depend on the slicing), the same on every
rank, and the combined attention must match the fp64 oracle over the whole sequence."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_sparse_11_b200 as dsa  # noqa: E402
import oracle.dsa_oracle as O  # noqa: E402
from long_context_sparse_11_b200.splitn import RankSlice, DeviceOps, run_emulated  # noqa: E402
from synth import make_decode, DecodeSpec  # noqa: E402
from test_gpu_kernels import bf16_dev, u8_dev, f32_dev, i32_dev, bf16_host, attn_errors  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


def test_split_n_over_four_emulated_ranks():
    spec = DecodeSpec("split", batch=1, ctx_lo=1, ctx_hi=1, rows_per_seq=3, k=512, n_layers=2, seed=37,
                      fixed_ctx=50000)
    inp = make_decode(spec)
    N, R, k = 50000, spec.rows_per_seq, spec.k
    bt = inp["block_table"][0]
    keys_pool, keys_scale = u8_dev(inp["idx_keys"]), f32_dev(inp["idx_key_scale"])
    kv_pools = [(u8_dev(inp["KV"][l]), f32_dev(inp["KV_scale"][l])) for l in range(2)]
    q_idx, w = bf16_dev(inp["q_idx"]), f32_dev(inp["w"])
    Q = [bf16_dev(x) for x in inp["Q"]]
    bounds = [0, 12800, 12864, 31040, N]              # page-aligned; one slice of a single page
    slices = []
    for r in range(4):
        lo, hi = bounds[r], bounds[r + 1]
        pages = i32_dev(bt[lo // 64:(hi + 63) // 64][None])
        lens = i32_dev(np.array([hi - lo]))
        slices.append(RankSlice(lo=lo, hi=hi, q_idx=q_idx, w=w,
                                keys=dsa.paged_view(keys_pool, keys_scale, pages, lens), seq_lens=lens, q=Q,
                                kv=[dsa.paged_view(p, s, pages, lens) for p, s in kv_pools], k=k,
                                rows_per_idx_row=R, softmax_scale=inp["softmax_scale"]))
    res = run_emulated(DeviceOps(), slices, lambda parts: torch.stack(parts))
    dsa.sync_status()
    # the unsplit selection on the same GPU
    full_lens = i32_dev(np.array([N]))
    full_keys = dsa.paged_view(keys_pool, keys_scale, i32_dev(bt[None]), full_lens)
    scores = torch.empty(1, (len(bt) * 64 + 3) // 4 * 4, dtype=torch.float32, device="cuda")
    q8, qs = dsa.quant_e4m3(q_idx)
    dsa.indexer_score(q8, w, full_keys, scores, q_scale=qs)
    full = dsa.topk(scores, k, row_len=full_lens, max_len=N).cpu().numpy()[0]
    idx0 = res[0][0].cpu().numpy()[0]
    assert sorted(idx0) == sorted(full)
    for idx, _ in res[1:]:                       # every rank holds the same set (order unspecified)
        assert sorted(idx.cpu().numpy()[0]) == sorted(idx0)
    for l in range(2):
        rows_kv = O.paged_rows(inp["KV"][l], inp["KV_scale"][l], bt, N)
        o, lse = res[0][1][l]
        o = O.bf16_to_f64(bf16_host(o))
        lse = lse.cpu().numpy()
        for r in range(R):
            ref, ref_lse = O.sparse_mla_row(O.bf16_to_f64(inp["Q"][l][r]), rows_kv, idx0, inp["softmax_scale"])
            ma, rel = attn_errors(o[r], ref)
            assert ma <= 2e-2 and rel <= 5e-3, (l, r, ma, rel)
            assert np.max(np.abs(lse[r] - ref_lse)) <= 2e-3

"""Split-N decode of one sequence over 2 ranks (gloo, CPU): the orchestration of
long_context_sparse_11_b200.splitn run by two processes with the oracle standing in for the CUDA
steps.  Every rank must end with the unsplit Top-k, bit for bit (same fp64 scores, same rank
rule), and the combined attention must equal the unsplit oracle's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle.dsa_oracle as O
from synth import make_decode, DecodeSpec

SPEC = DecodeSpec("split", batch=1, ctx_lo=1, ctx_hi=1, rows_per_seq=3, k=64, n_layers=2, seed=31,
                  fixed_ctx=5000)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _slice(inp, lo, hi, rank_rows=1):
    from long_context_sparse_11_b200.splitn import RankSlice
    bt = inp["block_table"][0]
    pages = bt[lo // 64:(hi + 63) // 64]
    R = inp["rows_per_seq"]
    return RankSlice(lo=lo, hi=hi, q_idx=inp["q_idx"][:rank_rows], w=inp["w"][:rank_rows],
                     keys=(inp["idx_keys"], inp["idx_key_scale"], pages, hi - lo), seq_lens=None,
                     q=[q[:rank_rows * R] for q in inp["Q"]],
                     kv=[(inp["KV"][l], inp["KV_scale"][l], pages, hi - lo) for l in range(len(inp["Q"]))],
                     k=inp["k"], rows_per_idx_row=R, softmax_scale=inp["softmax_scale"])


BOUNDS = [0, 1984, 5000]        # page-aligned split of 5,000 positions over 2 ranks


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))
    try:
        from long_context_sparse_11_b200.splitn import run_distributed, torch_all_gather
        from splitn_oracle_ops import OracleOps
        inp = make_decode(SPEC)
        s = _slice(inp, BOUNDS[rank], BOUNDS[rank + 1])

        def gather(a):
            return torch_all_gather(torch.from_numpy(np.ascontiguousarray(a))).numpy()

        idx, results = run_distributed(OracleOps(), s, gather)
        np.save(os.path.join(out, f"idx{rank}.npy"), idx)
        for l, (o, lse) in enumerate(results):
            np.save(os.path.join(out, f"o{rank}_{l}.npy"), o)
            np.save(os.path.join(out, f"lse{rank}_{l}.npy"), lse)
    finally:
        dist.destroy_process_group()


def test_two_rank_split_n_equals_unsplit_oracle(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    inp = make_decode(SPEC)
    ref = O.group_decode(inp)
    for rank in range(2):
        idx = np.load(tmp_path / f"idx{rank}.npy")
        assert np.array_equal(idx[0], ref["idx"][0])            # same positions, same order
        for l in range(2):
            o = np.load(tmp_path / f"o{rank}_{l}.npy")
            lse = np.load(tmp_path / f"lse{rank}_{l}.npy")
            for r in range(SPEC.rows_per_seq):
                assert np.max(np.abs(o[r] - ref["O"][l][r])) < 1e-10
                assert np.max(np.abs(lse[r] - ref["lse"][l][r])) < 1e-10
    # both ranks hold selected positions: the test exercises a real merge and a real combine
    sel = ref["idx"][0]
    assert (sel < BOUNDS[1]).any() and (sel >= BOUNDS[1]).any()


def test_emulated_ranks_with_a_slice_that_holds_no_selection():
    """Four ranks in one process (the single-GPU driver), one of whose slices is a single page:
    its part has no selected position (lse = -inf) and must drop out of the combination."""
    from long_context_sparse_11_b200.splitn import run_emulated
    from splitn_oracle_ops import OracleOps
    inp = make_decode(SPEC)
    ref = O.group_decode(inp)
    sel = set(int(i) for i in ref["idx"][0])
    page = next(p for p in range(20, 70) if not any(64 * p <= i < 64 * p + 64 for i in sel))
    bounds = [0, 1216, 64 * page, 64 * page + 64, 5000]          # rank 2 holds one unselected page
    assert 1216 < 64 * page
    slices = [_slice(inp, bounds[r], bounds[r + 1]) for r in range(4)]
    res = run_emulated(OracleOps(), slices, lambda parts: np.stack(parts))
    for idx, results in res:
        assert np.array_equal(idx[0], ref["idx"][0])
        for l in range(2):
            for r in range(SPEC.rows_per_seq):
                assert np.max(np.abs(results[l][0][r] - ref["O"][l][r])) < 1e-10

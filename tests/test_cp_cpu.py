"""Context-parallel prefill over 2 ranks (gloo, CPU): long_context_sparse_11_b200.cp run by two
processes with the oracle standing in for the library's group call.  The zigzag chunks must cover
every row once, and every row's selection and attention must equal the single-rank oracle's."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import oracle.dsa_oracle as O
from long_context_sparse_11_b200 import cp
from synth import make_prefill, PrefillSpec

SPEC = PrefillSpec("cp", L=101, k=16, n_layers=2, seed=41)


class OracleCpOps:
    @staticmethod
    def assemble(stacked, ranks, rows):
        return np.asarray(stacked)[np.asarray(ranks), np.asarray(rows)]

    def group(self, s, row0, n, pos0, keys, kvs):
        inp = {"L": pos0 + n, "k": s.k, "softmax_scale": s.softmax_scale, "k_idx": keys[:pos0 + n],
               "q_idx": {pos0 + i: s.q_idx[row0 + i] for i in range(n)},
               "w": {pos0 + i: s.w[row0 + i] for i in range(n)},
               "Q": [{pos0 + i: q[row0 + i] for i in range(n)} for q in s.q], "KV": [x[:pos0 + n] for x in kvs]}
        rows = range(pos0, pos0 + n)
        g = O.group_prefill(inp, rows)
        idx = np.stack([g["idx"][t] for t in rows])
        return idx, [(np.stack([g["O"][l][t] for t in rows]), np.stack([g["lse"][l][t] for t in rows]))
                     for l in range(len(s.q))]


def rank_rows(inp, G, r):
    c = -(-inp["L"] // (2 * G))

    def take(x):
        x = np.asarray(x)
        out = np.zeros((2 * c,) + x.shape[1:], dtype=x.dtype)
        for slot, (lo, n) in enumerate(cp.zigzag_chunks(inp["L"], G, r)):
            out[slot * c:slot * c + n] = x[lo:lo + n]
        return out
    return cp.RankRows(L=inp["L"], G=G, rank=r, q_idx=take(inp["q_idx"]), w=take(inp["w"]), k_idx=take(inp["k_idx"]),
                       q=[take(q) for q in inp["Q"]], kv=[take(x) for x in inp["KV"]], k=inp["k"],
                       softmax_scale=inp["softmax_scale"])


def test_zigzag_chunks_cover_every_row_once():
    for L, G in [(101, 2), (96, 3), (7, 4), (131072, 8)]:
        seen = np.zeros(L, dtype=int)
        work = []
        for r in range(G):
            w = 0
            for lo, n in cp.zigzag_chunks(L, G, r):
                seen[lo:lo + n] += 1
                w += sum(range(lo + 1, lo + n + 1))          # causal keys of the rows
            work.append(w)
        assert (seen == 1).all()
        if L >= 1000:
            assert max(work) / min(work) < 1.01               # early + late chunk: balanced causal work
        ranks, rows = cp.position_map(L, G)
        assert len(set(zip(ranks, rows))) == L


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))
    try:
        from long_context_sparse_11_b200.splitn import run_distributed, torch_all_gather
        inp = make_prefill(SPEC)

        def gather(a):  # gloo carries no 16-bit integers: bf16 bit patterns travel as int32
            a = np.ascontiguousarray(a)
            t = torch.from_numpy(a.astype(np.int32) if a.dtype == np.uint16 else a)
            return torch_all_gather(t).numpy().astype(a.dtype)

        res = run_distributed(OracleCpOps(), rank_rows(inp, ws, rank), gather, step=cp.group_step)
        for pos0, idx, layers in res:
            np.save(os.path.join(out, f"idx_{pos0}.npy"), idx)
            for l, (o, lse) in enumerate(layers):
                np.save(os.path.join(out, f"o_{pos0}_{l}.npy"), o)
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_prefill_equals_single_rank(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    inp = make_prefill(SPEC)
    ref = O.group_prefill(inp, range(SPEC.L))
    done = 0
    for r in range(2):
        for pos0, n in cp.zigzag_chunks(SPEC.L, 2, r):
            idx = np.load(tmp_path / f"idx_{pos0}.npy")
            for i in range(n):
                assert np.array_equal(idx[i], ref["idx"][pos0 + i])
                for l in range(2):
                    assert np.array_equal(np.load(tmp_path / f"o_{pos0}_{l}.npy")[i], ref["O"][l][pos0 + i])
            done += n
    assert done == SPEC.L

"""Context-parallel prefill of one sequence over G ranks, one process per GPU.

The L query rows are cut into 2G equal chunks and rank r takes chunks r and 2G - 1 - r: an early
and a late chunk, so that every rank has about the same causal work (a row at position t scores
t + 1 keys).  Each rank holds the indexer keys and the latent rows of its own tokens only.  One
IndexShare group step, on every rank:

1. all-gather the indexer keys and every layer's latent rows of all ranks' tokens, and lay them out
   in position order: the whole sequence's caches (the only data that crosses ranks);
2. for each of its chunks, one IndexShare group call: the chunk's rows at their positions, causal
   over the gathered caches (indexer + Top-k, then sparse MLA for every layer of the group).

A row's scores, selection and attention do not depend on which rank computes it, so the result is
the single-GPU result row by row.  The step is a generator that yields at each all-gather, run by
``splitn.run_distributed(ops, rows, all_gather, step=cp.group_step)`` (torch.distributed, NCCL on
GPUs) or ``splitn.run_emulated(..., step=cp.group_step)`` (all ranks in one process).  ``DeviceOps`` supplies the library's group call; any object with the
same two methods can stand in for it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import binding as dsa


def zigzag_chunks(L: int, G: int, r: int):
    """(position of the first row, rows) of rank r's two chunks of 2G near-equal chunks of L rows."""
    c = -(-L // (2 * G))
    out = []
    for j in (r, 2 * G - 1 - r):
        lo = min(j * c, L)
        out.append((lo, min((j + 1) * c, L) - lo))
    return out


def position_map(L: int, G: int):
    """For the all-gathered [G, 2c, ...] stack (rank r's rows: its first chunk, then its second,
    each padded to c rows): the (rank, local row) of every position 0..L-1, as two lists."""
    c = -(-L // (2 * G))
    ranks, rows = [0] * L, [0] * L
    for r in range(G):
        for slot, (lo, n) in enumerate(zigzag_chunks(L, G, r)):
            for i in range(n):
                ranks[lo + i], rows[lo + i] = r, slot * c + i
    return ranks, rows


@dataclass
class RankRows:
    """One rank's share of a prefill: its two chunks' rows of every input (each chunk padded to c
    rows), the sequence length and the group's settings."""
    L: int
    G: int
    rank: int
    q_idx: object            # [2c, 32, 128] bf16 indexer query rows
    w: object                # [2c, 32] fp32
    k_idx: object            # [2c, 128] bf16 indexer keys of this rank's tokens
    q: list                  # per layer: [2c, 64, 576] bf16
    kv: list                 # per layer: [2c, 576] bf16 latent rows of this rank's tokens
    k: int = 2048
    softmax_scale: float = 1.0 / 24.0
    indexer_dtype: int = dsa.DSA_BF16
    extra: dict = field(default_factory=dict)

    @property
    def chunks(self):
        return zigzag_chunks(self.L, self.G, self.rank)


def group_step(ops, s: RankRows):
    """The context-parallel group step of one rank (a generator: yields this rank's rows of a
    tensor, receives the [G, ...] stack).  Returns [(pos0, idx, [(out, lse) per layer]) per chunk]."""
    keys_all = yield s.k_idx
    kv_all = []
    for kv in s.kv:
        kv_all.append((yield kv))
    ranks, rows = position_map(s.L, s.G)
    keys = ops.assemble(keys_all, ranks, rows)
    kvs = [ops.assemble(x, ranks, rows) for x in kv_all]
    c = -(-s.L // (2 * s.G))
    results = []
    for slot, (pos0, n) in enumerate(s.chunks):
        if n == 0:
            continue
        results.append((pos0,) + ops.group(s, slot * c, n, pos0, keys, kvs))
    return results


class DeviceOps:
    """The library's group call over the gathered caches (device tensors on the current GPU)."""

    @staticmethod
    def assemble(stacked, ranks, rows):
        """[G, 2c, ...] gathered rows -> [L, ...] in position order (one gather copy)."""
        import torch
        r = torch.as_tensor(ranks, device=stacked.device, dtype=torch.long)
        i = torch.as_tensor(rows, device=stacked.device, dtype=torch.long)
        return stacked[r, i].contiguous()

    def group(self, s: RankRows, row0: int, n: int, pos0: int, keys, kvs):
        sl = slice(row0, row0 + n)
        g = dsa.IndexShareGroup(s.q_idx[sl], s.w[sl], dsa.dense_view(keys[:pos0 + n]), s.k, [q[sl] for q in s.q],
                                [dsa.dense_view(x[:pos0 + n]) for x in kvs], s.softmax_scale,
                                indexer_dtype=s.indexer_dtype, q_pos0=pos0)
        out, lse = g.forward()
        s.extra.setdefault("groups", []).append(g)   # keeps the outputs' buffers alive
        return g.idx, list(zip(out, lse))

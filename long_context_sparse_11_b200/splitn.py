"""Split-N decode of one long sequence over G ranks, one process per GPU.

Rank r holds the cache positions [lo_r, hi_r) of the sequence (its own pages of the indexer-key
and latent caches).  One IndexShare group step, on every rank:

1. a2-a4 on its slice: indexer scores of the slice's keys and their local Top-k;
2. its local Top-k as (score, global position) candidates, ordered by position;
3. gather every rank's candidates (rank order) and merge them into the sequence's Top-k, the
   same on every rank and equal to the unsplit Top-k (the best k of all keys are among the best k
   of their own slice; equal scores go to the lower position in both);
4. for every layer of the group, attention over the selected positions inside its slice
   (positions elsewhere are -1), with the log-sum-exp of its part;
5. gather every rank's (out, lse) and combine: out = sum_r exp(lse_r - lse) out_r.

Only candidates (2 x k values per index row per rank) and partial results cross ranks; no cache
row moves.  The step is written once, as a generator that yields at each collective, and run by
one of two drivers: ``run_distributed`` (torch.distributed all-gather, NCCL on GPUs) or
``run_emulated`` (all ranks in one process, one after another; what a single GPU can test); the
drivers also run other step generators (``cp.group_step``).
``DeviceOps`` supplies the steps from the CUDA library; any object with the same five methods
can stand in for it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import binding as dsa


@dataclass
class RankSlice:
    """One rank's share of a sequence: positions [lo, hi), its paged views, its query rows."""
    lo: int
    hi: int
    q_idx: object              # [rows, 32, 128] bf16 indexer query rows (row 0 of each step)
    w: object                  # [rows, 32] fp32 head weights
    keys: object               # paged view of this slice's indexer keys (batch = rows)
    seq_lens: object           # [rows] int32, every entry hi - lo (the views' lengths)
    q: list                    # per layer: [rows * R, 64, 576] bf16 query rows
    kv: list                   # per layer: paged view of this slice's latent rows (batch = rows)
    k: int = 2048
    rows_per_idx_row: int = 1
    softmax_scale: float = 1.0 / 24.0
    scratch: dict = field(default_factory=dict)

    @property
    def n_local(self) -> int:
        return self.hi - self.lo


def group_step(ops, s: RankSlice):
    """The split-N group step of one rank (a generator: yields a tensor to all-gather, receives the
    gathered [G, ...] stack).  Returns (idx_global [rows, k], [(out, lse) per layer])."""
    scores, idx_local = ops.score_topk(s)
    cs, ci = ops.candidates(s, scores, idx_local)
    cs_all = yield cs
    ci_all = yield ci
    idx_global, idx_here = ops.merge(s, ops.rank_major(cs_all), ops.rank_major(ci_all))
    results = []
    for layer in range(len(s.q)):
        out, lse = ops.attend(s, layer, idx_here)
        o_all = yield out
        l_all = yield lse
        results.append(ops.combine(o_all, l_all))
    return idx_global, results


def run_distributed(ops, s, all_gather, step=None):
    """Drive one rank's step (``group_step`` unless another step generator is given);
    all_gather(t) -> [G, *t.shape] stack in rank order (collective)."""
    gen = (step or group_step)(ops, s)
    try:
        t = next(gen)
        while True:
            t = gen.send(all_gather(t))
    except StopIteration as stop:
        return stop.value


def run_emulated(ops, slices, stack, step=None):
    """Drive every rank's step in one process, in lock step at each collective; stack(list) ->
    [G, ...].  Returns each rank's result."""
    gens = [(step or group_step)(ops, s) for s in slices]
    pending = [next(g) for g in gens]
    results = [None] * len(gens)
    while any(r is None for r in results):
        gathered = stack(pending)
        for i, g in enumerate(gens):
            try:
                pending[i] = g.send(gathered)
            except StopIteration as stop:
                results[i] = stop.value
    return results


def torch_all_gather(t):
    """all_gather over the default process group (NCCL or gloo), stacked in rank order."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, t.contiguous())
    return torch.stack(parts)


class DeviceOps:
    """The five steps from the CUDA library (device tensors on the current GPU)."""

    def score_topk(self, s: RankSlice):
        import torch
        rows = s.q_idx.shape[0]
        ld = (s.keys.max_pages * 64 + 3) // 4 * 4
        scores = s.scratch.get("scores")
        if scores is None or scores.shape != (rows, ld):
            scores = s.scratch["scores"] = torch.empty(rows, ld, dtype=torch.float32, device=s.q_idx.device)
        q8, qs = dsa.quant_e4m3(s.q_idx)
        dsa.indexer_score(q8, s.w, s.keys, scores, q_scale=qs)
        idx = dsa.topk(scores, s.k, row_len=s.seq_lens, max_len=s.n_local)
        return scores, idx

    def candidates(self, s: RankSlice, scores, idx_local):
        return dsa.split_candidates(scores, idx_local, s.n_local, s.lo)

    @staticmethod
    def rank_major(stacked):
        """[G, rows, k] -> [rows, G * k]: each row's candidates of all ranks, rank order."""
        G, rows, k = stacked.shape
        return stacked.permute(1, 0, 2).reshape(rows, G * k).contiguous()

    def merge(self, s: RankSlice, cand_score, cand_idx):
        return dsa.split_merge(cand_score, cand_idx, s.k, s.lo, s.hi)

    def attend(self, s: RankSlice, layer: int, idx_here):
        return dsa.sparse_mla_attn(s.q[layer], s.kv[layer], idx_here, s.k, s.softmax_scale,
                                   q_rows_per_idx_row=s.rows_per_idx_row)

    def combine(self, o_parts, lse_parts):
        return dsa.combine_partials(o_parts, lse_parts)

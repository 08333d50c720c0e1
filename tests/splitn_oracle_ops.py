"""The split-N steps computed by the fp64 oracle (test infrastructure): stands in for the CUDA
library in the CPU tests of the split-N orchestration.  Arrays are numpy; a rank's keys and
latent rows come as (pool, scale, block-table row of its pages, n_local)."""
import numpy as np

import oracle.dsa_oracle as O


class OracleOps:
    def score_topk(self, s):
        pool, scale, bt, n = s.keys
        keys = O.paged_rows(pool, scale, bt, n)
        q8, sq = O.quantize_e4m3_rows(s.q_idx, 128)
        qv = O.e4m3_to_f64(q8) * sq.reshape(-1, 32, 1)
        sc = O.indexer_scores(qv, np.asarray(s.w, dtype=np.float64), keys, [n] * len(qv))
        idx = np.stack([O.topk_row(sc[r], n, s.k) for r in range(len(qv))])
        return sc, idx

    def candidates(self, s, scores, idx_local):
        rows, k = idx_local.shape
        cs, ci = np.full((rows, k), -np.inf), np.full((rows, k), -1, dtype=np.int64)
        for r in range(rows):
            sel = np.sort(idx_local[r][idx_local[r] >= 0])
            cs[r, :len(sel)] = scores[r, sel]
            ci[r, :len(sel)] = s.lo + sel
        return cs, ci

    @staticmethod
    def rank_major(stacked):
        stacked = np.asarray(stacked)
        G, rows, k = stacked.shape
        return stacked.transpose(1, 0, 2).reshape(rows, G * k)

    def merge(self, s, cand_score, cand_idx):
        rows, n_cand = cand_score.shape
        ig = np.full((rows, s.k), -1, dtype=np.int64)
        for r in range(rows):
            pos = O.topk_row(cand_score[r], n_cand, s.k)
            ig[r] = np.where(pos >= 0, cand_idx[r][np.maximum(pos, 0)], -1)
        il = np.where((ig >= s.lo) & (ig < s.hi), ig - s.lo, -1)
        return ig, il

    def attend(self, s, layer, idx_here):
        pool, scale, bt, n = s.kv[layer]
        rows_kv = O.paged_rows(pool, scale, bt, n)
        Q = O.bf16_to_f64(s.q[layer])
        out, lse = np.zeros((len(Q), 64, 512)), np.zeros((len(Q), 64))
        for row in range(len(Q)):
            out[row], lse[row] = O.sparse_mla_row(Q[row], rows_kv, idx_here[row // s.rows_per_idx_row],
                                                  s.softmax_scale)
        return out, lse

    def combine(self, o_parts, lse_parts):
        o_parts, lse_parts = np.asarray(o_parts), np.asarray(lse_parts)
        m = lse_parts.max(axis=0)
        safe_m = np.where(np.isfinite(m), m, 0.0)
        wgt = np.where(np.isfinite(lse_parts), np.exp(lse_parts - safe_m), 0.0)
        L = wgt.sum(axis=0)
        out = (wgt[..., None] * o_parts).sum(axis=0) / np.where(L > 0, L, 1.0)[..., None]
        lse = np.where(L > 0, safe_m + np.log(np.where(L > 0, L, 1.0)), -np.inf)
        return out, lse

"""dsa_topk_no_alloc: Top-k for callers that cannot allocate device memory.

Some callers own no allocator of their own (an engine that reserved the whole device pool
up front) or must not call cudaMalloc / cudaFree because of the device-wide synchronisation
those calls can cause.  This entry point keeps its scratch in a fixed array inside the
library.  Its output must be the oracle's Top-k set and match the workspace-based dsa_topk on
the same scores, on two calls in a row (the second call runs on scratch left over by the
first), for explicit row lengths and for causal rows.  This file is collected last on purpose.
"""
import numpy as np
import pytest

import long_context_sparse_11_b200 as dsa
from long_context_sparse_11_b200 import binding as B
import oracle.dsa_oracle as O


def test_no_alloc_rejects_more_rows_than_its_scratch_holds():
    lib = dsa.load()
    rc = lib.dsa_topk_no_alloc(16, 64, 33, None, 1, 64, 8, 16, None)
    assert rc == B.DSA_ERR_INVALID_ARG
    assert "at most 32 rows" in lib.dsa_last_error().decode()


def _rows(rng, rows, L):
    s = rng.normal(size=(rows, L)).astype(np.float32)
    s[1] = np.round(s[1] * 8) / 8                 # heavy ties
    s[2] = 0.5                                    # one bin holds the whole row
    s[3] = np.where(rng.random(L) < 30000 / L, 0.5, rng.normal(size=L) - 8.0).astype(np.float32)
    # row 3: about 30,000 equal values in the threshold bin, the rest below it (the bin is
    # larger than the 16,384 global candidates, smaller than 65,536)
    return s


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_no_alloc_topk_matches_oracle_and_workspace_topk_on_two_calls(causal):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    rng = np.random.default_rng(5 + causal)
    for call, (rows, L, k) in enumerate([(20, 100000, 2048), (32, 70000, 512)]):
        s = _rows(rng, rows, L)
        ld = (L + 3) // 4 * 4
        buf = np.zeros((rows, ld), dtype=np.float32)
        buf[:, :L] = s
        scores = torch.from_numpy(buf).cuda()
        if causal:
            c0 = L - rows + 1                         # row r holds c0 + r candidates, the last all L
            lens = np.array([c0 + r for r in range(rows)])
            kw = dict(row_len=None, causal_len0=c0, max_len=L)
        else:
            lens = np.array([L - (r * 1013) % (L // 3) for r in range(rows)], dtype=np.int32)
            lens[3] = L
            lens[-1] = k // 2                         # a row shorter than k
            kw = dict(row_len=torch.from_numpy(lens.astype(np.int32)).cuda(), max_len=L)
        ref = dsa.topk(scores, k, **kw)
        out = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
        dsa.topk_no_alloc(scores, k, out, **kw)
        dsa.sync_status()
        a, b = ref.cpu().numpy(), out.cpu().numpy()
        for r in range(rows):
            expect = O.topk_row(s[r].astype(np.float64), int(lens[r]), k)
            assert sorted(b[r]) == sorted(expect), (call, r)
            assert sorted(a[r]) == sorted(b[r]), (call, r)

"""Parity of each CUDA kernel (through the C ABI) with the fp64 oracle, on small seeded
inputs spanning several tiles and ragged tails.  Needs a B200.

Tolerances:
* e4m3 quantisation and Top-k on identical fp32 scores: bit-exact / exact sets.
* indexer scores: |gpu - oracle| <= 2e-5 * max|oracle row| + 1e-6 (fp32 accumulation of
  exact bf16/e4m3 products over 128 dims, then 32 heads).
* Top-k from GPU scores: sets equal except swaps among candidates whose oracle score lies
  within 1e-3 relative (plus 1e-6 of the row's max) of the oracle's k-th score.
* attention (bf16 output): max-abs <= 2e-2 and relative L2 <= 5e-3 against the oracle run
  on the GPU's own indices; LSE within 2e-3.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_sparse_11_b200 as dsa  # noqa: E402
import oracle.dsa_oracle as O  # noqa: E402
from synth import make_prefill, make_decode, PrefillSpec, DecodeSpec, WORKLOADS  # noqa: E402
from synth.generators import bf16_bits_np, e4m3_codes_np, normal_np  # noqa: E402

DEV = "cuda"
SCALE = 1.0 / math.sqrt(576)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def u8_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def i32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def bf16_host(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


def check_topk_sets(gpu_idx, ref_scores, n, k):
    """North-star Top-k criterion for one row; returns number of tolerated swaps."""
    g = [int(i) for i in gpu_idx if i >= 0]
    assert len(g) == min(k, n) and len(set(g)) == len(g), (len(g), n, k)
    assert all(0 <= i < n for i in g)
    assert all(int(i) == -1 for i in gpu_idx[min(k, n):])
    if n <= k:
        assert set(g) == set(range(n))
        return 0
    e = O.topk_row(ref_scores, n, k)
    ks = ref_scores[e[k - 1]]
    band = 1e-3 * abs(ks) + 1e-6 * np.max(np.abs(ref_scores[:n]))
    diff = set(g) ^ set(int(i) for i in e)
    for i in diff:
        assert abs(ref_scores[i] - ks) <= band, (i, ref_scores[i], ks)
    return len(diff) // 2


def attn_errors(o_gpu, o_ref):
    d = o_gpu - o_ref
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-30))


# ----------------------------------------------------------------------------- a1


def test_quant_e4m3_bit_exact():
    n = 1000
    x = normal_np(11, 0, n * 128).reshape(n, 128) * np.exp(normal_np(12, 0, n))[:, None]
    x[3] = 0.0
    x[5, 7] = 3e4
    bits = bf16_bits_np(x)
    codes, scale = dsa.quant_e4m3(bf16_dev(bits))
    torch.cuda.synchronize()
    rc, rs = O.quantize_e4m3_rows(bits, 128)
    assert np.array_equal(scale.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


def test_cache_write_e4m3_bit_exact():
    """Decode-side a1: new rows quantised into their paged slots, bit-exact with the oracle for
    index keys (128) and latent rows (576), other slots untouched; a row whose page is not in the
    block table is skipped and reported."""
    spec = DecodeSpec("c", batch=3, ctx_lo=100, ctx_hi=700, rows_per_seq=1, k=8, n_layers=1, seed=12)
    inp = make_decode(spec)
    bt, ctx = inp["block_table"], inp["ctx"]
    rng = np.random.default_rng(3)
    for dim, pool, scale in ((128, inp["idx_keys"], inp["idx_key_scale"]), (576, inp["KV"][0], inp["KV_scale"][0])):
        pairs = sorted({(int(b), int(t)) for b, t in zip(rng.integers(0, 3, 80), rng.integers(0, 100, 80))})[:40]
        seq = np.array([q[0] for q in pairs], dtype=np.int32)
        pos = np.array([q[1] for q in pairs], dtype=np.int32)
        x = normal_np(20 + dim, 0, len(pairs) * dim).reshape(-1, dim) * 3.0
        x[5] = 0.0                      # all-zero row: scale 1
        x[7, 3] = 2e4                   # one large element: the rest of its row rounds to small codes
        bits = bf16_bits_np(x)
        ref_pool, ref_scale = O.cache_write_e4m3(pool, scale, bt, bits, seq, pos)
        pool_d, scale_d = u8_dev(pool), f32_dev(scale)
        dsa.cache_write_e4m3(bf16_dev(bits), i32_dev(pos), i32_dev(bt), pool_d, scale_d, seq=i32_dev(seq))
        dsa.sync_status()
        assert np.array_equal(pool_d.cpu().numpy(), ref_pool)
        assert np.array_equal(scale_d.cpu().numpy(), ref_scale)
    # sequence 0 at a position past its pages (block-table entry -1): skipped and reported
    t_out = int((ctx[0] + 63) // 64) * 64   # first logical page past the sequence (or past max_pages)
    seq = np.array([0, 1], dtype=np.int32)
    pos = np.array([t_out, 5], dtype=np.int32)
    bits = bf16_bits_np(normal_np(40, 0, 2 * 128).reshape(2, 128))
    pool_d, scale_d = u8_dev(inp["idx_keys"]), f32_dev(inp["idx_key_scale"])
    dsa.cache_write_e4m3(bf16_dev(bits), i32_dev(pos), i32_dev(bt), pool_d, scale_d, seq=i32_dev(seq))
    with pytest.raises(dsa.DsaError) as err:
        dsa.sync_status()
    assert err.value.status == dsa.binding.DSA_ERR_BOUNDS
    ref_pool, ref_scale = O.cache_write_e4m3(inp["idx_keys"], inp["idx_key_scale"], bt, bits[1:], seq[1:], pos[1:])
    assert np.array_equal(pool_d.cpu().numpy(), ref_pool) and np.array_equal(scale_d.cpu().numpy(), ref_scale)


def test_cache_write_pools_in_one_launch_equals_the_oracle():
    """A decode step's writes into two latent pools and one key pool through one launch: every pool
    bit-exact with the oracle's write of its own rows."""
    spec = DecodeSpec("c", batch=4, ctx_lo=100, ctx_hi=900, rows_per_seq=1, k=8, n_layers=2, seed=14)
    inp = make_decode(spec)
    bt, ctx = inp["block_table"], inp["ctx"]
    pos = (ctx - 1).astype(np.int32)                                # the current token of each sequence
    targets = [(576, inp["KV"][0], inp["KV_scale"][0]), (576, inp["KV"][1], inp["KV_scale"][1]),
               (128, inp["idx_keys"], inp["idx_key_scale"])]
    writes, refs = [], []
    for i, (dim, pool, scale) in enumerate(targets):
        bits = bf16_bits_np(normal_np(50 + i, 0, 4 * dim).reshape(4, dim) * 2.0)
        refs.append(O.cache_write_e4m3(pool, scale, bt, bits, np.arange(4), pos))
        writes.append((bf16_dev(bits), u8_dev(pool), f32_dev(scale)))
    before = dsa.load().dsa_launch_count()
    dsa.CacheWriteBatch(writes, i32_dev(pos), i32_dev(bt))()
    assert dsa.load().dsa_launch_count() == before + 1
    dsa.sync_status()
    for (x, pool_d, scale_d), (ref_pool, ref_scale) in zip(writes, refs):
        assert np.array_equal(pool_d.cpu().numpy(), ref_pool)
        assert np.array_equal(scale_d.cpu().numpy(), ref_scale)


# ----------------------------------------------------------------------------- a4


def _tie_scores(rows, L, seed):
    s = normal_np(seed, 0, rows * L).reshape(rows, L)
    s = np.round(s * 64) / 64          # many exact ties
    s[0, :] = 1.0                      # a row of all-equal scores
    return s.astype(np.float32)


@pytest.mark.parametrize("rows,L,k", [(300, 777, 128), (40, 5000, 2048), (3, 100000, 2048), (2, 70001, 1),
                                      (5, 3000, 1000)])
def test_topk_exact_on_given_scores(rows, L, k):
    s = _tie_scores(rows, L, rows + L)
    ld = (L + 3) // 4 * 4
    buf = np.full((rows, ld), np.nan, dtype=np.float32)
    buf[:, :L] = s
    lens = np.array([L - (r * 37) % (L // 2 + 1) for r in range(rows)], dtype=np.int32)
    lens[-1] = min(k // 2 + 1, L)    # a row shorter than k
    out = dsa.topk(f32_dev(buf), k, row_len=i32_dev(lens), max_len=L)
    got = out.cpu().numpy()
    for r in range(rows):
        n = int(lens[r])
        ref = O.topk_row(s[r].astype(np.float64), n, k)
        assert set(got[r][got[r] >= 0]) == set(ref[ref >= 0]), r
        assert (got[r][min(k, n):] == -1).all()


def test_topk_segmented_crowded_threshold_bin():
    """Segmented mode (few long rows) where one segment holds thousands of candidates equal to the
    k-th score: the per-CTA candidate buffer overflows and the rest take the direct path."""
    rows, L, k = 2, 100000, 2048
    s = np.round(normal_np(77, 0, rows * L).reshape(rows, L) * 64) / 64
    s[0, 20000:24000] = 2.5                 # fewer than k scores lie above 2.5 in a N(0,1) row
    s[1, 50000:56000] = 2.25
    s = s.astype(np.float32)
    out = dsa.topk(f32_dev(s), k, row_len=i32_dev(np.full(rows, L, dtype=np.int32)), max_len=L)
    got = out.cpu().numpy()
    for r in range(rows):
        ref = O.topk_row(s[r].astype(np.float64), L, k)
        assert set(got[r]) == set(ref), r


@pytest.mark.parametrize("k", [2048, 100, 1])
def test_topk_long_rows_in_row_mode(k):
    """Row mode (one CTA per row) on rows of 16K-32K candidates with awkward value patterns:
    heavy ties, all-equal scores, values rising along the row, and outliers on a regular
    stride.  Each row's set equals the oracle's."""
    rows, L = 8, 32768
    s = normal_np(91, 0, rows * L).reshape(rows, L)
    s[1] = np.round(s[1] * 8) / 8                        # heavy ties
    s[2] = 1.0                                            # all equal: the band holds every score
    s[3] = np.arange(L) / L + 1e-3 * s[3]                 # rising: the top-k sits at the end
    s[4, ::64] += 50.0                                    # outliers on a stride of 64
    s[5, 8::64] += 50.0                                   # the same, shifted
    s = s.astype(np.float32)
    lens = np.array([L, L, L, L, L, L, 16384, 20001], dtype=np.int32)
    out = dsa.topk(f32_dev(s), k, row_len=i32_dev(lens), max_len=L)
    got = out.cpu().numpy()
    for r in range(rows):
        ref = O.topk_row(s[r].astype(np.float64), int(lens[r]), k)
        assert set(got[r]) == set(ref), r


def test_topk_causal_lengths():
    rows, L, k = 64, 600, 256
    s = normal_np(3, 0, rows * L).reshape(rows, L).astype(np.float32)
    out = dsa.topk(f32_dev(s), k, causal_len0=500, max_len=L)   # row r has min(500 + r, 600)
    got = out.cpu().numpy()
    for r in range(rows):
        n = min(500 + r, L)
        ref = O.topk_row(s[r].astype(np.float64), n, k)
        assert set(got[r]) == set(ref)


# ----------------------------------------------------------------------------- a2 + a3


def _indexer_case(L, n_q, q_pos0, fp8, seed):
    q = normal_np(seed, 0, n_q * 32 * 128).reshape(n_q, 32, 128)
    kk = normal_np(seed + 1, 0, L * 128).reshape(L, 128)
    w = normal_np(seed + 2, 0, n_q * 32).reshape(n_q, 32).astype(np.float32)
    if not fp8:
        qb, kb = bf16_bits_np(q), bf16_bits_np(kk)
        return dict(q=bf16_dev(qb), k=bf16_dev(kb), w=f32_dev(w), qv=O.bf16_to_f64(qb), kv=O.bf16_to_f64(kb),
                    wv=w.astype(np.float64), qs=None, ks=None)
    sq = (0.01 + 0.02 * np.abs(normal_np(seed + 3, 0, n_q * 32))).astype(np.float32).reshape(n_q, 32)
    sk = (0.01 + 0.02 * np.abs(normal_np(seed + 4, 0, L))).astype(np.float32)
    q8 = e4m3_codes_np(q / sq[:, :, None] * 0.01)
    k8 = e4m3_codes_np(kk / sk[:, None] * 0.01)
    qv = O.e4m3_to_f64(q8) * sq[:, :, None].astype(np.float64)
    kv = O.e4m3_to_f64(k8) * sk[:, None].astype(np.float64)
    return dict(q=u8_dev(q8), k=u8_dev(k8), w=f32_dev(w), qv=qv, kv=kv, wv=w.astype(np.float64),
                qs=f32_dev(sq), ks=f32_dev(sk))


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("L,n_q,q_pos0", [(300, 300, 0), (1000, 77, 900), (4500, 40, 4460)])
def test_indexer_prefill(fp8, L, n_q, q_pos0):
    c = _indexer_case(L, n_q, q_pos0, fp8, 100 + L + n_q)
    ld = (L + 3) // 4 * 4
    scores = torch.full((n_q, ld), float("nan"), device=DEV)
    view = dsa.dense_view(c["k"], c["ks"])
    dsa.indexer_score(c["q"], c["w"], view, scores, q_scale=c["qs"], q_pos0=q_pos0)
    dsa.sync_status()
    got = scores.cpu().numpy().astype(np.float64)
    lens = [min(q_pos0 + r + 1, L) for r in range(n_q)]
    ref = O.indexer_scores(c["qv"], c["wv"], c["kv"], lens)
    for r in range(n_q):
        n = lens[r]
        tol = 2e-5 * np.max(np.abs(ref[r, :n])) + 1e-6
        assert np.max(np.abs(got[r, :n] - ref[r, :n])) <= tol, r
        assert np.all(np.isnan(got[r, n:])), r       # nothing written past the row


def test_indexer_decode_paged():
    spec = DecodeSpec("t", batch=5, ctx_lo=1, ctx_hi=1000, rows_per_seq=1, k=64, n_layers=1, seed=21)
    ctx = np.array([1, 64, 65, 700, 1000])
    inp = make_decode(spec, ctx=ctx)
    bt, P = inp["block_table"], inp["n_pages"]
    q8, sq = O.quantize_e4m3_rows(inp["q_idx"], 128)
    ld = bt.shape[1] * 64
    scores = torch.full((5, ld), float("nan"), device=DEV)
    view = dsa.paged_view(u8_dev(inp["idx_keys"]), f32_dev(inp["idx_key_scale"]), i32_dev(bt), i32_dev(ctx))
    dsa.indexer_score(u8_dev(q8), f32_dev(inp["w"]), view, scores, q_scale=f32_dev(sq))
    dsa.sync_status()
    got = scores.cpu().numpy()
    qv = O.e4m3_to_f64(q8) * sq.reshape(5, 32, 1)
    for b in range(5):
        n = int(ctx[b])
        keys = O.paged_rows(inp["idx_keys"], inp["idx_key_scale"], bt[b], n)
        ref = O.indexer_scores(qv[b:b + 1], inp["w"][b:b + 1], keys, [n])[0]
        assert np.max(np.abs(got[b, :n] - ref[:n])) <= 2e-5 * np.max(np.abs(ref[:n])) + 1e-6
        assert np.all(np.isnan(got[b, n:]))


def test_indexer_decode_paged_one_long_sequence():
    """One 200K-token sequence: the launch splits its keys into short units (4 tiles per CTA)."""
    spec = DecodeSpec("t", batch=1, ctx_lo=1, ctx_hi=1, rows_per_seq=1, k=64, n_layers=1, seed=23)
    ctx = np.array([200003])
    inp = make_decode(spec, ctx=ctx)
    bt = inp["block_table"]
    q8, sq = O.quantize_e4m3_rows(inp["q_idx"], 128)
    ld = bt.shape[1] * 64
    scores = torch.full((1, ld), float("nan"), device=DEV)
    view = dsa.paged_view(u8_dev(inp["idx_keys"]), f32_dev(inp["idx_key_scale"]), i32_dev(bt), i32_dev(ctx))
    dsa.indexer_score(u8_dev(q8), f32_dev(inp["w"]), view, scores, q_scale=f32_dev(sq))
    dsa.sync_status()
    got = scores.cpu().numpy()[0]
    n = int(ctx[0])
    qv = O.e4m3_to_f64(q8) * sq.reshape(1, 32, 1)
    keys = O.paged_rows(inp["idx_keys"], inp["idx_key_scale"], bt[0], n)
    ref = O.indexer_scores(qv, inp["w"], keys, [n])[0]
    assert np.max(np.abs(got[:n] - ref[:n])) <= 2e-5 * np.max(np.abs(ref[:n])) + 1e-6
    assert np.all(np.isnan(got[n:]))


# ----------------------------------------------------------------------------- a6


def _mla_ref(Q, KV, idx_rows, rows, rpi=1):
    outs, lses = {}, {}
    for r in rows:
        outs[r], lses[r] = O.sparse_mla_row(Q[r], KV, idx_rows[r // rpi], SCALE)
    return outs, lses


@pytest.mark.parametrize("L,k", [(300, 128), (1000, 200), (2500, 2048)])
def test_sparse_mla_dense_bf16(L, k):
    n_q = 150
    Qb = bf16_bits_np(normal_np(31, 0, n_q * 64 * 576)).reshape(n_q, 64, 576)
    KVb = bf16_bits_np(normal_np(32, 0, L * 576)).reshape(L, 576)
    # index rows: a causal Top-k of random scores for rows at positions L - n_q + r
    sc = normal_np(33, 0, n_q * L).reshape(n_q, L)
    idx = np.stack([O.topk_row(sc[r], L - n_q + r + 1, k) for r in range(n_q)]).astype(np.int32)
    idx[7, :] = -1                                              # an empty row
    out, lse = dsa.sparse_mla_attn(bf16_dev(Qb), dsa.dense_view(bf16_dev(KVb)), i32_dev(idx), k, SCALE)
    dsa.sync_status()
    o = O.bf16_to_f64(bf16_host(out))
    l = lse.cpu().numpy()
    Q, KV = O.bf16_to_f64(Qb), O.bf16_to_f64(KVb)
    rows = list(range(0, n_q, 7)) + [n_q - 1]
    ref_o, ref_l = _mla_ref(Q, KV, idx, rows)
    for r in rows:
        if r == 7:
            assert np.all(o[r] == 0) and np.all(np.isneginf(l[r]))
            continue
        ma, rl = attn_errors(o[r], ref_o[r])
        assert ma <= 2e-2 and rl <= 5e-3, (r, ma, rl)
        assert np.max(np.abs(l[r] - ref_l[r])) <= 2e-3


@pytest.mark.parametrize("L,k", [(700, 200), (3000, 2048)])
def test_sparse_mla_dense_bf16_many_rows(L, k):
    """At least 2 rows per SM: every persistent CTA takes whole rows in turn and writes them
    directly (no key splits, no combine pass: the prefill schedule); checked like the test
    above, with padding inside rows as well."""
    n_q = 400
    Qb = bf16_bits_np(normal_np(51, 0, n_q * 64 * 576)).reshape(n_q, 64, 576)
    KVb = bf16_bits_np(normal_np(52, 0, L * 576)).reshape(L, 576)
    sc = normal_np(53, 0, n_q * L).reshape(n_q, L)
    idx = np.stack([O.topk_row(sc[r], min(L, L - n_q + r + 1), k) for r in range(n_q)]).astype(np.int32)
    idx[7, :] = -1                                              # an empty row
    idx[11, 3::5] = -1                                          # padding scattered inside a row
    idx[12, 130:] = -1                                          # a row that ends inside its second tile
    out, lse = dsa.sparse_mla_attn(bf16_dev(Qb), dsa.dense_view(bf16_dev(KVb)), i32_dev(idx), k, SCALE)
    dsa.sync_status()
    o = O.bf16_to_f64(bf16_host(out))
    l = lse.cpu().numpy()
    Q, KV = O.bf16_to_f64(Qb), O.bf16_to_f64(KVb)
    rows = sorted(set(list(range(0, n_q, 13)) + [11, 12, n_q - 1]))
    ref_o, ref_l = _mla_ref(Q, KV, idx, rows)
    for r in rows + [7]:
        if r == 7:
            assert np.all(o[r] == 0) and np.all(np.isneginf(l[r]))
            continue
        ma, rl = attn_errors(o[r], ref_o[r])
        assert ma <= 2e-2 and rl <= 5e-3, (r, ma, rl)
        assert np.max(np.abs(l[r] - ref_l[r])) <= 2e-3


def test_sparse_mla_k_covers_history_is_dense():
    L = 200
    Qb = bf16_bits_np(normal_np(41, 0, L * 64 * 576)).reshape(L, 64, 576)
    KVb = bf16_bits_np(normal_np(42, 0, L * 576)).reshape(L, 576)
    idx = np.stack([O.topk_row(np.zeros(L), t + 1, 256) for t in range(L)]).astype(np.int32)
    out, _ = dsa.sparse_mla_attn(bf16_dev(Qb), dsa.dense_view(bf16_dev(KVb)), i32_dev(idx), 256, SCALE)
    o = O.bf16_to_f64(bf16_host(out))
    Q, KV = O.bf16_to_f64(Qb), O.bf16_to_f64(KVb)
    for t in (0, 1, 127, 128, 199):
        ref, _ = O.dense_causal_attention_row(Q[t], KV[:t + 1], SCALE)
        ma, rl = attn_errors(o[t], ref)
        assert ma <= 2e-2 and rl <= 5e-3, (t, ma, rl)


@pytest.mark.parametrize("B,R,k", [(2, 3, 256), (3, 5, 2048), (40, 1, 512), (2, 3, 2048)])
def test_sparse_mla_paged_fp8_mtp(B, R, k):
    spec = DecodeSpec("t", batch=B, ctx_lo=100, ctx_hi=5000, rows_per_seq=R, k=k, n_layers=1, seed=50 + B)
    inp = make_decode(spec)
    ctx, bt = inp["ctx"], inp["block_table"]
    idx = np.stack([O.topk_row(normal_np(60 + b, 0, int(ctx[b])), int(ctx[b]), k) for b in range(B)]
                   ).astype(np.int32)
    view = dsa.paged_view(u8_dev(inp["KV"][0]), f32_dev(inp["KV_scale"][0]), i32_dev(bt), i32_dev(ctx))
    out, lse = dsa.sparse_mla_attn(bf16_dev(inp["Q"][0]), view, i32_dev(idx), k, SCALE, q_rows_per_idx_row=R)
    dsa.sync_status()
    o = O.bf16_to_f64(bf16_host(out))
    l = lse.cpu().numpy()
    for b in range(min(B, 6)):
        kv = O.paged_rows(inp["KV"][0], inp["KV_scale"][0], bt[b], int(ctx[b]))
        for r in range(R):
            row = b * R + r
            ref, rl_ = O.sparse_mla_row(O.bf16_to_f64(inp["Q"][0][row]), kv, idx[b], SCALE)
            ma, rl = attn_errors(o[row], ref)
            assert ma <= 2e-2 and rl <= 5e-3, (row, ma, rl)
            assert np.max(np.abs(l[row] - rl_)) <= 2e-3


# ----------------------------------------------------------------------------- bounded waits


def test_bounded_wait_returns_timeout_and_context_survives():
    lib = dsa.load()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.dsa_debug_bounded_wait(50_000_000, s) == 0
    assert lib.dsa_sync_status(s) == dsa.binding.DSA_ERR_TIMEOUT
    assert lib.dsa_sync_status(s) == 0          # status word was cleared
    x = torch.ones(1000, device=DEV)
    assert float(x.sum()) == 1000.0             # the context still works

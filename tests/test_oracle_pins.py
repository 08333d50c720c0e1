"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties one oracle function to something the pages print, a closed form, an
invariant, a library routine for a special case, or brute force on tiny inputs.  The
``test_planted_*`` tests mutate a copy of an oracle function with a plausible mistake
and check that the matching pin catches it.
"""
import inspect
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from synth import make_prefill, make_decode, WORKLOADS, PrefillSpec, DecodeSpec

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))
SCALE = 1.0 / math.sqrt(576)


# ----------------------------------------------------------------------------- number formats


def test_bf16_decoder_all_patterns_match_library():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_to_f64(bits)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert O.bf16_to_f64(np.array([0x3F80, 0xC000, 0x0001]))[2] == 2.0 ** -133


def test_e4m3_decoder_all_codes_match_library_and_hand_values():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_to_f64(codes)
    assert (((got == ref) | (np.isnan(got) & np.isnan(ref)))).all()
    hand = O.e4m3_to_f64(np.array([0x7E, 0x01, 0x38, 0x08, 0xB8], dtype=np.uint8))
    assert list(hand) == [448.0, 2.0 ** -9, 1.0, 2.0 ** -6, -1.0]


def test_e4m3_encoder_matches_library_in_range():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.normal(0, 100, 20000), rng.normal(0, 1e-2, 5000),
                        np.ldexp(1.0, np.arange(-12, 9))]).astype(np.float32)
    v = np.clip(v, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (O._encode_e4m3_rne_sat(v) == ref).all()


def test_e4m3_encoder_ties_to_even_and_saturation():
    enc = O._encode_e4m3_rne_sat
    # 1.0625 lies halfway between 1.0 (m=0) and 1.125 (m=1): even -> 1.0
    # 1.1875 lies halfway between 1.125 (m=1) and 1.25 (m=2): even -> 1.25
    # subnormal step 2^-9: 0.5 step ties to 0, 1.5 steps ties to 2, 0.75 step rounds to 1
    v = np.array([1.0625, 1.1875, 500.0, -1e9, 2.0 ** -10, 3 * 2.0 ** -10, 3 * 2.0 ** -11],
                 dtype=np.float32)
    assert list(enc(v)) == [0x38, 0x3A, 0x7E, 0xFE, 0x00, 0x02, 0x01]


def test_quantize_rows_scale_rule():
    x = np.array([[0.0] * 127 + [2.0], [0.0] * 128, [-3.0] + [1.5] * 127], dtype=np.float32)
    from synth.generators import bf16_bits_np
    codes, scale = O.quantize_e4m3_rows(bf16_bits_np(x), 128)
    assert scale[0] == np.float32(2.0) / np.float32(448.0)
    assert scale[1] == 1.0 and (codes[1] == 0).all()
    assert codes[0, 127] == 0x7E and codes[2, 0] == 0xFE     # amax element maps to +-448
    back = O.e4m3_to_f64(codes[2]) * scale[2]
    assert abs(back[0] + 3.0) < 1e-6 and np.all(np.abs(back[1:] - 1.5) <= 1.5 * 2 ** -4)


# ----------------------------------------------------------------------------- indexer


def _unit_case():
    """q[t,h] = a_h e_{i_h}, k[s] = e_s: x[t,h,s] = a_h [i_h == s], closed form below."""
    H, D, N = 32, 128, 16
    rng = np.random.default_rng(3)
    a = rng.normal(size=(2, H))
    ih = rng.integers(0, N, size=(2, H))
    q = np.zeros((2, H, D))
    for t in range(2):
        for h in range(H):
            q[t, h, ih[t, h]] = a[t, h]
    k = np.eye(N, D)
    w = rng.normal(size=(2, H))
    expect = np.zeros((2, N))
    for t in range(2):
        for h in range(H):
            expect[t, ih[t, h]] += w[t, h] * max(a[t, h], 0.0)
    return q, w, k, expect


def test_indexer_closed_form_unit_vectors(fn=None):
    fn = fn or O.indexer_scores
    q, w, k, expect = _unit_case()
    got = fn(q, w, k, [16, 9])
    assert np.allclose(got[0], expect[0], rtol=0, atol=1e-12)
    assert np.allclose(got[1, :9], expect[1, :9], rtol=0, atol=1e-12)
    assert np.all(np.isneginf(got[1, 9:]))


def test_indexer_invariants():
    rng = np.random.default_rng(5)
    q, w, k = rng.normal(size=(3, 32, 128)), rng.normal(size=(3, 32)), rng.normal(size=(40, 128))
    I = O.indexer_scores(q, w, k, [40] * 3)
    assert np.allclose(O.indexer_scores(q, w, 2.5 * k, [40] * 3), 2.5 * I)       # positive homogeneity
    assert np.allclose(O.indexer_scores(q, -w, k, [40] * 3), -I)                 # linear in w
    qp, kn = np.abs(q), -np.abs(k)            # every dot product <= 0: ReLU zeroes all heads
    assert (O.indexer_scores(qp, w, kn, [40] * 3) == 0).all()


# ----------------------------------------------------------------------------- top-k


def _rank_select(s, n, k):
    """Brute force: position i is kept iff fewer than k entries beat it (larger, or equal and earlier)."""
    keep = []
    for i in range(n):
        beat = sum(1 for j in range(n) if s[j] > s[i] or (s[j] == s[i] and j < i))
        if beat < k:
            keep.append(i)
    return set(keep)


def test_topk_brute_force_tiny(fn=None):
    fn = fn or O.topk_row
    rng = np.random.default_rng(11)
    for trial in range(300):
        n = int(rng.integers(1, 12))
        k = int(rng.integers(1, 8))
        s = rng.integers(-3, 4, size=n).astype(float)        # many ties
        got = fn(s, n, k)
        assert set(int(i) for i in got if i >= 0) == _rank_select(s, n, k)
        assert (got[min(k, n):] == -1).all()


def test_topk_exhaustive_sets_equal_best_sum():
    s = np.array([0.3, -1.0, 2.0, 0.3, 5.0, -0.2, 0.0])
    for k in range(1, 8):
        best = max(itertools.combinations(range(7), k), key=lambda c: (sum(s[list(c)]), [-i for i in c]))
        assert set(O.topk_row(s, 7, k)) == set(best)


# ----------------------------------------------------------------------------- attention


def _rand_qkv(L, seed=0):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(64, 576)), rng.normal(size=(L, 576))


def test_sparse_equals_dense_when_k_covers_history(fn=None):
    fn = fn or O.sparse_mla_row
    Q, KV = _rand_qkv(37)
    for t in (0, 5, 36):
        idx = O.topk_row(np.random.default_rng(t).normal(size=t + 1), t + 1, 64)
        o1, l1 = fn(Q, KV, idx, SCALE)
        o2, l2 = O.dense_causal_attention_row(Q, KV[:t + 1], SCALE)
        assert np.allclose(o1, o2, rtol=1e-12, atol=1e-12) and np.allclose(l1, l2, rtol=1e-12)


def test_first_row_is_its_own_value():
    Q, KV = _rand_qkv(4)
    o, lse = O.sparse_mla_row(Q, KV, np.array([0, -1, -1]), SCALE)
    assert np.array_equal(o, np.broadcast_to(KV[0, :512], (64, 512)))
    assert np.allclose(lse, SCALE * Q @ KV[0])


def test_attention_weights_sum_to_one_and_order_free():
    Q, KV = _rand_qkv(50, 1)
    KV2 = KV.copy()
    KV2[:, :512] = 0.75
    idx = np.array([3, 17, 40, 2, -1, 9])
    o, _ = O.sparse_mla_row(Q, KV2, idx, SCALE)
    assert np.allclose(o, 0.75, atol=1e-14)
    o1, l1 = O.sparse_mla_row(Q, KV, idx, SCALE)
    o2, l2 = O.sparse_mla_row(Q, KV, idx[::-1], SCALE)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2)


def test_empty_selection():
    Q, KV = _rand_qkv(3)
    o, l = O.sparse_mla_row(Q, KV, np.array([-1, -1]), SCALE)
    assert (o == 0).all() and np.isneginf(l).all()


# ----------------------------------------------------------------------------- group / MTP / schedule


def test_group_shared_layers_reuse_full_indices_exactly():
    spec = PrefillSpec("t", L=48, k=8, n_layers=4, seed=9)
    inp = make_prefill(spec)
    rows = [0, 3, 7, 20, 47]
    g = O.group_prefill(inp, rows)
    for t in rows:
        assert len([i for i in g["idx"][t] if i >= 0]) == min(8, t + 1)
        for l in range(4):       # every layer equals attention with the Full layer's indices
            o, ls = O.sparse_mla_row(O.bf16_to_f64(inp["Q"][l][t]), O.bf16_to_f64(inp["KV"][l]),
                                     g["idx"][t], inp["softmax_scale"])
            assert np.array_equal(o, g["O"][l][t])
    # rows with t + 1 <= k select the whole causal history: dense attention
    o, _ = O.dense_causal_attention_row(O.bf16_to_f64(inp["Q"][2][3]), O.bf16_to_f64(inp["KV"][2][:4]),
                                        inp["softmax_scale"])
    assert np.allclose(o, g["O"][2][3], atol=1e-12)


def test_decode_mtp_rows_share_row0_indices():
    spec = DecodeSpec("t", batch=2, ctx_lo=70, ctx_hi=200, rows_per_seq=3, k=16, n_layers=2, seed=1)
    inp = make_decode(spec)
    g = O.group_decode(inp)
    for b in range(2):
        n = int(inp["ctx"][b])
        kv = O.paged_rows(inp["KV"][1], inp["KV_scale"][1], inp["block_table"][b], n)
        for r in range(3):
            o, _ = O.sparse_mla_row(O.bf16_to_f64(inp["Q"][1][b * 3 + r]), kv, g["idx"][b], inp["softmax_scale"])
            assert np.array_equal(o, g["O"][1][b * 3 + r])
        assert (g["idx"][b] < n).all()


def _per_row_decode_inputs():
    spec = DecodeSpec("t", batch=2, ctx_lo=70, ctx_hi=260, rows_per_seq=3, k=16, n_layers=2, seed=3,
                      topk_per_row=True)
    return make_decode(spec)


def _reuse_inputs_with_query_row(inp, r):
    """The same decode step under the reuse policy, with draft row r's indexer query and weights
    standing as each sequence's own."""
    R = inp["rows_per_seq"]
    return dict(inp, q_idx=inp["q_idx"][r::R], w=inp["w"][r::R], topk_per_row=False)


def test_per_row_topk_with_equal_row_queries_is_the_reuse_policy(fn=None):
    """V1 reduces to R7 when all rows of a sequence carry row 0's indexer query and weights."""
    fn = fn or O.group_decode_per_row
    inp = _per_row_decode_inputs()
    R = inp["rows_per_seq"]
    same = dict(inp, q_idx=np.repeat(inp["q_idx"][::R], R, axis=0), w=np.repeat(inp["w"][::R], R, axis=0))
    g, ref = fn(same), O.group_decode(_reuse_inputs_with_query_row(inp, 0))
    for b in range(2):
        for r in range(R):
            assert np.array_equal(g["idx"][b * R + r], ref["idx"][b])
            for l in range(2):
                assert np.array_equal(g["O"][l][b * R + r], ref["O"][l][b * R + r])
                assert g["lse"][l][b * R + r] == pytest.approx(ref["lse"][l][b * R + r], abs=0, rel=0)


def test_per_row_topk_row_r_is_the_reuse_policy_with_row_r_query(fn=None):
    """Row b*R + r of V1 equals row b*R + r of R7 run with row r's indexer query: each row keeps
    the selection of its own query, over its own sequence's keys."""
    fn = fn or O.group_decode_per_row
    inp = _per_row_decode_inputs()
    R = inp["rows_per_seq"]
    g = fn(inp)
    differ = 0
    for r in range(R):
        ref = O.group_decode(_reuse_inputs_with_query_row(inp, r))
        for b in range(2):
            assert np.array_equal(g["idx"][b * R + r], ref["idx"][b])
            differ += not np.array_equal(g["idx"][b * R + r], g["idx"][b * R])
            for l in range(2):
                assert np.array_equal(g["O"][l][b * R + r], ref["O"][l][b * R + r])
    assert differ > 0      # the draft rows' own queries select other sets than row 0's


def test_paged_rows_follow_block_table():
    spec = DecodeSpec("t", batch=3, ctx_lo=65, ctx_hi=300, rows_per_seq=1, k=8, n_layers=1, seed=2)
    inp = make_decode(spec)
    bt = inp["block_table"]
    used = np.concatenate([bt[b, :(int(inp["ctx"][b]) + 63) // 64] for b in range(3)])
    assert sorted(used) == list(range(inp["n_pages"]))          # a permutation of the pool
    rows = O.paged_rows(inp["KV"][0], inp["KV_scale"][0], bt[1], 130)
    p, s = bt[1][129 // 64], 129 % 64
    assert np.array_equal(rows[129], O.e4m3_to_f64(inp["KV"][0][p, s]) * float(inp["KV_scale"][0][p, s]))


def test_cache_write_fills_the_slots_paged_rows_reads(fn=None):
    """Writing every position of a sequence, in any order, makes its paged rows read back as the
    dequantised per-token quantisation of the written rows; other sequences' slots are untouched."""
    fn = fn or O.cache_write_e4m3
    spec = DecodeSpec("t", batch=3, ctx_lo=65, ctx_hi=300, rows_per_seq=1, k=8, n_layers=1, seed=6)
    inp = make_decode(spec)
    bt, ctx = inp["block_table"], inp["ctx"]
    for dim, pool, scale in ((128, inp["idx_keys"], inp["idx_key_scale"]), (576, inp["KV"][0], inp["KV_scale"][0])):
        n = int(ctx[1])
        x = np.asarray(make_prefill(PrefillSpec("x", L=n, k=8), layers=[0])["KV"][0][:, :dim])
        order = np.random.default_rng(dim).permutation(n)
        new_pool, new_scale = fn(pool, scale, bt, x[order], np.full(n, 1), order)
        codes, sc = O.quantize_e4m3_rows(x, dim)
        assert np.array_equal(O.paged_rows(new_pool, new_scale, bt[1], n),
                              O.e4m3_to_f64(codes) * sc.astype(np.float64)[:, None])
        for b in (0, 2):
            m = int(ctx[b])
            assert np.array_equal(O.paged_rows(new_pool, new_scale, bt[b], m), O.paged_rows(pool, scale, bt[b], m))


def test_schedule_matches_pages():
    sch = O.layer_schedule(GOLD["n_layers"]["value"])
    full = [l for l, f, _ in sch if f]
    assert full[:5] == GOLD["full_layers_0based_printed"]["value"]
    assert full[-1] == GOLD["full_layers_0based_printed"]["last"]
    assert len(full) == GOLD["n_full"]["value"]
    shared = [l for l, f, _ in sch if not f]
    assert len(shared) == GOLD["n_shared"]["value"]
    assert round(100 * len(shared) / len(sch), 1) == GOLD["shared_fraction_pct"]["value"]
    for l, f, p in sch:
        assert sch[p][1] and 0 <= l - p <= 3 and (f == (p == l))


def test_param_arithmetic_matches_pages():
    assert O.indexer_param_count() == GOLD["params_per_indexer"]["value"]
    assert GOLD["n_shared"]["value"] * O.indexer_param_count() == GOLD["params_removed"]["value"]


# ----------------------------------------------------------------------------- planted mistakes


def _mutant(fn, old, new):
    src = inspect.getsource(fn)
    assert old in src, (old, fn.__name__)
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns[fn.__name__]


@pytest.mark.parametrize("old,new", [
    ("np.maximum(x, 0.0)", "x"),                 # dropped ReLU
    ("w[t] @ np.maximum", "w[0] @ np.maximum"),  # wrong query row of the weights
    ("k[:n].T", "k[:n][::-1].T"),               # reversed key order
])
def test_planted_indexer_mistakes_are_caught(old, new):
    bad = _mutant(O.indexer_scores, old, new)
    with pytest.raises(AssertionError):
        test_indexer_closed_form_unit_vectors(bad)


@pytest.mark.parametrize("old,new", [
    ("np.arange(n), -s", "-np.arange(n), -s"),   # ties to the higher index
    ("order[:min(k, n)]", "order[1:min(k, n) + 1]"),
])
def test_planted_topk_mistakes_are_caught(old, new):
    bad = _mutant(O.topk_row, old, new)
    with pytest.raises(AssertionError):
        test_topk_brute_force_tiny(bad)


@pytest.mark.parametrize("old,new", [
    ("softmax_scale * (Q @ kv.T)", "(Q @ kv.T)"),       # dropped scale
    ("kv[:, :D_V]", "kv[:, -D_V:]"),                    # value from the wrong dims
    ("sel = sel[sel >= 0]", "sel = np.abs(sel)"),        # padding not masked
])
def test_planted_attention_mistakes_are_caught(old, new):
    bad = _mutant(O.sparse_mla_row, old, new)
    with pytest.raises(AssertionError):
        test_sparse_equals_dense_when_k_covers_history(bad)


@pytest.mark.parametrize("old,new", [
    ("qv[row:row + 1], w[row:row + 1]", "qv[b * R:b * R + 1], w[b * R:b * R + 1]"),   # row 0's query for all
    ("kvrows, idx[row]", "kvrows, idx[b * R]"),                                        # row 0's selection
    ('paged_rows(inp["KV"][l]', 'paged_rows(inp["KV"][0]'),                             # layer 0's cache
])
def test_planted_per_row_policy_mistakes_are_caught(old, new):
    bad = _mutant(O.group_decode_per_row, old, new)
    with pytest.raises(AssertionError):
        test_per_row_topk_row_r_is_the_reuse_policy_with_row_r_query(bad)


@pytest.mark.parametrize("old,new", [
    ("t % PAGE] = codes[r]", "(t + 1) % PAGE] = codes[r]"),             # slot off by one
    ("block_table[b][t // PAGE]", "block_table[0][t // PAGE]"),          # first sequence's pages
    ("scale[page, t % PAGE] = sc[r]", "scale[page, t % PAGE] = 1.0"),    # scale not stored
])
def test_planted_cache_write_mistakes_are_caught(old, new):
    bad = _mutant(O.cache_write_e4m3, old, new)
    with pytest.raises(AssertionError):
        test_cache_write_fills_the_slots_paged_rows_reads(bad)


# ----------------------------------------------------------------------------- group selection (Full layer)
#
# The Full layer's selection inside the group functions is pinned against scores computed
# here by plain loops over heads, dims and the causal candidates s <= t (decode: s < N_b), with
# FP8 values produced by torch's own e4m3 conversion at the per-vector scale amax / 448, and
# the rank rule of _rank_select.  The inputs give the 32 heads of a query, and the keys of
# different tokens, magnitudes several octaves apart, so that a scale taken per token instead
# of per head, or a key scale applied to the wrong token, changes the selected sets.


def _torch_e4m3_values(x32, vec_len):
    """Per-vector e4m3 round trip through torch's float8_e4m3fn conversion: scale = amax / 448
    in fp32 (1 when amax = 0), x / scale saturated to +-448, returned as fp64 values."""
    x = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).reshape(-1, vec_len)
    amax = x.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    v = (x / scale[:, None]).clamp(-448.0, 448.0)
    back = v.to(torch.float8_e4m3fn).to(torch.float64) * scale.to(torch.float64)[:, None]
    return back.reshape(np.shape(x32)).numpy()


def _loop_scores(q, w, keys, n):
    """I[s] = sum_h w[h] * max(0, sum_d q[h,d] * keys[s,d]) for s < n, by plain loops."""
    out = []
    for s in range(n):
        tot = 0.0
        for h in range(q.shape[0]):
            x = math.fsum(float(q[h, d]) * float(keys[s, d]) for d in range(q.shape[1]))
            tot += float(w[h]) * max(0.0, x)
        out.append(tot)
    return np.array(out)


def _octave_prefill_inputs(seed=21, L=40, k=6):
    """Tiny prefill group whose indexer query heads and key tokens span many octaves (the head
    weights undo the query heads' spread, so that every head moves the scores)."""
    from synth.generators import bf16_bits_np
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(L, 32, 128)) * (2.0 ** (-np.arange(32) / 2.0))[None, :, None]
    kk = rng.normal(size=(L, 128)) * (2.0 ** rng.integers(-6, 7, size=L))[:, None]
    inp = make_prefill(PrefillSpec("oct", L=L, k=k, n_layers=1, seed=seed))
    inp["q_idx"] = bf16_bits_np(q)
    inp["k_idx"] = bf16_bits_np(kk)
    inp["w"] = (inp["w"] * (2.0 ** (np.arange(32) / 2.0))[None, :]).astype(np.float32)  # every head counts
    return inp


def _check_prefill_selection(fn, fp8):
    inp = _octave_prefill_inputs()
    L, k = inp["L"], inp["k"]
    rows = list(range(L))
    g = fn(inp, rows, fp8_indexer=fp8)
    qv = O.bf16_to_f64(inp["q_idx"])
    kv = O.bf16_to_f64(inp["k_idx"])
    if fp8:
        qv = _torch_e4m3_values(qv.astype(np.float32), 128)     # one scale per (token, head)
        kv = _torch_e4m3_values(kv.astype(np.float32), 128)     # one scale per key token
    for t in rows:
        sc = _loop_scores(qv[t], inp["w"][t], kv, t + 1)        # candidates s = 0 .. t
        got = g["idx"][t]
        assert set(int(i) for i in got if i >= 0) == _rank_select(sc, t + 1, k), t
        assert (got[min(k, t + 1):] == -1).all()


def test_group_prefill_selection_is_the_loop_definition(fn=None):
    _check_prefill_selection(fn or O.group_prefill, fp8=False)


def test_group_prefill_fp8_selection_is_the_loop_definition(fn=None):
    _check_prefill_selection(fn or O.group_prefill, fp8=True)


def test_prefill_tables_reuse_gives_the_same_group():
    inp = _octave_prefill_inputs(seed=4)
    for fp8 in (False, True):
        tab = O.prefill_tables(inp, fp8)
        a = O.group_prefill(inp, [3, 17, 39], fp8_indexer=fp8)
        b = O.group_prefill(inp, [3, 17, 39], fp8_indexer=fp8, tables=tab)
        for t in (3, 17, 39):
            assert np.array_equal(a["idx"][t], b["idx"][t]) and np.array_equal(a["O"][0][t], b["O"][0][t])


def _octave_decode_inputs(seed=12):
    """Tiny decode batch whose query heads span many octaves; key pool as generated."""
    from synth.generators import bf16_bits_np
    spec = DecodeSpec("oct", batch=3, ctx_lo=70, ctx_hi=200, rows_per_seq=2, k=12, n_layers=1, seed=seed)
    inp = make_decode(spec)
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(3, 32, 128)) * (2.0 ** (-np.arange(32) / 2.0))[None, :, None]
    inp["q_idx"] = bf16_bits_np(q)
    inp["w"] = (inp["w"] * (2.0 ** (np.arange(32) / 2.0))[None, :]).astype(np.float32)  # every head counts
    return inp


def _dense_cache_by_pages(pool, scale, bt, b, n):
    """Sequence b's first n cache rows, read page by page of its block table (torch e4m3 decode)."""
    rows = np.zeros((n, pool.shape[2]))
    vals = torch.from_numpy(np.ascontiguousarray(pool)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for lp in range((n + 63) // 64):
        p = int(bt[b][lp])
        for j in range(64):
            s = lp * 64 + j
            if s < n:
                rows[s] = vals[p, j] * float(scale[p, j])
    return rows


def test_group_decode_selection_is_the_loop_definition(fn=None):
    fn = fn or O.group_decode
    inp = _octave_decode_inputs()
    g = fn(inp)
    qv = _torch_e4m3_values(O.bf16_to_f64(inp["q_idx"]).astype(np.float32), 128)
    for b in range(len(inp["ctx"])):
        n = int(inp["ctx"][b])
        keys = _dense_cache_by_pages(inp["idx_keys"], inp["idx_key_scale"], inp["block_table"], b, n)
        sc = _loop_scores(qv[b], inp["w"][b], keys, n)          # candidates s = 0 .. N_b - 1
        got = g["idx"][b]
        assert set(int(i) for i in got if i >= 0) == _rank_select(sc, n, inp["k"]), b


@pytest.mark.parametrize("edits", [
    [('quantize_e4m3_rows(np.asarray(inp["q_idx"][t])[None], IDX_DIM)',
      'quantize_e4m3_rows(np.asarray(inp["q_idx"][t])[None], IDX_HEADS * IDX_DIM)'),
     ("sq.reshape(1, IDX_HEADS, 1)", "sq.reshape(1, 1, 1)")],          # one query scale per token, not per head
    [("[t + 1])[0]", "[t])[0]")],                                       # query t scores only s < t
    [("topk_row(sc, t + 1, k)", "topk_row(sc, t, k)")],                 # query t selects among s < t
    [('wt = np.asarray(inp["w"][t]', 'wt = np.asarray(inp["w"][0]')],  # the first row's head weights
])
def test_planted_group_prefill_fp8_mistakes_are_caught(edits):
    bad = _mutant_src(O.group_prefill, edits)
    with pytest.raises(AssertionError):
        test_group_prefill_fp8_selection_is_the_loop_definition(bad)


@pytest.mark.parametrize("old,new", [
    ('keys = e4m3_to_f64(k8) * sk.reshape(-1, 1)', 'keys = e4m3_to_f64(k8) * sk[::-1].reshape(-1, 1)'),  # wrong token's scale
    ('keys = e4m3_to_f64(k8) * sk.reshape(-1, 1)', 'keys = e4m3_to_f64(k8) * 1.0'),                      # scale dropped
])
def test_planted_key_scale_mistakes_are_caught(old, new):
    bad_tables = _mutant(O.prefill_tables, old, new)

    def bad(inp, rows, fp8_indexer=False):
        return O.group_prefill(inp, rows, fp8_indexer, tables=bad_tables(inp, fp8_indexer))
    with pytest.raises(AssertionError):
        test_group_prefill_fp8_selection_is_the_loop_definition(bad)


@pytest.mark.parametrize("edits", [
    [('quantize_e4m3_rows(inp["q_idx"], IDX_DIM)', 'quantize_e4m3_rows(inp["q_idx"], IDX_HEADS * IDX_DIM)'),
     ("sq.reshape(-1, IDX_HEADS, 1)", "sq.reshape(-1, 1, 1)")],              # per-token query scale
    [("w[b:b + 1], keys, [n])", "w[b:b + 1], keys, [n - 1])")],            # the newest token left out
    [('inp["idx_key_scale"], bt[b], n)', 'inp["idx_key_scale"], bt[0], n)')],  # first sequence's pages
])
def test_planted_group_decode_mistakes_are_caught(edits):
    bad = _mutant_src(O.group_decode, edits)
    with pytest.raises(AssertionError):
        test_group_decode_selection_is_the_loop_definition(bad)


def _mutant_src(fn, edits):
    src = inspect.getsource(fn)
    for old, new in edits:
        assert old in src, (old, fn.__name__)
        src = src.replace(old, new)
    ns = dict(vars(O))
    exec(compile(src, "<mutant>", "exec"), ns)
    return ns[fn.__name__]


# ----------------------------------------------------------------------------- inputs of the path (R12, R13)


def test_layer_norm_closed_forms(fn=None):
    fn = fn or O.layer_norm
    x = np.array([[1.0, 3.0] * 64, [5.0] * 128, [-2.0, 0.0, 2.0, 0.0] * 32])
    g, b = np.full(128, 2.0), np.full(128, 0.5)
    y = fn(x, g, b)
    # row 0: mean 2, biased variance 1 -> +-1 / sqrt(1 + eps) ; row 1: constant -> beta
    assert np.allclose(y[0, :2], [0.5 - 2 / math.sqrt(1 + 1e-6), 0.5 + 2 / math.sqrt(1 + 1e-6)], atol=1e-12)
    assert np.allclose(y[1], 0.5, atol=1e-12)
    # row 2: mean 0, variance 2 -> values / sqrt(2 + eps)
    assert np.allclose(y[2, :3], 0.5 + 2 * np.array([-2.0, 0.0, 2.0]) / math.sqrt(2 + 1e-6), atol=1e-12)
    z = fn(np.random.default_rng(1).normal(3, 5, size=(4, 128)), np.ones(128), np.zeros(128))
    assert np.allclose(z.mean(axis=1), 0, atol=1e-12) and np.allclose((z ** 2).mean(axis=1), 1, atol=1e-5)


def test_rms_norm_closed_forms(fn=None):
    fn = fn or O.rms_norm
    g = np.linspace(0.5, 1.5, 512)
    x = np.full((1, 512), -3.0)
    assert np.allclose(fn(x, g), -3.0 / math.sqrt(9.0 + 1e-6) * g, atol=1e-12)
    r = np.random.default_rng(2).normal(size=(3, 512))
    assert np.allclose(fn(r, np.ones(512)), fn(1000.0 * r, np.ones(512)), atol=1e-6)   # scale invariant
    assert np.allclose((fn(r, np.ones(512)) ** 2).mean(axis=1), 1.0, atol=1e-5)


def test_rope_closed_forms(fn=None):
    fn = fn or O.rope_pairs
    d, th = 64, 8.0e6
    for i in (0, 1, 17, 31):
        for p in (0, 1, 1000, (1 << 20) - 1):
            e = np.zeros(d)
            e[2 * i] = 1.0
            y = fn(e, p, th)
            a = p * th ** (-2 * i / d)
            assert abs(y[2 * i] - math.cos(a)) < 1e-12 and abs(y[2 * i + 1] - math.sin(a)) < 1e-12
            assert np.count_nonzero(np.abs(y) > 1e-15) <= 2
    v = np.random.default_rng(3).normal(size=(5, d))
    assert np.array_equal(fn(v, np.zeros(5), th), v)                              # position 0: no turn
    assert np.allclose(np.linalg.norm(fn(v, np.arange(5) * 7.0, th), axis=1), np.linalg.norm(v, axis=1))
    # relative position: <R(a, m), R(b, n)> depends on m - n only
    a_, b_ = v[0], v[1]
    s1 = fn(a_, 100.0, th) @ fn(b_, 37.0, th)
    s2 = fn(a_, 5100.0, th) @ fn(b_, 5037.0, th)
    assert abs(s1 - s2) < 1e-9


def test_indexer_projections_closed_forms_and_param_count(fn=None):
    fn = fn or O.indexer_projections
    rng = np.random.default_rng(4)
    T = 3
    cq, x = rng.normal(size=(T, 2048)), rng.normal(size=(T, 6144))
    Wq = np.zeros((4096, 2048))
    Wq[np.arange(2048), np.arange(2048)] = 1.0                 # heads 0..15 copy cq, heads 16..31 are 0
    Wk = np.zeros((128, 6144))
    Wk[np.arange(128), 6000 + np.arange(128) % 100] = 1.0      # key dim j reads hidden dim 6000 + j % 100
    Ww = np.zeros((32, 6144))
    Ww[np.arange(32), 3 * np.arange(32)] = 2.0
    g, b = np.full(128, 1.5), np.full(128, -0.25)
    q, k, w = fn(cq, x, Wq, Wk, Ww, g, b)
    assert q.shape == (T, 32, 128) and k.shape == (T, 128) and w.shape == (T, 32)
    assert np.array_equal(q[:, :16].reshape(T, 2048), cq) and (q[:, 16:] == 0).all()
    kk = x[:, 6000 + np.arange(128) % 100]
    mu, var = kk.mean(axis=1, keepdims=True), kk.var(axis=1, keepdims=True)
    assert np.allclose(k, (kk - mu) / np.sqrt(var + 1e-6) * 1.5 - 0.25, atol=1e-12)
    assert np.array_equal(w, 2.0 * x[:, 3 * np.arange(32)])
    assert Wq.size + Wk.size + Ww.size + g.size + b.size == O.indexer_param_count() == GOLD["params_per_indexer"]["value"]


def test_mla_latent_rows_closed_forms(fn=None):
    fn = fn or O.mla_latent_rows
    rng = np.random.default_rng(5)
    x = rng.normal(size=(4, 6144))
    Wd = np.zeros((512, 6144))
    Wd[np.arange(512), np.arange(512)] = 1.0
    Wr = np.zeros((64, 6144))
    Wr[np.arange(64), 1000 + np.arange(64)] = 1.0
    g = np.linspace(0.9, 1.1, 512)
    pos = np.array([0, 1, 77, (1 << 20) - 1])
    y = fn(x, Wd, Wr, g, pos)
    assert y.shape == (4, 576)
    c = x[:, :512]
    assert np.allclose(y[:, :512], c / np.sqrt((c ** 2).mean(axis=1, keepdims=True) + 1e-6) * g, atol=1e-12)
    assert np.array_equal(y[0, 512:], x[0, 1000:1064])                            # position 0: not turned
    for t in range(1, 4):
        for i in (0, 9, 31):
            a = pos[t] * 8.0e6 ** (-2 * i / 64)
            u, v = x[t, 1000 + 2 * i], x[t, 1001 + 2 * i]
            assert abs(y[t, 512 + 2 * i] - (u * math.cos(a) - v * math.sin(a))) < 1e-9
            assert abs(y[t, 513 + 2 * i] - (u * math.sin(a) + v * math.cos(a))) < 1e-9


def test_rope_query_turns_only_the_rope_dims():
    rng = np.random.default_rng(6)
    q = rng.normal(size=(2, 64, 576))
    y = O.rope_query(q, np.array([0, 500]))
    assert np.array_equal(y[:, :, :512], q[:, :, :512]) and np.array_equal(y[0], q[0])
    assert np.allclose(y[1, 7, 512:], O.rope_pairs(q[1, 7, 512:], 500))
    # a query and a latent key turned to their positions: the RoPE logit depends on their distance
    kr = rng.normal(size=64)
    s1 = O.rope_query(q[:1], np.array([900]))[0, 3, 512:] @ O.rope_pairs(kr, 400)
    s2 = O.rope_query(q[:1], np.array([1500]))[0, 3, 512:] @ O.rope_pairs(kr, 1000)
    assert abs(s1 - s2) < 1e-9


@pytest.mark.parametrize("fn,test,old,new", [
    ("layer_norm", "test_layer_norm_closed_forms", "var + eps", "var"),                  # eps dropped
    ("layer_norm", "test_layer_norm_closed_forms", "mean(axis=-1, keepdims=True)\n", "mean()\n"),  # over the tensor
    ("rms_norm", "test_rms_norm_closed_forms", "(x ** 2).mean(", "np.abs(x).mean("),      # mean |x| for rms
    ("rope_pairs", "test_rope_closed_forms", "out[..., 1::2] = x[..., 0::2] * s + x[..., 1::2] * c",
     "out[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c"),                            # turned the wrong way
    ("rope_pairs", "test_rope_closed_forms", "np.arange(0, d, 2, dtype=np.float64) / d",
     "np.arange(0, d // 2, dtype=np.float64) / d"),                                       # theta^(-i/64)
    ("indexer_projections", "test_indexer_projections_closed_forms_and_param_count",
     "layer_norm(x @ np.asarray(Wk, dtype=np.float64).T, gamma, beta)",
     "layer_norm(x @ np.asarray(Wk, dtype=np.float64).T, beta, gamma)"),                  # affine swapped
    ("mla_latent_rows", "test_mla_latent_rows_closed_forms", "rope_pairs(x @ np.asarray(W_kr, dtype=np.float64).T, pos)",
     "rope_pairs(x @ np.asarray(W_kr, dtype=np.float64).T, pos + 1)"),                    # position off by one
])
def test_planted_input_path_mistakes_are_caught(fn, test, old, new):
    bad = _mutant(getattr(O, fn), old, new)
    with pytest.raises(AssertionError):
        globals()[test](bad)

"""The shared input generator: published SplitMix64 values, host/torch agreement, recipes."""
import numpy as np
import torch

from synth.generators import (splitmix64_np, normal_np, normal_torch, bf16_bits_np,
                              bf16_bits_torch, ar1_keys_np)
from synth import make_prefill, PrefillSpec, decode_context_lengths, WORKLOADS


def test_splitmix64_published_sequence():
    # First outputs of SplitMix64 seeded with 1234567 (reference implementation by S. Vigna).
    got = splitmix64_np(1234567, np.arange(5, dtype=np.uint64))
    assert [int(v) for v in got] == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                                     4593380528125082431, 16408922859458223821]


def test_numpy_and_torch_streams_agree():
    a = normal_np(99, 1000, 5000)
    b = normal_torch(99, 1000, 5000, device="cpu", chunk=777).numpy()
    # float64 libm results may differ in the last bit; the rounded values the path uses agree
    assert np.abs(a - b).max() <= 4 * np.finfo(np.float64).eps * np.abs(a).max()
    assert np.array_equal(a.astype(np.float32), b.astype(np.float32))
    assert np.array_equal(bf16_bits_np(a).view(np.int16),
                          bf16_bits_torch(torch.from_numpy(a)).view(torch.int16).numpy())


def test_random_access_slices():
    full = normal_np(5, 0, 4000)
    assert np.array_equal(full[1234:2345], normal_np(5, 1234, 1111))


def test_normal_moments():
    x = normal_np(1, 0, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_ar1_drift():
    k = ar1_keys_np(3, 4000, 16, 0.99)
    lag1 = np.mean([np.corrcoef(k[:-1, d], k[1:, d])[0, 1] for d in range(16)])
    assert 0.97 < lag1 < 1.0 and abs(k.std() - 1) < 0.3


def test_decode_lengths_in_range():
    ctx = decode_context_lengths(WORKLOADS["decode_b32_mtp4"])
    assert len(ctx) == 32 and ctx.min() >= 65536 and ctx.max() <= 262144


def test_prefill_shapes():
    inp = make_prefill(PrefillSpec("x", L=40, k=8), layers=[0, 1])
    assert inp["q_idx"].shape == (40, 32, 128) and inp["Q"][1].shape == (40, 64, 576)
    assert inp["KV"][0].dtype == np.uint16 and inp["w"].dtype == np.float32


def test_per_row_topk_recipe_keeps_row0_of_the_reuse_recipe():
    import dataclasses
    from synth import make_decode
    spec = WORKLOADS["decode_b32_mtp4_verify"]
    assert spec.topk_per_row and spec.rows_per_seq == 5
    small = dataclasses.replace(spec, batch=3, ctx_lo=100, ctx_hi=400, k=32, n_layers=1)
    reuse = make_decode(dataclasses.replace(small, topk_per_row=False))
    per_row = make_decode(small)
    R = small.rows_per_seq
    assert per_row["q_idx"].shape == (3 * R, 32, 128) and per_row["w"].shape == (3 * R, 32)
    assert np.array_equal(per_row["q_idx"][::R], reuse["q_idx"]) and np.array_equal(per_row["w"][::R], reuse["w"])
    assert not np.array_equal(per_row["q_idx"][1::R], reuse["q_idx"])
    for key in ("ctx", "block_table", "idx_keys", "idx_key_scale"):
        assert np.array_equal(per_row[key], reuse[key])
    assert np.array_equal(per_row["Q"][0], reuse["Q"][0]) and np.array_equal(per_row["KV"][0], reuse["KV"][0])
    on_torch = make_decode(small, device="cpu")
    assert np.array_equal(on_torch["q_idx"].view(torch.int16).numpy(), per_row["q_idx"].view(np.int16))
    assert np.array_equal(on_torch["w"].numpy(), per_row["w"])

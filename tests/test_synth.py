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

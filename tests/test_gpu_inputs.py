"""The steps that produce the path's inputs, through the C ABI, against the fp64 oracle (needs a B200).

* indexer projections (R12): q from the query latent, LayerNorm key and head weights from the
  hidden state; T = 1, 129 and 300 tokens (ragged 128-row tiles), the full 2,048 / 6,144 widths.
* latent KV rows (R13): RMSNorm of the rank-512 compression and RoPE of 64 dims at positions up to
  2^20 - 1; query RoPE in place.
Tolerance: bf16 outputs within 2^-8 of the value plus 1e-3 of the tensor's largest magnitude
(one bf16 rounding of an fp32 result whose accumulation error is far smaller); fp32 outputs
within 1e-4 of the largest magnitude.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_sparse_11_b200 as dsa  # noqa: E402
import oracle.dsa_oracle as O  # noqa: E402
from synth.generators import bf16_bits_np, normal_np  # noqa: E402
from test_gpu_kernels import bf16_dev, f32_dev, i32_dev, bf16_host  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


def _bf16(seed, shape, std=1.0):
    return bf16_bits_np(normal_np(seed, 0, int(np.prod(shape))) * std).reshape(shape)


def _close_bf16(got, ref):
    tol = 2.0 ** -8 * np.abs(ref) + 1e-3 * np.max(np.abs(ref))
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


@pytest.mark.parametrize("T", [1, 129, 300])
def test_indexer_projections(T):
    cq, x = _bf16(61, (T, 2048)), _bf16(62, (T, 6144))
    Wq, Wkw = _bf16(63, (4096, 2048), 2048 ** -0.5), _bf16(64, (160, 6144), 6144 ** -0.5)
    gamma = (1.0 + 0.1 * normal_np(65, 0, 128)).astype(np.float32)
    beta = (0.1 * normal_np(66, 0, 128)).astype(np.float32)
    q, k, w = dsa.indexer_project(bf16_dev(cq), bf16_dev(x), bf16_dev(Wq), bf16_dev(Wkw), f32_dev(gamma), f32_dev(beta))
    dsa.sync_status()
    rq, rk, rw = O.indexer_projections(O.bf16_to_f64(cq), O.bf16_to_f64(x), O.bf16_to_f64(Wq),
                                       O.bf16_to_f64(Wkw[:128]), O.bf16_to_f64(Wkw[128:]), gamma, beta)
    _close_bf16(O.bf16_to_f64(bf16_host(q)), rq)
    _close_bf16(O.bf16_to_f64(bf16_host(k)), rk)
    gw = w.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(gw - rw)) <= 1e-4 * np.max(np.abs(rw))


def test_mla_latent_rows_and_query_rope():
    T = 200
    x = _bf16(71, (T, 6144))
    Wkv = _bf16(72, (576, 6144), 6144 ** -0.5)
    gamma = (1.0 + 0.1 * normal_np(73, 0, 512)).astype(np.float32)
    pos = np.concatenate([[0, 1, 2, 63, 64, 12345, (1 << 20) - 1, 5_000_000],
                          np.random.default_rng(7).integers(0, 1 << 20, size=T - 8)]).astype(np.int32)
    lat = dsa.mla_latent(bf16_dev(x), bf16_dev(Wkv), f32_dev(gamma), i32_dev(pos))
    dsa.sync_status()
    ref = O.mla_latent_rows(O.bf16_to_f64(x), O.bf16_to_f64(Wkv[:512]), O.bf16_to_f64(Wkv[512:]), gamma, pos)
    got = O.bf16_to_f64(bf16_host(lat))
    _close_bf16(got[:, :512], ref[:, :512])
    _close_bf16(got[:, 512:], ref[:, 512:])
    # the query side: dims 512..575 turned in place, the rest untouched
    q = _bf16(74, (6, 64, 576))
    qd = bf16_dev(q)
    qpos = pos[:6]
    dsa.rope_query(qd, i32_dev(qpos))
    dsa.sync_status()
    gq = bf16_host(qd)
    assert np.array_equal(gq[:, :, :512], q[:, :, :512])
    rq = O.rope_query(O.bf16_to_f64(q), qpos)
    _close_bf16(O.bf16_to_f64(gq[:, :, 512:]), rq[:, :, 512:])


@pytest.mark.parametrize("q_rank,hidden", [(64, 64), (192, 320)])
def test_indexer_projections_small_widths(q_rank, hidden):
    """The projections at the smallest widths the library takes (one or a few 64-wide K blocks)."""
    T = 70
    cq, x = _bf16(81, (T, q_rank)), _bf16(82, (T, hidden))
    Wq, Wkw = _bf16(83, (4096, q_rank), q_rank ** -0.5), _bf16(84, (160, hidden), hidden ** -0.5)
    gamma, beta = np.full(128, 1.25, dtype=np.float32), np.full(128, -0.5, dtype=np.float32)
    q, k, w = dsa.indexer_project(bf16_dev(cq), bf16_dev(x), bf16_dev(Wq), bf16_dev(Wkw), f32_dev(gamma), f32_dev(beta))
    dsa.sync_status()
    rq, rk, rw = O.indexer_projections(O.bf16_to_f64(cq), O.bf16_to_f64(x), O.bf16_to_f64(Wq),
                                       O.bf16_to_f64(Wkw[:128]), O.bf16_to_f64(Wkw[128:]), gamma, beta)
    _close_bf16(O.bf16_to_f64(bf16_host(q)), rq)
    _close_bf16(O.bf16_to_f64(bf16_host(k)), rk)
    assert np.max(np.abs(w.cpu().numpy() - rw)) <= 1e-4 * np.max(np.abs(rw))


"""Measurement arithmetic of bench.py (CPU): the algorithmic work each bench line divides by.

Closed forms: a causal prefill of L rows has L(L+1)/2 indexer pairs of 8,192 flops
(32 heads x 128 dims x 2) and sum_t min(k, t+1) selected keys of 139,264 attention flops
(64 heads x (576 + 512) x 2); a decode sequence of context N reads 132 B per key in the
indexer (128-byte e4m3 code + 4-byte scale) and gathers 580 B per selected key.  The reference
arm's JSON line is checked end to end on the smallest workload.
"""
import numpy as np

import bench
from synth import WORKLOADS


def test_prefill_32k_counts():
    c = bench.algorithmic_counts(WORKLOADS["prefill_32k"])
    L, k = 32768, 2048
    assert c["tokens"] == L and c["mla_rows"] == L
    assert c["indexer_flops"] == 8192.0 * L * (L + 1) / 2                    # 4.40e12
    sel = k * (k + 1) / 2 + (L - k) * k                                       # rows t < k keep t + 1 keys
    assert c["mla_flops_per_layer"] == 139264.0 * sel                         # 9.05e12
    assert abs(c["indexer_flops"] - 4.398e12) / 4.398e12 < 1e-3
    assert abs(c["mla_flops_per_layer"] - 9.054e12) / 9.054e12 < 1e-3


def test_decode_counts():
    spec = WORKLOADS["decode_b32_mtp4"]
    ctx = np.array([1000, 5000, 70000])
    c = bench.algorithmic_counts(spec, ctx)
    sel = 1000 + 2048 + 2048
    assert c["tokens"] == 3 * 5
    assert c["indexer_bytes"] == 132.0 * ctx.sum()
    assert c["mla_flops_per_layer"] == 139264.0 * sel * 5
    assert c["mla_bytes_per_layer"] == sel * 580.0 + 15 * 64 * (576 + 512) * 2.0


def test_decode_per_row_topk_counts():
    # every row scores the same keys with its own query and gathers its own selection
    ctx = np.array([1000, 5000, 70000])
    reuse = bench.algorithmic_counts(WORKLOADS["decode_b32_mtp4"], ctx)
    c = bench.algorithmic_counts(WORKLOADS["decode_b32_mtp4_verify"], ctx)
    sel = 1000 + 2048 + 2048
    assert c["tokens"] == reuse["tokens"] == 15
    assert c["indexer_flops"] == 5 * reuse["indexer_flops"] == 5 * 8192.0 * ctx.sum()
    assert c["indexer_bytes"] == reuse["indexer_bytes"]          # the keys are needed once
    assert c["mla_flops_per_layer"] == reuse["mla_flops_per_layer"]
    assert c["mla_bytes_per_layer"] == 5 * sel * 580.0 + 15 * 64 * (576 + 512) * 2.0


def test_workload_configs_name_every_bench_workload():
    for name in ["tiny_prefill", "prefill_32k", "prefill_128k_fp8", "decode_b32_mtp4", "decode_b32_d0",
                 "decode_b32_mtp4_verify", "decode_1m_mtp5"]:
        spec, cfg = bench.workload_config(name)
        assert cfg["workload"] == name
    spec, cfg = bench.workload_config("decode_b32_d0")
    assert spec.rows_per_seq == 1 and cfg["rows_per_seq"] == 1


def test_mla_dram_bytes_per_row_is_queries_plus_outputs():
    # the ncu-derived traffic per query row sits just above the queries in and outputs out
    q_out = 64 * 576 * 2 + 64 * 512 * 2
    assert q_out <= bench.MLA_DRAM_BYTES_PER_ROW_BF16 <= 1.1 * q_out


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints exactly one JSON line
    with the contract keys; it runs here on the CPU on the smallest workload."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_prefill", "--steps", "1", "--warmup", "0", "--ref-seconds", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "tiny_prefill"

#!/usr/bin/env python
"""Benchmark of the DSA + IndexShare step on B200: query tokens/s per IndexShare group.

A step is one pass of the whole hot path over one batch of synthetic input: the Full layer's
indexer scores + Top-k into the reuse handle, then sparse MLA for the Full layer and its 3
Shared layers (decode: the current token's rows are first written into the paged FP8 caches,
and a 78-layer step runs the 21 groups of the schedule).  Inputs are generated on the device by
the seeded generator before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl reference]

Default (``all``): the headline line is causal prefill of 131,072 tokens with the FP8 indexer
(the largest single-GPU prefill workload), timed over exactly K steps; the same process then
measures the other workloads (512-token tiny prefill, 32K bf16 prefill, batch-32 decode with 4
MTP draft rows and without, 1M-token 78-layer decode) and reports each under ``workloads``, each
timed over at least two seconds of steps so that the clock sampler sees it.

One JSON line is printed by rank 0.  Multi-GPU (torchrun): every rank runs its own independent
problem (weak scaling, no collective on the data path); the time is the max over ranks of the
CUDA-event time.  ``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
headline workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import gc
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "query tokens/s per IndexShare group"
UNIT = "query tokens/s"
HEADLINE = "prefill_128k_fp8"
SUB_WORKLOADS = ["tiny_prefill", "prefill_32k", "decode_b32_mtp4", "decode_b32_d0", "decode_1m_mtp5"]
ALL_WORKLOADS = ["tiny_prefill", "prefill_32k", "prefill_128k_fp8", "decode_b32_mtp4", "decode_b32_d0",
                 "decode_b32_mtp4_verify", "decode_1m_mtp5"]

# sparse_mla_kernel<bf16>, L=8,192 prefill launch (8,192 query rows): ncu measured 672.8 MB read
# + 505.5 MB written = 143,832 B per query row (queries 73,728 B in, outputs 65,536 B out, the
# rest index rows and the latent rows' first touch).
MLA_DRAM_BYTES_PER_ROW_BF16 = (672.825600e6 + 505.489152e6) / 8192


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default="all", choices=["all"] + ALL_WORKLOADS)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    p.add_argument("--ref-seconds", type=float, default=150.0, help="reference arm total budget")
    p.add_argument("--seq-len", type=int, default=None, help="override L of a prefill workload (profiling)")
    p.add_argument("--min-timed-s", type=float, default=2.0,
                   help="least timed seconds of each workload under 'workloads' (clock samples)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sub", action="store_true", help="headline workload only")
    p.add_argument("--graph", choices=["auto", "on", "off"], default="auto",
                   help="replay each step as one captured CUDA graph (auto: decode workloads)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args(argv)


# ----------------------------------------------------------------------------- distributed


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    """Max of a per-rank timer over all ranks (the job's time is its slowest rank)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, steps, ws, total_ms_max):
    """Whole-job tokens/s: every rank processes its own problem per step (weak scaling)."""
    return tokens_per_rank * ws * steps / (total_ms_max / 1e3)


# ----------------------------------------------------------------------------- workload


def workload_config(name, seq_len=None):
    import dataclasses
    from synth import WORKLOADS
    spec = WORKLOADS[name]
    if seq_len is not None and hasattr(spec, "L"):
        spec = dataclasses.replace(spec, L=seq_len)
    if name.startswith("decode"):
        cfg = {"workload": name, "batch": spec.batch, "context": f"U[{spec.ctx_lo},{spec.ctx_hi}]",
               "rows_per_seq": spec.rows_per_seq, "k": spec.k, "layers": spec.n_layers,
               "cache": "paged e4m3 (64-token pages), device-resident across steps; the step writes its "
                        "current token's rows into every pool first (one launch)", "indexer": "e4m3",
               "topk": "one per query row" if spec.topk_per_row else "row 0's, reused by the draft rows"}
        if spec.n_layers > 4:
            cfg["schedule"] = "Full at layers 0, 1, 2+4g; 21 groups per step"
        return spec, cfg
    return spec, {"workload": name, "seq_len": spec.L, "k": spec.k, "layers_per_group": spec.n_layers,
                  "indexer": "e4m3" if spec.indexer_fp8 else "bf16", "latent_kv": "bf16 [L,576]",
                  "heads": 64, "indexer_heads": 32}


def workload_dtype(name):
    return "bf16" if name in ("tiny_prefill", "prefill_32k") else "bf16+e4m3"


def algorithmic_counts(spec, ctx=None):
    """Algorithmic work of one group: indexer flops/bytes, MLA flops per layer, query tokens."""
    if hasattr(spec, "L"):
        L, k = spec.L, spec.k
        pairs = L * (L + 1) // 2
        sel = sum(min(k, t + 1) for t in range(L))
        return {"tokens": L, "indexer_flops": 8192.0 * pairs, "mla_flops_per_layer": 139264.0 * sel,
                "mla_rows": L, "indexer_bytes": None, "mla_gather_bytes_per_layer": 1152.0 * sel}
    import numpy as np
    ctx = np.asarray(ctx)
    R = spec.rows_per_seq
    sel = float(np.minimum(ctx, spec.k).sum())
    # per-row Top-k: R indexer queries per sequence over the same keys (the keys' bytes are still
    # needed once), and up to R distinct selections per sequence to gather
    scored = R if spec.topk_per_row else 1
    return {"tokens": len(ctx) * R, "indexer_flops": 8192.0 * float(ctx.sum()) * scored,
            "mla_flops_per_layer": 139264.0 * sel * R, "mla_rows": len(ctx) * R,
            "indexer_bytes": 132.0 * float(ctx.sum()),
            "mla_bytes_per_layer": sel * scored * 580.0 + len(ctx) * R * 64 * (576 + 512) * 2.0}


class Workload:
    """Device inputs and the IndexShare groups of one step (1 group, or 21 for 78 layers)."""

    def __init__(self, spec, name, dev):
        import torch
        import long_context_sparse_11_b200 as dsa
        from synth import make_prefill, make_decode, make_decode_indexer, make_decode_new_tokens
        self.name, self.spec = name, spec
        self.groups, self.step_inputs, self.layers_per_group, self.writes = [], [], [], []
        if name.startswith("decode"):
            inp = make_decode(spec, device=dev)
            self.inp = inp
            B = len(inp["ctx"])
            ctx_d = torch.from_numpy(inp["ctx"].astype("int32")).to(dev)
            bt_d = torch.from_numpy(inp["block_table"]).to(dev)
            # per-row Top-k: every query row is its own entry of the views (same pages, same length)
            rows = spec.rows_per_seq if spec.topk_per_row else 1
            kvs = [dsa.paged_view(inp["KV"][l], inp["KV_scale"][l], bt_d, ctx_d, rows_per_seq=rows)
                   for l in range(spec.n_layers)]
            fulls = [l for l in range(spec.n_layers) if dsa.layer_is_full(l)] if spec.n_layers > 4 else [0]
            ends = fulls[1:] + [spec.n_layers]
            new = make_decode_new_tokens(spec, B, range(spec.n_layers), fulls, device=dev)
            self.pos = torch.from_numpy((inp["ctx"] - 1).astype("int32")).to(dev)   # the current token
            self.bt = bt_d
            for l in range(spec.n_layers):
                self.writes.append((new["kv"][l], inp["KV"][l], inp["KV_scale"][l]))
            for f, e in zip(fulls, ends):
                ind = inp if f == 0 else make_decode_indexer(spec, f, inp["n_pages"], B, dev)
                self.writes.append((new["key"][f], ind["idx_keys"], ind["idx_key_scale"]))
                keys = dsa.paged_view(ind["idx_keys"], ind["idx_key_scale"], bt_d, ctx_d, rows_per_seq=rows)
                g = dsa.IndexShareGroup(ind["q_idx"], ind["w"], keys, spec.k, inp["Q"][f:e], kvs[f:e],
                                        inp["softmax_scale"], indexer_dtype=dsa.DSA_E4M3,
                                        q_rows_per_idx_row=spec.rows_per_seq // rows, first_layer=f)
                self.groups.append(g)
                self.layers_per_group.append(e - f)
                # a decode step's new inputs: the indexer query and weights, the MLA query rows
                self.step_inputs += [ind["q_idx"], ind["w"]] + list(inp["Q"][f:e])
            self.step_inputs += [x for x, _, _ in self.writes]     # and the current token's rows
            self.write_all = dsa.CacheWriteBatch(self.writes, self.pos, self.bt)   # one launch per step
            self.counts = algorithmic_counts(spec, inp["ctx"])
        else:
            inp = make_prefill(spec, device=dev)
            self.inp = inp
            g = dsa.IndexShareGroup(inp["q_idx"], inp["w"], dsa.dense_view(inp["k_idx"]), spec.k, inp["Q"],
                                    [dsa.dense_view(x) for x in inp["KV"]], inp["softmax_scale"],
                                    indexer_dtype=dsa.DSA_E4M3 if spec.indexer_fp8 else dsa.DSA_BF16)
            self.groups.append(g)
            self.layers_per_group.append(spec.n_layers)
            # a prefill step's inputs: everything the group reads
            self.step_inputs = [inp["q_idx"], inp["w"], inp["k_idx"]] + list(inp["Q"]) + list(inp["KV"])
            self.counts = algorithmic_counts(spec)

    @property
    def outputs(self):
        return [t for g in self.groups for t in g.out + g.lse]

    def forward(self):
        if self.writes:
            self.write_all()
        for g in self.groups:
            g.forward()


def indexer_alone(wl, spec, dev, stream):
    """Prefill a2+a3 kernel alone, for its tensor-pipe fraction: the group's indexer query rows in
    blocks of up to 8,192 rows against all keys (causal), scores into one [rows, L] fp32 block,
    CUDA events around the launches (outside the timed steps).  FP8 inputs are quantised first,
    untimed, as the group does on its own."""
    import torch
    import long_context_sparse_11_b200 as dsa
    inp, L = wl.inp, spec.L
    q, w = inp["q_idx"], inp["w"]
    q_scale = None
    if spec.indexer_fp8:
        q, q_scale = dsa.quant_e4m3(inp["q_idx"])
        k8, k_scale = dsa.quant_e4m3(inp["k_idx"])
        keys = dsa.dense_view(k8, k_scale)
    else:
        keys = dsa.dense_view(inp["k_idx"])
    R = min(L, 8192)
    scores = torch.empty(R, L, dtype=torch.float32, device=dev)

    def run():
        for r0 in range(0, L, R):
            n = min(R, L - r0)
            dsa.indexer_score(q[r0:r0 + n], w[r0:r0 + n], keys, scores[:n],
                              q_scale=None if q_scale is None else q_scale[r0 * 32:(r0 + n) * 32], q_pos0=r0)

    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run()
    e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    del scores
    return ms, (L + R - 1) // R


def input_projections(L, dev, stream, reps=3):
    """The steps that produce the path's inputs for L tokens, timed alone: the indexer projections
    (q from a 2,048-rank query latent, LayerNorm key and head weights from the 6,144-wide hidden
    state) and the latent KV rows (rank-512 compression + RMSNorm, 64 RoPE dims), on seeded random
    bf16 weights of those shapes.  Returns their times and tensor-pipe throughput."""
    import torch
    import long_context_sparse_11_b200 as dsa
    g = torch.Generator(device=dev).manual_seed(11)

    def rnd(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device=dev) * std).to(torch.bfloat16)
    cq, x = rnd(L, 2048), rnd(L, 6144)
    Wq, Wkw, Wkv = rnd(4096, 2048, std=2048 ** -0.5), rnd(160, 6144, std=6144 ** -0.5), rnd(576, 6144, std=6144 ** -0.5)
    gamma, beta, rms = (torch.ones(128, device=dev), torch.zeros(128, device=dev), torch.ones(512, device=dev))
    pos = torch.arange(L, dtype=torch.int32, device=dev)
    q_out, k_out, w_out = dsa.indexer_project(cq, x, Wq, Wkw, gamma, beta)
    lat = dsa.mla_latent(x, Wkv, rms, pos)
    res = {}
    for name, fn, flops in (
            ("indexer_projections", lambda: dsa.indexer_project(cq, x, Wq, Wkw, gamma, beta, q_out, k_out, w_out),
             2.0 * L * (2048 * 4096 + 6144 * 160)),
            ("latent_rows", lambda: dsa.mla_latent(x, Wkv, rms, pos, out=lat), 2.0 * L * 6144 * 576)):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = {"ms": round(ms, 4), "tflops": round(flops / (ms / 1e3) / 1e12, 1)}
    dsa.sync_status()
    del cq, x, Wq, Wkw, Wkv, q_out, k_out, w_out, lat
    gc.collect()
    torch.cuda.empty_cache()
    return res


def independent_full_layers(wl, spec, stream, flush, reps=3):
    """The same sequence run as 4 independent Full layers: each layer its own group call of one
    layer (its own a1-a4 on the indexer inputs, then its own a6), back to back on the stream."""
    import torch
    import long_context_sparse_11_b200 as dsa
    inp = wl.inp
    groups = [dsa.IndexShareGroup(inp["q_idx"], inp["w"], dsa.dense_view(inp["k_idx"]), spec.k, [inp["Q"][l]],
                                  [dsa.dense_view(inp["KV"][l])], inp["softmax_scale"],
                                  indexer_dtype=dsa.DSA_E4M3 if spec.indexer_fp8 else dsa.DSA_BF16)
              for l in range(spec.n_layers)]
    for g in groups:
        g.forward()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for g in groups:
            g.forward()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    dsa.sync_status()
    del groups
    gc.collect()
    torch.cuda.empty_cache()
    return statistics.mean(times)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(1.0)   # nvidia-smi's start-up: the first sample should fall inside the timed region
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(dev_index):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[dev_index]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def fp8_dense_peak(dev):
    """Dense e4m3 GEMM throughput on this GPU: the library FP8 GEMM (cuBLASLt through
    torch._scaled_mm, 8192^3, bf16 out), best of 10 after warm-up; None if unavailable."""
    import torch
    try:
        n = 8192
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        best = float("inf")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(10):
            e0.record()
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:
        return None


# ----------------------------------------------------------------------------- CPU oracle sample


def host_inputs(spec, name, inp):
    """The oracle's view of a workload: host arrays (bf16 as uint16 bits) and, for prefill, the
    whole-sequence fp64 tables converted once, so that a timed call does only its rows' work."""
    import numpy as np
    import oracle.dsa_oracle as O
    import torch

    def host_bits(t):
        return t.view(torch.int16).cpu().numpy().view(np.uint16)

    if name.startswith("decode"):
        nl = 4 if len(inp["Q"]) <= 4 else 1   # the first IndexShare group (layers 0..3, or layer 0 of 78)
        return {"ctx": inp["ctx"], "block_table": inp["block_table"], "k": spec.k, "rows_per_seq": spec.rows_per_seq,
                "softmax_scale": spec.softmax_scale, "q_idx": host_bits(inp["q_idx"]), "w": inp["w"].cpu().numpy(),
                "idx_keys": inp["idx_keys"].cpu().numpy(), "idx_key_scale": inp["idx_key_scale"].cpu().numpy(),
                "Q": [host_bits(q) for q in inp["Q"][:nl]], "KV": [x.cpu().numpy() for x in inp["KV"][:nl]],
                "KV_scale": [x.cpu().numpy() for x in inp["KV_scale"][:nl]], "n_layers_timed": nl}
    host = {"L": spec.L, "k": spec.k, "softmax_scale": spec.softmax_scale, "k_idx": host_bits(inp["k_idx"]),
            "q_idx": _LazyRows(inp["q_idx"]), "w": _LazyRows(inp["w"], bf16=False),
            "Q": [_LazyRows(q) for q in inp["Q"]], "KV": [host_bits(x) for x in inp["KV"]]}
    host["tables"] = O.prefill_tables(host, spec.indexer_fp8)
    return host


def oracle_rows_per_second(spec, name, host, budget_s, seed_rows=0):
    """Time the fp64 oracle on a bounded sample of rows of the same workload (host cores).
    Returns (rows per second, sample description, seconds)."""
    import numpy as np
    import oracle.dsa_oracle as O
    if name.startswith("decode"):
        nl = host["n_layers_timed"]
        policy = O.group_decode_per_row if spec.topk_per_row else O.group_decode
        order = list(np.random.default_rng(seed_rows).permutation(len(host["ctx"])))
        done, t0 = 0, time.perf_counter()
        while order and time.perf_counter() - t0 < budget_s:
            policy(host, seqs=[order.pop()])
            done += spec.rows_per_seq
        el = time.perf_counter() - t0
        return done / el, (f"{done // spec.rows_per_seq} whole sequences (all {spec.rows_per_seq} rows, indexer, "
                           f"Top-k and {nl} layer(s) of the first group)"), el
    L = spec.L
    rng = np.random.default_rng(seed_rows)
    rows_done, el = 0, 0.0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s or rows_done == 0:
        rows = sorted(int(r) for r in rng.integers(0, L, size=2))
        O.group_prefill(host, rows, fp8_indexer=spec.indexer_fp8, tables=host["tables"])
        rows_done += 2
    el = time.perf_counter() - t0
    return rows_done / el, (f"{rows_done} uniformly drawn query rows, 2 per oracle call (indexer + Top-k + "
                            f"{len(host['Q'])} layers each; whole-sequence tables converted once, untimed)"), el


class _LazyRows:
    """Row access to a device tensor for the oracle (copies one row to the host on demand)."""

    def __init__(self, t, bf16=True):
        self.t, self.bf16 = t, bf16

    def __getitem__(self, i):
        import numpy as np
        import torch
        r = self.t[i]
        if self.bf16:
            return r.view(torch.int16).cpu().numpy().view(np.uint16)
        return r.cpu().numpy()


def cpu_cores():
    """(threads the oracle's BLAS calls use, note): the oracle is numpy fp64 in one process."""
    try:
        from threadpoolctl import threadpool_info
        th = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        th = 1
    th = max(1, min(th, len(os.sched_getaffinity(0))))
    return th, (f"numpy fp64 in one process: the loop over rows runs on one core, its matrix products "
                f"(BLAS) on {th} threads; {len(os.sched_getaffinity(0))} host cores available")


# ----------------------------------------------------------------------------- our arm


def measure(name, args, ws, rank, local, headline):
    """Build one workload, time it and return its measurement (rank 0's view of the max over ranks)."""
    import ctypes
    import torch
    import long_context_sparse_11_b200 as dsa

    lib = dsa.load()
    dev = torch.device("cuda", local)
    spec, cfg = workload_config(name, args.seq_len if headline else None)
    mem0 = torch.cuda.memory_allocated(dev)
    wl = Workload(spec, name, dev)
    counts = wl.counts
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.int32, device=dev)   # 1 GiB > 126 MB L2
    decode = name.startswith("decode")

    # trace events per group: the Full layer's a1-a4 phase and each layer's sparse MLA launch
    # (recorded once so that torch creates the CUDA events before their handles are passed on)
    traces = []
    for g, nl in zip(wl.groups, wl.layers_per_group):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 + 2 * nl)]
        for e in evs:
            e.record(stream)
        traces.append(evs)
    torch.cuda.synchronize()
    arrs = [(ctypes.c_void_p * len(evs))(*[e.cuda_event for e in evs]) for evs in traces]
    assert all(e.cuda_event for evs in traces for e in evs)

    def step(traced):
        for g, arr in zip(wl.groups, arrs):
            g.args.trace_events = ctypes.cast(arr, ctypes.c_void_p) if traced else None
        wl.forward()

    for _ in range(args.warmup):
        step(False)
    dsa.sync_status()
    torch.cuda.synchronize()
    n0 = lib.dsa_launch_count()
    t0 = time.perf_counter()
    step(False)
    torch.cuda.synchronize()
    est_ms = 1e3 * (time.perf_counter() - t0)
    launches_per_step = lib.dsa_launch_count() - n0

    # many short kernels (decode): the step is captured once as a CUDA graph and replayed
    use_graph = args.graph == "on" or (args.graph == "auto" and decode)
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(False)
        graph.replay()
        torch.cuda.synchronize()
        dsa.sync_status()
        t0 = time.perf_counter()
        for _ in range(5):
            graph.replay()
        torch.cuda.synchronize()
        est_ms = 1e3 * (time.perf_counter() - t0) / 5

    def run_step():
        if graph is not None:
            graph.replay()
        else:
            wl.forward()

    mla_ms, idx_ms = [], []

    def timed_steps(n, traced):
        out = []
        for _ in range(n):
            flush.fill_(1)                                  # evict L2 between steps (untimed)
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            if traced:
                step(True)
            else:
                run_step()
            s1.record(stream)
            if traced or n <= 64:
                s1.synchronize()
            out.append((s0, s1))
            if traced:
                for evs, nl in zip(traces, wl.layers_per_group):
                    idx_ms.append(evs[0].elapsed_time(evs[1]))
                    mla_ms.extend(evs[2 + 2 * l].elapsed_time(evs[3 + 2 * l]) for l in range(nl))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in out]

    # the headline times exactly K steps; the other workloads at least min_timed_s of steps
    steps = args.steps
    if not headline:
        steps = max(steps, int(math.ceil(1e3 * args.min_timed_s / max(est_ms, 1e-3))))
        steps = int(max_over_ranks(float(steps), ws))
    torch.cuda.synchronize()
    barrier(ws)                                             # all ranks start the timed steps together
    with ClockSampler(gpu_smi_id(local)) as clk:
        # eager steps carry the library's phase events; graph replays are timed on their own and
        # the phase split comes from eager steps run afterwards
        t_steps = timed_steps(steps, traced=graph is None)
    torch.cuda.synchronize()
    barrier(ws)
    if graph is not None:
        timed_steps(min(steps, 20), traced=True)
        torch.cuda.synchronize()
    launches = launches_per_step * steps
    dsa.sync_status()
    total_ms = max_over_ranks(sum(t_steps), ws)
    ms_per_step = total_ms / steps
    n_groups = len(wl.groups)
    value = job_throughput(counts["tokens"] * n_groups, steps, ws, total_ms)
    clocks = clk.summary()

    hbm, bf16_peak, peak_kind = measured_peaks()
    mla_avg = statistics.mean(mla_ms)
    idx_avg = statistics.mean(idx_ms)
    mla_tf = counts["mla_flops_per_layer"] / (mla_avg / 1e3) / 1e12
    traffic = None
    if not decode:
        # DRAM bytes (read + write) of one bf16 launch grow with the query rows (queries in,
        # outputs out; the latent rows stay in L2): measured by ncu at 8,192 rows, scaled.
        traffic = {"bytes_per_launch": round(MLA_DRAM_BYTES_PER_ROW_BF16 * counts["mla_rows"]),
                   "source": "ncu dram__bytes_read.sum + dram__bytes_write.sum at L=8192, scaled by query rows"}
    mla_roof = {"kernel": "sparse_mla_kernel (a6)", "bound": "tensor", "achieved": round(mla_tf, 1),
                "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(mla_tf / bf16_peak, 4),
                "peak_source": f"{peak_kind} bf16 dense (burst)",
                "traffic": traffic["bytes_per_launch"] if traffic else None,
                "algorithmic_flops_per_launch": counts["mla_flops_per_layer"], "avg_launch_ms": round(mla_avg, 4)}
    if traffic:
        mla_roof["traffic_source"] = traffic["source"]
    phases = {"indexer_topk_ms": round(idx_avg, 4), "mla_ms_per_layer": round(mla_avg, 4),
              "indexer_topk_tflops": round(counts["indexer_flops"] / (idx_avg / 1e3) / 1e12, 1),
              "groups_per_step": n_groups}
    if counts.get("mla_gather_bytes_per_layer"):
        # context for the sparse MLA roofline: the selected 1,152-byte latent rows it gathers from
        # L2 into shared memory per launch, as an aggregate rate (the kernel's limiter, not HBM)
        phases["mla_gather_tbs"] = round(counts["mla_gather_bytes_per_layer"] / (mla_avg / 1e3) / 1e12, 2)
    roofline = mla_roof
    if counts.get("indexer_bytes"):
        gbs = counts["indexer_bytes"] / (idx_avg / 1e3) / 1e9
        phases["indexer_topk_gbs"] = round(gbs, 1)
        phases["indexer_topk_hbm_frac"] = round(gbs / hbm, 4)
        mla_gbs = counts["mla_bytes_per_layer"] / (mla_avg / 1e3) / 1e9
        phases["mla_gbs"] = round(mla_gbs, 1)
        if wl.spec.rows_per_seq == 1:
            # one row per sequence: 139,264 flops per 580 gathered bytes, a memory-bound kernel
            mla_roof = {"kernel": "sparse_mla_kernel<paged e4m3> (a6, a7)", "bound": "hbm",
                        "achieved": round(mla_gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(mla_gbs / hbm, 4),
                        "peak_source": f"{peak_kind} HBM copy", "traffic": None,
                        "algorithmic_bytes_per_launch": counts["mla_bytes_per_layer"],
                        "avg_launch_ms": round(mla_avg, 4)}
            roofline = mla_roof
        if idx_avg * n_groups > mla_avg * sum(wl.layers_per_group):
            roofline = {"kernel": "indexer_kernel<e4m3,paged> + topk (a2-a4)", "bound": "hbm",
                        "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                        "peak_source": f"{peak_kind} HBM copy", "traffic": None,
                        "algorithmic_bytes_per_launch": counts["indexer_bytes"], "avg_launch_ms": round(idx_avg, 4)}
            phases["mla_roofline"] = mla_roof
    if n_groups > 1:
        phases["step_ms_all_layers"] = round(ms_per_step, 4)
    if not decode:
        # the indexer kernel alone against the tensor peak of its input type (e4m3: the measured
        # bf16 peak x 2, the nominal fp8 / bf16 ratio)
        ia_ms, ia_launches = indexer_alone(wl, wl.spec, dev, stream)
        ia_tf = counts["indexer_flops"] / (ia_ms / 1e3) / 1e12
        ia_peak = bf16_peak * (2.0 if wl.spec.indexer_fp8 else 1.0)
        phases["indexer_alone"] = {"ms": round(ia_ms, 4), "launches": ia_launches, "tflops": round(ia_tf, 1),
                                   "peak": round(ia_peak, 1), "frac": round(ia_tf / ia_peak, 4),
                                   "peak_source": f"{peak_kind} bf16 dense (burst)" +
                                   (" x 2 (fp8 / bf16 nominal)" if wl.spec.indexer_fp8 else "")}
        if wl.spec.indexer_fp8:
            f8 = fp8_dense_peak(dev)
            if f8:
                phases["indexer_alone"].update({
                    "fp8_gemm_tflops": round(f8, 1), "frac_of_fp8_gemm": round(ia_tf / f8, 4),
                    "fp8_gemm_source": "library e4m3 GEMM on this GPU (torch._scaled_mm, 8192^3, bf16 out, "
                                       "best of 10)"})
        proj = input_projections(wl.spec.L, dev, stream)
        for v in proj.values():
            v.update({"peak": bf16_peak, "frac": round(v["tflops"] / bf16_peak, 4),
                      "peak_source": f"{peak_kind} bf16 dense (burst)"})
        phases["input_projections"] = proj
        # the IndexShare group against the same sequence run as 4 independent Full layers, both timed
        full_ms = independent_full_layers(wl, wl.spec, stream, flush)
        phases["indexshare_vs_independent_full_layers"] = {
            "group_ms": round(ms_per_step, 3), "independent_full_layers_ms": round(full_ms, 3),
            "ratio": round(ms_per_step / full_ms, 4),
            "how": "both timed with CUDA events, L2 flushed before each; the 4 independent layers are 4 "
                   "one-layer group calls that each run their own a1-a4 and a6"}

    per_set = torch.cuda.memory_allocated(dev) - mem0   # one set of inputs, outputs and workspace

    def make_twin():
        """A second set of device inputs/outputs (the same seeded data), so that one step's upload
        can run while the previous step computes; None when the GPU has no room for it (the free
        device memory plus what the caching allocator holds unused, against one set's bytes and a
        3 GiB margin; an allocation that still fails falls back to one set)."""
        free, _ = torch.cuda.mem_get_info(dev)
        avail = free + torch.cuda.memory_reserved(dev) - torch.cuda.memory_allocated(dev)
        if avail < per_set + (3 << 30):
            return None
        try:
            wl2 = Workload(spec, name, dev)
            wl2.forward()
            g2 = None
            if graph is not None:
                g2 = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g2):
                    wl2.forward()
            torch.cuda.synchronize()
        except torch.cuda.OutOfMemoryError:
            wl2 = g2 = None
            gc.collect()
            torch.cuda.empty_cache()
            return None
        return wl2, (g2.replay if g2 is not None else wl2.forward), g2

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, stream, ws, run_step, make_twin)

    cpu = None
    if headline and rank == 0 and not args.no_cpu_baseline and ws == 1:
        host = host_inputs(spec, name, wl.inp)
        v, sample, el = oracle_rows_per_second(spec, name, host, args.cpu_seconds)
        cores, note = cpu_cores()
        cpu = {"value": round(v, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(el, 1), "threads_note": note}
        del host
    cfg.update({"l2": "flushed (1 GiB write) between timed steps", "parallelism": f"replicas x{ws}",
                "cuda_graph": graph is not None})
    res = {"value": round(value, 1), "ms_per_step": round(ms_per_step, 4), "steps": steps, "warmup": args.warmup,
           "dtype": workload_dtype(name), "config": cfg, "roofline": roofline, "phases": phases, "e2e": e2e,
           "gpu_launches": launches, "clocks": clocks}
    if cpu is not None:
        res["cpu_baseline"] = cpu
    del graph, wl, flush, traces, arrs
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_ours(args, ws, rank, local):
    import torch
    import long_context_sparse_11_b200 as dsa
    from long_context_sparse_11_b200.build import build

    build()
    dsa.load()
    torch.cuda.set_device(torch.device("cuda", local))
    head_name = HEADLINE if args.workload == "all" else args.workload
    head = measure(head_name, args, ws, rank, local, headline=True)
    subs = {}
    if args.workload == "all" and not args.no_sub:
        for name in SUB_WORKLOADS:
            subs[name] = measure(name, args, ws, rank, local, headline=False)
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
                "data": "synthetic (seeded SplitMix64 normals)", "config": head["config"],
                "roofline": head["roofline"], "phases": head["phases"], "cpu_baseline": head.get("cpu_baseline"),
                "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"]}
        if subs:
            line["workloads"] = subs
        print(json.dumps(line), flush=True)


def run_e2e(args, wl, stream, ws, run_step, make_twin=None):
    """Same metric through the public API with host buffers: every step copies its inputs from
    pinned host memory to the device, runs the groups and reads the outputs back.  Uploads and
    downloads run on their own streams; with a second set of device buffers (when the GPU has room)
    consecutive steps alternate between the two sets, so step i+1's upload overlaps step i's
    compute and step i-1's download.  A step's compute waits for its own upload and for the download
    of the outputs its buffer set held two steps earlier."""
    import torch
    import long_context_sparse_11_b200 as dsa
    host_in = [t.cpu().pin_memory() for t in wl.step_inputs]
    host_out = [torch.empty_like(o, device="cpu").pin_memory() for o in wl.outputs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(2, min(args.steps, 5))
    if wl.name.startswith("decode"):
        steps = 50                      # short steps: enough of them for a stable ratio
    sets = [(wl, run_step)]
    twin = make_twin() if make_twin is not None else None
    if twin is not None:
        sets.append((twin[0], twin[1]))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    last = [{"computed": None, "downloaded": None} for _ in sets]
    count = [0]

    def one():
        b = count[0] % len(sets)
        count[0] += 1
        w, run = sets[b]
        ev_in, ev_comp, ev_out = torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()
        if last[b]["computed"] is not None:
            s_in.wait_event(last[b]["computed"])       # this set's previous step has read its inputs
        with torch.cuda.stream(s_in):
            for h, d in zip(host_in, w.step_inputs):
                d.copy_(h, non_blocking=True)
            ev_in.record(s_in)
        stream.wait_event(ev_in)
        if last[b]["downloaded"] is not None:
            stream.wait_event(last[b]["downloaded"])   # this set's previous outputs are on the host
        run()
        ev_comp.record(stream)
        s_out.wait_event(ev_comp)
        with torch.cuda.stream(s_out):
            for h, d in zip(host_out, w.outputs):
                h.copy_(d, non_blocking=True)
            ev_out.record(s_out)
        last[b]["computed"], last[b]["downloaded"] = ev_comp, ev_out

    for _ in sets:
        one()
    torch.cuda.synchronize()
    barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)                                # no upload starts before the timer
    for _ in range(steps):
        one()
    for l in last:
        stream.wait_event(l["downloaded"])
    e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), ws)
    dsa.sync_status()
    tokens = wl.counts["tokens"] * len(wl.groups)
    res = {"value": round(tokens * ws * steps / (ms / 1e3), 1), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
           "ms_per_step": round(ms / steps, 3), "device_buffer_sets": len(sets)}
    del host_in, host_out, sets, twin
    gc.collect()
    return res


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, ws, rank):
    """fp64 oracle on the host cores: each step a bounded sample of the same (headline) workload."""
    if rank != 0:
        return
    import torch
    name = HEADLINE if args.workload == "all" else args.workload
    spec, cfg = workload_config(name, args.seq_len)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    from synth import make_prefill, make_decode
    if name.startswith("decode"):
        inp = make_decode(spec, device=dev)
    else:
        inp = make_prefill(spec, device=dev)
    host = host_inputs(spec, name, inp)                    # untimed set-up: host copies, fp64 tables
    per_step = max(1.0, args.ref_seconds / (args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_rows_per_second(spec, name, host, per_step, seed_rows=99)
    tot_rows, tot_s, sample = 0.0, 0.0, ""
    for i in range(args.steps):
        v, sample, el = oracle_rows_per_second(spec, name, host, per_step, seed_rows=i)
        tot_rows += v * el
        tot_s += el
    value = tot_rows / tot_s
    cfg.update({"parallelism": "host cores, rank 0 only"})
    cores, note = cpu_cores()
    cpu = {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"per step: {sample}, about {per_step:.1f} s", "threads_note": note}
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64 normals)", "config": cfg, "cpu_baseline": cpu,
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    if args.gpus != ws and ws > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {ws}", file=sys.stderr)
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

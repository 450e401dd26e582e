#!/usr/bin/env python
"""Benchmark of the RaZeR hot path on B200.

Workload (one step): the Llama-3-8B decode projections in RaZeR weight format.
Each step quantizes the three fp16 weight matrices (4096x4096, 14336x4096,
4096x14336; N(0, 0.02^2) with 0.1% x10 outliers) and runs the W4A16 GEMV at
batch 1, 4 and 16 (fp16 activations N(0, 1), fp16 outputs) on each of them.
The GEMVs of step s read the packed weights written by step s-1 (two packed
sets alternate), so between writing and reading a packed matrix more than
600 MB of other traffic has passed through the 126 MB L2; the fp16 inputs
(268 MB) are larger than L2 as well.

value  = algorithmic bytes of all ranks' steps / max-over-ranks device time
         (quantizer: 2 B read for the amax pass + 2 B read + 0.5625 B written
         per weight; GEMV: 0.5625 N K + 2 B K + 2 B N bytes per call).
Breakdown: per-call device times (CUDA events on the launching stream), the
activation quantizer on 2048x4096 bf16 with outlier channels, and the
tcgen05 GEMM on the prefill shapes when the library supports it.

--impl reference times the CPU oracle (single thread, as it stands) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RaZeR W4A16 GEMV HBM GB/s & GEMM TFLOP/s vs B200 roofline; quantize GB/s"
SHAPES = [(4096, 4096), (14336, 4096), (4096, 14336)]  # (N, K) of the Llama-3-8B projections
BATCHES = [1, 4, 16]
WORKLOAD = ("llama3-8b-decode-w4a16: quantize the 3 projections (one batched call) + GEMV of the 3 projections at "
            "B=1, 4, 16 (fp16; one batched call per B)")


def quant_bytes(N, K):
    return N * K * (2 + 2 + 0.5625)


def gemv_bytes(B, N, K):
    return 0.5625 * N * K + 2 * B * K + 2 * B * N


def step_bytes():
    return sum(quant_bytes(N, K) for N, K in SHAPES) + sum(gemv_bytes(B, N, K) for N, K in SHAPES for B in BATCHES)


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank number (device time in ms) over all ranks."""
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


TRAFFIC_SOURCES = {  # the files each timed call's kernels are built from
    "quantize_batch": ["quantize.cu", "razer_internal.cuh"],
    "gemv_batch": ["gemv_tma.cu", "gemv.cu", "sm100_async.cuh", "razer_internal.cuh"],
}


def source_hash(files):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantization_razer_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str):
    """DRAM bytes per call from the committed ncu summary, if it was taken on
    the current sources of that kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get("kernels", {}).get(kernel)
    if not e or e.get("source_hash") != source_hash(TRAFFIC_SOURCES[kernel]):
        return None
    return e.get("bytes_per_call")


def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (every one is a launch of this
    library's kernels in the bench step), or None if the graph cannot be read."""
    try:
        from cuda.bindings import runtime as rt

        h = g.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(h, 0)
        err, nodes, n = rt.cudaGraphGetNodes(h, n)
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
        return sum(1 for t in kinds if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------
def run_reference(args, rank):
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from bit_quantization_razer_b200 import workloads

    oracle.build()
    rows_per_shape = 8
    ws = [workloads.weight(N, K, seed=100 + i) for i, (N, K) in enumerate(SHAPES)]
    xs = {B: [workloads.vectors(B, K, seed=10 + B) for _, K in SHAPES] for B in BATCHES}

    def one_step():
        nbytes = 0.0
        for i, (N, K) in enumerate(SHAPES):
            w = ws[i]
            ts = oracle.tensor_scale(w.numpy(), 0)  # full-tensor amax pass
            sub = w[:rows_per_shape].numpy()
            codes, scales, _, _ = oracle.quantize(sub, 0, ts=ts)
            nbytes += N * K * 2 + rows_per_shape * K * 2.5625
            for B in BATCHES:
                oracle.gemm_ref(xs[B][i].numpy(), codes, scales, ts, 0)
                nbytes += gemv_bytes(B, rows_per_shape, K)
        return nbytes

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    tot = 0.0
    for _ in range(args.steps):
        tot += one_step()
    dt = time.perf_counter() - t0
    value = tot / dt / 1e9
    sample = f"per step: full amax pass of each projection + quantize and GEMV (B=1,4,16) of {rows_per_shape} rows of each"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------
def cpu_baseline_sample():
    """The oracle as it stands, single-threaded, on a bounded sample (~10 s)."""
    import oracle
    from bit_quantization_razer_b200 import workloads

    oracle.build()
    ws = [workloads.weight(N, K, seed=100 + i) for i, (N, K) in enumerate(SHAPES)]
    x = {B: [workloads.vectors(B, K, seed=10 + B) for _, K in SHAPES] for B in BATCHES}
    rows = 64
    t0 = time.perf_counter()
    nbytes = 0.0
    for i, (N, K) in enumerate(SHAPES):
        ts = oracle.tensor_scale(ws[i].numpy(), 0)
        codes, scales, _, _ = oracle.quantize(ws[i][:rows].numpy(), 0, ts=ts)
        nbytes += N * K * 2 + rows * K * 2.5625
        for B in BATCHES:
            oracle.gemm_ref(x[B][i].numpy(), codes, scales, ts, 0)
            nbytes += gemv_bytes(B, rows, K)
    dt = time.perf_counter() - t0
    res = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"per projection: full amax pass + quantize and GEMV (B=1,4,16) of {rows} rows ({dt:.1f} s)"}
    try:
        res["all_cores"] = cpu_baseline_all_cores(ws, x, rows)
    except Exception as e:  # the single-thread figure stands on its own
        res["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    try:
        res["gemm"] = cpu_gemm_sample()
    except Exception as e:
        res["gemm"] = {"unavailable": f"{type(e).__name__}: {e}"}
    return res


def cpu_gemm_sample():
    """The oracle's GEMM reference (double accumulation, single thread) on the
    prefill GEMM shapes: timed on two sampled row counts, and the full
    product's time extrapolated from the fit (a fixed part -- the oracle
    decodes the weights once per call -- plus a part per row of X), labelled
    as an extrapolation."""
    import oracle
    import torch
    from bit_quantization_razer_b200 import workloads

    out = {}
    for M, N, K, r1, r2 in ((4096, 4096, 4096, 4, 20), (4096, 14336, 4096, 2, 6)):
        codes, scales = workloads.random_packed(N, K, "weight", seed=N + K, max_scale_code=40)
        t = []
        for rows in (r1, r2):
            X = workloads.vectors(rows, K, seed=M + rows, dtype=torch.bfloat16)
            xb = oracle.Bf16Bits(workloads.to_numpy_bits(X))
            t0 = time.perf_counter()
            oracle.gemm_ref(xb, codes.numpy(), scales.numpy(), 0.01, 0)
            t.append(time.perf_counter() - t0)
        per_row = max((t[1] - t[0]) / (r2 - r1), 1e-12)
        fixed = max(t[0] - r1 * per_row, 0.0)
        full = fixed + M * per_row
        out[f"{M}x{N}x{K}"] = {"value": 2.0 * M * N * K / full / 1e9, "unit": "GFLOP/s", "cores": 1, "kind": "oracle",
                               "extrapolated": True, "extrapolated_full_s": full,
                               "sample": f"{r1} and {r2} rows of {M} timed ({t[0]:.2f} s, {t[1]:.2f} s), fixed + per-row fit"}
    return out


def _oracle_rows_worker(rank, nproc, ws, x, rows, tsbuf, start, mid, done):
    """One process of the multi-core oracle run: the amax pass over its share
    of each projection's rows, then (with the tensor scale of the whole
    matrix, the maximum of every process's share) the quantizer and the
    GEMVs of its share of the `rows` sampled rows."""
    import oracle

    oracle.build()
    start.wait()
    for i, (N, K) in enumerate(SHAPES):
        r0, r1 = rank * N // nproc, (rank + 1) * N // nproc
        tsbuf[rank, i] = oracle.tensor_scale(ws[i][r0:r1].numpy(), 0)
    mid.wait()
    q0, q1 = rank * rows // nproc, (rank + 1) * rows // nproc
    for i, (N, K) in enumerate(SHAPES):
        ts = float(tsbuf[:, i].max())
        if q1 > q0:
            codes, scales, _, _ = oracle.quantize(ws[i][q0:q1].numpy(), 0, ts=ts)
            for B in BATCHES:
                oracle.gemm_ref(x[B][i].numpy(), codes, scales, ts, 0)
    done.wait()


def cpu_baseline_all_cores(ws, x, rows):
    """The same sample with the same oracle, unchanged, split over one process
    per host core (up to 16; spawned, so no process inherits a CUDA context):
    the amax pass and the sampled rows are divided by rows.  Wall time between
    two barriers shared by every process (start-up and exit excluded)."""
    import torch
    import torch.multiprocessing as mp

    nproc = max(1, min(os.cpu_count() or 1, 16))
    ctx = mp.get_context("spawn")
    shared = [w.share_memory_() for w in ws]
    xs = {B: [t.share_memory_() for t in v] for B, v in x.items()}
    tsbuf = torch.zeros((nproc, len(SHAPES)), dtype=torch.float32).share_memory_()
    start, mid, done = ctx.Barrier(nproc + 1), ctx.Barrier(nproc), ctx.Barrier(nproc + 1)
    procs = [ctx.Process(target=_oracle_rows_worker, args=(r, nproc, shared, xs, rows, tsbuf, start, mid, done))
             for r in range(nproc)]
    for p in procs:
        p.start()
    try:
        start.wait(timeout=600)
        t0 = time.perf_counter()
        done.wait(timeout=600)
        dt = time.perf_counter() - t0
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    if any(p.exitcode != 0 for p in procs):
        raise RuntimeError("an oracle process failed")
    nbytes = sum(N * K * 2 + rows * K * 2.5625 + sum(gemv_bytes(B, rows, K) for B in BATCHES) for N, K in SHAPES)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": nproc, "kind": "oracle",
            "sample": f"the single-core sample split by rows over {nproc} processes ({dt:.2f} s)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="razer", choices=["razer", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the breakdown / e2e / GEMM legs")
    ap.add_argument("--no-soak", action="store_true", help="skip the 1.5 s pre-timing load for the clock sampler")
    ap.add_argument("--kernel", choices=["quantize", "quantize_batch", "act_quantize", "dequant", "gemv", "gemv_batch", "gemv_variant",
                             "gemm"],
                    help="profiling mode: run one call on --shape in a loop (for ncu)")
    ap.add_argument("--shape", default="4096,4096", help="N,K (gemm: M,N,K; quantize_batch: N1,K1,N2,K2,...)")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.kernel:
        run_single_kernel(args)
        return

    import torch

    import bit_quantization_razer_b200 as R
    from bit_quantization_razer_b200 import workloads

    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    R.load()
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    # inputs (host-generated, seeded), resident in HBM before timing
    W = [workloads.weight(N, K, seed=100 + i).to(dev) for i, (N, K) in enumerate(SHAPES)]
    X = {B: [workloads.vectors(B, K, seed=10 + B).to(dev) for _, K in SHAPES] for B in BATCHES}
    # two packed sets (codes, scales, ts [3]) alternate between steps
    packed = [([torch.empty((N, K // 2), dtype=torch.uint8, device=dev) for N, K in SHAPES],
               [torch.empty((N, K // 16), dtype=torch.uint8, device=dev) for N, K in SHAPES],
               torch.empty(len(SHAPES), dtype=torch.float32, device=dev)) for _ in range(2)]
    Y = {B: [torch.empty((B, N), dtype=torch.float16, device=dev) for N, _ in SHAPES] for B in BATCHES}
    wsz = max(R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K) for N, K in SHAPES for B in BATCHES)

    # one batched GEMV call per B over the three (distinct) projections: the
    # products of one call share no weights, so no call reads a matrix that
    # another product of the same call also streams
    def gemv_problems(pk, B):
        return [(X[B][i], pk[0][i], pk[1][i], pk[2][i:i + 1]) for i in range(len(SHAPES))]

    wsz = max([wsz] + [R.razer_gemv_batch_workspace_size(gemv_problems(packed[0], B)) for B in BATCHES])
    ws = torch.empty(max(wsz, 16), dtype=torch.uint8, device=dev)

    def step(s):
        cur, prev = packed[s % 2], packed[(s + 1) % 2]
        R.razer_quantize_weights_batch(W, "weight", codes=cur[0], scales=cur[1], ts=cur[2])
        for B in BATCHES:
            R.razer_gemv_batch(gemv_problems(prev, B), "weight", torch.float16, outs=Y[B], workspace=ws)

    # the first GEMVs read the second packed set: fill it; warm every path
    step(1)
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    # one CUDA graph per step parity (the launches of a step replay without
    # host overhead; the work inside is unchanged)
    graphs = []
    for par in range(2):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            step(par)
        graphs.append(g)
    for g in graphs:
        g.instantiate()
    kernels_per_step = graph_kernel_nodes(graphs[0])
    for s in range(3):
        graphs[s % 2].replay()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        # keep the same load running ~1.5 s first: nvidia-smi needs time to
        # start and the timed region itself lasts only milliseconds
        t_end = time.time() + (0.0 if args.no_soak else 1.5)
        s = 0
        while time.time() < t_end:
            graphs[s % 2].replay()
            s += 1
            if s % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(args.steps):
            graphs[s % 2].replay()
        t1.record(stream)
        torch.cuda.synchronize()
    elapsed_ms = t0.elapsed_time(t1)
    if pg:
        elapsed_ms = max_over_ranks(elapsed_ms, pg, dev)
        pg.barrier()
    ms_per_step = elapsed_ms / args.steps
    value = step_bytes() * args.steps * world / (elapsed_ms / 1e3) / 1e9

    # per-call device time: a graph of back-to-back calls of one kind, each on
    # its own copy of the operands so that the copies together exceed L2
    l2 = 126 * 2 ** 20
    breakdown, by_kind = {}, {}
    for i, (N, K) in enumerate(SHAPES):
        ncopy = max(2, -(-2 * l2 // (N * K * 2)))
        Wc = [W[i]] + [W[i].clone() for _ in range(ncopy - 1)]
        outs = [(torch.empty_like(packed[0][0][i]), torch.empty_like(packed[0][1][i]), torch.empty(1, dtype=torch.float32, device=dev))
                for _ in range(ncopy)]
        for r in range(ncopy):
            R.razer_quantize_weights(Wc[r], "weight", codes=outs[r][0], scales=outs[r][1], ts=outs[r][2])
        ms = time_graph(lambda: [R.razer_quantize_weights(Wc[r], "weight", codes=outs[r][0], scales=outs[r][1], ts=outs[r][2])
                                 for r in range(ncopy)], ncopy, stream)
        nb = quant_bytes(N, K)
        breakdown[f"quantize_{N}x{K}"] = {"ms": ms, "GB/s": nb / ms / 1e6}
        del Wc
        npk = max(2, -(-2 * l2 // (N * K * 9 // 16)))
        pk = [outs[r % len(outs)] for r in range(npk)]
        pk = [(c.clone(), sc.clone(), t.clone()) for (c, sc, t) in pk]
        for B in BATCHES:
            ms = time_graph(lambda: [R.razer_gemv(X[B][i], *pk[r], "weight", torch.float16, out=Y[B][i], workspace=ws)
                                     for r in range(npk)], npk, stream)
            nb = gemv_bytes(B, N, K)
            breakdown[f"gemv_{N}x{K}_b{B}"] = {"ms": ms, "GB/s": nb / ms / 1e6}
        del pk, outs
    # the step's quantize call: all three projections in one batched call,
    # two weight sets alternating (536 MB of fp16 input, > 2x L2)
    Wsets = [W, [w.clone() for w in W]]
    qouts = [([torch.empty_like(c) for c in packed[0][0]], [torch.empty_like(c) for c in packed[0][1]], torch.empty_like(packed[0][2]))
             for _ in range(2)]
    ms = time_graph(lambda: [R.razer_quantize_weights_batch(Wsets[r], "weight", codes=qouts[r][0], scales=qouts[r][1], ts=qouts[r][2])
                             for r in range(2)], 2, stream)
    nb = sum(quant_bytes(N, K) for N, K in SHAPES)
    breakdown["quantize_batch_3proj"] = {"ms": ms, "GB/s": nb / ms / 1e6}
    by_kind["quantize"] = [ms, nb, 1]
    # the step's GEMV calls: one batched call per B over the three
    # projections, each on three copies of the packed weights (3 x 75 MB, > L2)
    pks = [packed[0]] + [([c.clone() for c in packed[0][0]], [c.clone() for c in packed[0][1]], packed[0][2].clone()) for _ in range(2)]
    by_kind["gemv"] = [0.0, 0.0, 0]
    for B in BATCHES:
        ms = time_graph(lambda: [R.razer_gemv_batch(gemv_problems(pks[r], B), "weight", torch.float16, outs=Y[B], workspace=ws)
                                 for r in range(3)], 3, stream)
        nb = sum(gemv_bytes(B, N, K) for N, K in SHAPES)
        breakdown[f"gemv_batch_3proj_b{B}"] = {"ms": ms, "GB/s": nb / ms / 1e6}
        by_kind["gemv"][0] += ms
        by_kind["gemv"][1] += nb
        by_kind["gemv"][2] += 1
    del Wsets, qouts, pks
    torch.cuda.empty_cache()
    dominant = max(by_kind, key=lambda k: by_kind[k][0])
    dom_ms, dom_bytes, n_calls = by_kind[dominant]
    achieved = dom_bytes / dom_ms / 1e6  # GB/s over that kind's calls
    kname = "quantize_batch" if dominant == "quantize" else "gemv_batch"
    traffic = traffic_for(kname)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic, "kernel": ("razer_quantize_weights_batch of the 3 projections (amax, fused quantize + "
                                               "next-amax, quantize kernels)" if dominant == "quantize"
                                               else "razer_gemv_batch of the 3 projections, per B (bulk-tensor + split-K "
                                                    "reduce kernels)"),
                "algorithmic_bytes_per_call": dom_bytes / n_calls, "peak_source": peak_src,
                "nominal_peak": 8000.0, "frac_nominal": achieved / 8000.0,
                "timing": "CUDA events around CUDA-graph replays of at least 50 back-to-back calls on operand copies "
                          "larger than L2 (median of 5 replays)"}
    if traffic:
        # the same time against the DRAM bytes ncu counted for one call (a
        # pass may find part of its matrix still in L2 from the previous pass)
        dram = traffic / (dom_ms / n_calls) / 1e6
        roofline.update({"dram_achieved": dram, "dram_frac": dram / hbm, "dram_frac_nominal": dram / 8000.0})

    extras = {}
    if not args.no_extras and rank == 0:
        extras = run_extras(R, workloads, dev, stream, hbm, bf16)

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_extras:
        e2e = run_e2e(R, workloads, dev, stream, args, world, pg)

    # kernel nodes of the captured step graph: init + amax + 2 fused stages +
    # quantize + finalize for the quantizer batch, main + reduction kernel per
    # batched GEMV call
    launches_per_step = kernels_per_step if kernels_per_step is not None else 6 + 2 * len(BATCHES)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": None, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (268 MB fp16 weights per step); packed weights double-buffered "
                         "across steps so each GEMV reads weights written one step (600+ MB of traffic) earlier",
                   "bytes_per_step": step_bytes()},
        "roofline": roofline,
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * args.steps,
        "breakdown": breakdown,
    }
    line.update(extras)
    if e2e:
        line["e2e"] = e2e
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_single_kernel(args):
    """One API call on one shape, 3 warm-up + --iters timed calls (ncu target)."""
    import torch

    import bit_quantization_razer_b200 as R
    from bit_quantization_razer_b200 import workloads

    dev = torch.device("cuda", 0)
    dims = [int(v) for v in args.shape.split(",")]
    if args.kernel in ("quantize", "dequant", "gemv"):
        N, K = dims
        w = workloads.weight(N, K, seed=1).to(dev)
        c, s, t = R.razer_quantize_weights(w)
        x = workloads.vectors(args.batch, K, seed=2).to(dev)
        y = torch.empty((args.batch, N), dtype=torch.float16, device=dev)
        out = torch.empty((N, K), dtype=torch.float16, device=dev)
        wsb = R.razer_workspace_size(R.RAZER_OP_GEMV, args.batch, N, K)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)

        def call():
            if args.kernel == "quantize":
                R.razer_quantize_weights(w, codes=c, scales=s, ts=t)
            elif args.kernel == "dequant":
                R.razer_dequant(c, s, t, "weight", torch.float16, out=out)
            else:
                R.razer_gemv(x, c, s, t, "weight", torch.float16, out=y, workspace=ws)
    elif args.kernel == "quantize_batch":
        Ws = [workloads.weight(dims[2 * i], dims[2 * i + 1], seed=1 + i).to(dev) for i in range(len(dims) // 2)]
        cs, ss, ts = R.razer_quantize_weights_batch(Ws)

        def call():
            R.razer_quantize_weights_batch(Ws, codes=cs, scales=ss, ts=ts)
    elif args.kernel == "gemv_batch":
        # the GEMV at --batch on each N,K pair of --shape, one batched call
        pairs = [(dims[2 * i], dims[2 * i + 1]) for i in range(len(dims) // 2)]
        probs = []
        for i, (N, K) in enumerate(pairs):
            c, s, t = R.razer_quantize_weights(workloads.weight(N, K, seed=1 + i).to(dev))
            probs.append((workloads.vectors(args.batch, K, seed=2 + i).to(dev), c, s, t))
        ys = R.razer_gemv_batch(probs, "weight", torch.float16)
        ws = torch.empty(max(16, R.razer_gemv_batch_workspace_size(probs)), dtype=torch.uint8, device=dev)

        def call():
            R.razer_gemv_batch(probs, "weight", torch.float16, outs=ys, workspace=ws)
    elif args.kernel == "gemv_variant":
        # the pages' kernel format: blocks of 128, FP16 scale words, +-5/+-8
        N, K = dims
        V = [5.0, -5.0, 8.0, -8.0]
        c, s, t = R.razer_quantize_variant(workloads.weight(N, K, seed=1).to(dev), 128, "f16_scale", V)
        x = workloads.vectors(args.batch, K, seed=2).to(dev)
        y = torch.empty((args.batch, N), dtype=torch.float16, device=dev)
        ws = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMV, args.batch, N, K)), dtype=torch.uint8, device=dev)

        def call():
            R.razer_gemv_variant(x, c, s, t, 128, "f16_scale", V, torch.float16, out=y, workspace=ws)
    elif args.kernel == "act_quantize":
        M, K = dims
        xa = workloads.outlier_activations(M, K, seed=3).to(dev)
        c = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((M, K // 16), dtype=torch.uint8, device=dev)
        t = torch.empty(1, dtype=torch.float32, device=dev)
        h = torch.empty(4, dtype=torch.int64, device=dev)

        def call():
            R.razer_quantize_acts(xa, None, "act", codes=c, scales=s, ts_out=t, meta_hist=h)
    else:
        M, N, K = dims
        w = workloads.weight(N, K, seed=1).to(dev)
        c, s, t = R.razer_quantize_weights(w)
        X = workloads.vectors(M, K, seed=4, dtype=torch.bfloat16).to(dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsg = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMM, M, N, K)), dtype=torch.uint8, device=dev)

        def call():
            R.razer_gemm(X, c, s, t, "weight", torch.bfloat16, out=Y, workspace=wsg)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        call()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"kernel": args.kernel, "shape": dims, "batch": args.batch,
                      "ms_per_call": e0.elapsed_time(e1) / args.iters}), flush=True)


def time_graph(fn, ncalls, stream, reps=5):
    """Median device time of one call in a back-to-back sequence: fn() issues
    `ncalls` calls; fn() is captured enough times for at least 50 calls per
    CUDA graph (so the graph launch itself is amortised), and the graph is
    replayed `reps` times between events."""
    import torch

    inner = max(1, -(-50 // ncalls))
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(inner):
            fn()
    g.replay()
    torch.cuda.synchronize()
    times = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / (ncalls * inner))
    del g
    return statistics.median(times)


def run_extras(R, workloads, dev, stream, hbm, bf16):
    import torch

    out = {}
    # online activation quantizer: 2048 x 4096 bf16, 8 outlier channels x50
    Xa = [workloads.outlier_activations(2048, 4096, seed=300 + i).to(dev) for i in range(8)]  # 8 x 16.8 MB > L2
    codes = torch.empty((2048, 2048), dtype=torch.uint8, device=dev)
    scales = torch.empty((2048, 256), dtype=torch.uint8, device=dev)
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    hist = torch.empty(4, dtype=torch.int64, device=dev)
    # both dynamic-scale paths (identical outputs).  X is read from HBM once
    # by either: the single-pass kernel holds it in shared memory, the
    # two-pass form's second read comes from L2 (16.8 MB; the 8 rotating
    # inputs together exceed L2, so every first read is from HBM).  Bytes per
    # element: 2 in + 0.5625 out from HBM; the two-pass form's algorithmic
    # count is 4.5625 (X read twice).
    paths = {}
    for path in ("two_pass", "single_pass"):
        prev = R.razer_set_quantize_path(path)
        try:
            ms_p = time_graph(lambda: [R.razer_quantize_acts(Xa[r], None, "act", codes=codes, scales=scales, ts_out=ts, meta_hist=hist)
                                       for r in range(8)], 8, stream)
        finally:
            R.razer_set_quantize_path(prev)
        paths[path] = ms_p
    ms = paths["two_pass"]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 2048 * 4096
    h = hist.cpu().tolist()
    nblk = n // 16
    out["act_quantize"] = {"ms": ms, "default_path": "two_pass",
                           "paths": {p: {"ms": m, "GB/s_hbm_bytes": n * 2.5625 / m / 1e6, "frac_hbm_bytes": n * 2.5625 / m / 1e6 / hbm,
                                         "GB/s_algorithmic": n * (4.5625 if p == "two_pass" else 2.5625) / m / 1e6}
                                     for p, m in paths.items()},
                           "meta_fraction": {"+5": h[0] / nblk, "-5": h[1] / nblk},
                           "effective_fraction": {"+5": h[2] / nblk, "-5": h[3] / nblk}}
    # tcgen05 GEMM on the prefill shapes
    try:
        Xg = workloads.vectors(4096, 4096, seed=400, dtype=torch.bfloat16).to(dev)
        res = {}
        for N, K in [(4096, 4096), (14336, 4096)]:
            w = workloads.weight(N, K, seed=401).to(dev)
            c, s, t = R.razer_quantize_weights(w)
            Yg = torch.empty((4096, N), dtype=torch.bfloat16, device=dev)
            wsg = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMM, 4096, N, K)), dtype=torch.uint8, device=dev)
            for _ in range(3):
                R.razer_gemm(Xg, c, s, t, "weight", torch.bfloat16, out=Yg, workspace=wsg)
            reps = 20
            e0.record(stream)
            for _ in range(reps):
                R.razer_gemm(Xg, c, s, t, "weight", torch.bfloat16, out=Yg, workspace=wsg)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            tf = 2 * 4096 * N * K / ms / 1e9
            res[f"{4096}x{N}x{K}"] = {"ms": ms, "TFLOP/s": tf, "frac": tf / bf16, "frac_nominal_2250": tf / 2250.0}
        out["gemm"] = res
    except R.RazerError as e:
        out["gemm"] = {"unavailable": str(e)}
    # W4A4: activations quantized online (E4M3 + 1-bit meta), weights offline;
    # the call decodes both operands and runs the tcgen05 product
    try:
        M, N, K = 4096, 4096, 4096
        ca, sa, ta, _ = R.razer_quantize_acts(workloads.outlier_activations(M, K, seed=402).to(dev), hist=False)
        cw, sw, tw = R.razer_quantize_weights(workloads.weight(N, K, seed=403).to(dev))
        Yw = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsw = torch.empty(R.razer_workspace_size(R.RAZER_OP_GEMM_W4A4, M, N, K), dtype=torch.uint8, device=dev)
        call = lambda: R.razer_gemm_w4a4(ca, sa, ta, cw, sw, tw, "act", "weight", torch.bfloat16, out=Yw, workspace=wsw)
        for _ in range(3):
            call()
        reps = 20
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        tf = 2 * M * N * K / ms / 1e9
        res = {f"{M}x{N}x{K}": {"ms": ms, "TFLOP/s": tf, "frac": tf / bf16, "includes": "decode of both operands + tcgen05 product"}}
        # the online path from bf16 activations: quantize (dynamic ts) + product
        Xa = workloads.outlier_activations(M, K, seed=402).to(dev)
        online = lambda: R.razer_gemm_w4a4_online(Xa, cw, sw, tw, None, "act", "weight", torch.bfloat16, out=Yw, workspace=wsw)
        two = lambda: (R.razer_quantize_acts(Xa, None, "act", codes=ca, scales=sa, ts_out=ta, hist=False),
                       R.razer_gemm_w4a4(ca, sa, ta, cw, sw, tw, "act", "weight", torch.bfloat16, out=Yw, workspace=wsw))
        for name, fn in (("online_fused", online), ("online_two_calls", two)):
            for _ in range(3):
                fn()
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            msn = e0.elapsed_time(e1) / reps
            res[f"{M}x{N}x{K}_{name}"] = {"ms": msn, "TFLOP/s": 2 * M * N * K / msn / 1e9,
                                           "includes": "activation quantization (dynamic ts) + decode + product"}
        out["gemm_w4a4"] = res
    except R.RazerError as e:
        out["gemm_w4a4"] = {"unavailable": str(e)}
    # accuracy ablation: quantization MSE of RaZeR, plain NVFP4 and
    # FourOverSix on a decode-shape weight matrix and on outlier activations
    # (error sums on the GPU, razer_quant_error)
    abl = {}
    for name, X, razer_fmt in (("weights_14336x4096_fp16", workloads.weight(14336, 4096, seed=404).to(dev), "weight"),
                               ("activations_2048x4096_bf16", workloads.outlier_activations(2048, 4096, seed=405).to(dev), "act")):
        res = {}
        for fmt, dec in (("nvfp4", "nvfp4"), ("four_over_six", "nvfp4"), (razer_fmt, razer_fmt)):
            if fmt == "act":
                c, s, t, _ = R.razer_quantize_acts(X, None, "act", hist=False)
            else:
                c, s, t = R.razer_quantize_weights(X, fmt)
            res[fmt] = float(R.razer_quant_error(X, c, s, t, dec).cpu()[0]) / X.numel()
        res["razer_over_nvfp4"] = res[razer_fmt] / res["nvfp4"]
        res["four_over_six_over_nvfp4"] = res["four_over_six"] / res["nvfp4"]
        abl[name] = res
    out["accuracy_ablation_mse"] = abl
    # format variants on a 4096x4096 weight matrix: the block-size study
    # (RaZeR with +-5/+-8 vs plain NVFP4 rounding at blocks of 16..128) and the
    # weights-only search over special-value pairs +-a/+-b (E3M3, block 16)
    Wv = workloads.weight(4096, 4096, seed=406).to(dev)
    mse = lambda block, sfmt, V: float(R.razer_quant_error_variant(Wv, block, sfmt, V, *R.razer_quantize_variant(Wv, block, sfmt, V))
                                       .cpu()[0]) / Wv.numel()
    blocks = {}
    for block in (16, 32, 64, 128):
        blocks[f"block{block}"] = {"nvfp4": mse(block, "nvfp4", []), "razer_pm5_pm8": mse(block, "weight", [5.0, -5.0, 8.0, -8.0])}
        blocks[f"block{block}"]["razer_over_nvfp4"] = blocks[f"block{block}"]["razer_pm5_pm8"] / blocks[f"block{block}"]["nvfp4"]
    allowed = [2.5, 3.5, 4.5, 5.0, 5.5, 6.5, 7.0, 7.5, 8.0, 8.5, 9.0, 9.5]
    pairs = sorted((mse(16, "weight", [a, -a, b, -b]), a, b) for i, a in enumerate(allowed) for b in allowed[i + 1:])
    # the pages' own kernel format: blocks of 128 with an FP16 scale word
    blocks["block128_f16_scale"] = {"razer_pm5_pm8": mse(128, "f16_scale", [5.0, -5.0, 8.0, -8.0]),
                                    "plain": mse(128, "f16_scale", [])}
    out["format_variants_4096x4096"] = {"block_size_study_mse": blocks,
                                        "special_value_search_top5": [{"pair": f"+-{a}/+-{b}", "mse": m} for m, a, b in pairs[:5]],
                                        "pairs_searched": len(pairs)}
    # W4A16 GEMV on variant weights (14336x4096, fp16): the pages' kernel
    # format (blocks of 128, FP16 scale words) and a per-model pair at block 16;
    # 8 weight copies rotate so every call streams its weights from HBM
    N, K = 14336, 4096
    gv = {}
    for name, block, sfmt, V in (("block128_f16_scale_pm5_pm8", 128, "f16_scale", [5.0, -5.0, 8.0, -8.0]),
                                 ("block16_e3m3_pm5_pm7", 16, "weight", [5.0, -5.0, 7.0, -7.0])):
        c0, s0 = workloads.random_packed_variant(N, K, block, sfmt, len(V), seed=407)
        c0, s0 = c0.to(dev), s0.to(dev)
        copies = [(c0.clone(), s0.clone()) for _ in range(8)]
        tsv = torch.tensor([1.0 if sfmt == "f16_scale" else 2.0 ** -9], dtype=torch.float32, device=dev)
        res = {}
        for B in (1, 16):
            xv = workloads.vectors(B, K, seed=408).to(dev)
            yv = torch.empty((B, N), dtype=torch.float16, device=dev)
            wsv = torch.empty(R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K), dtype=torch.uint8, device=dev)
            ms = time_graph(lambda: [R.razer_gemv_variant(xv, cc, ss, tsv, block, sfmt, V, torch.float16, out=yv, workspace=wsv)
                                     for cc, ss in copies], 8, stream)
            nbytes = N * K // 2 + s0.numel() + 2 * B * K + 2 * B * N
            res[f"B{B}"] = {"ms": ms, "GB/s": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm}
        gv[name] = res
    out["gemv_variant_14336x4096"] = gv
    # prefill GEMM on variant weights (M = 4096, 4096 x 4096): the pages'
    # format with fp16 activations and a per-model pair at block 16 with bf16
    # activations; the time includes the decode of the weight copy
    M, N, K = 4096, 4096, 4096
    gmv = {}
    for name, block, sfmt, V, xdt in (("block128_f16_scale_pm5_pm8_fp16", 128, "f16_scale", [5.0, -5.0, 8.0, -8.0], torch.float16),
                                      ("block16_e3m3_pm5_pm7_bf16", 16, "weight", [5.0, -5.0, 7.0, -7.0], torch.bfloat16)):
        c0, s0 = workloads.random_packed_variant(N, K, block, sfmt, len(V), seed=409)
        c0, s0 = c0.to(dev), s0.to(dev)
        tsv = torch.tensor([1.0 if sfmt == "f16_scale" else 2.0 ** -9], dtype=torch.float32, device=dev)
        Xv = workloads.vectors(M, K, seed=410, dtype=xdt).to(dev)
        Yv = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsv = torch.empty(R.razer_workspace_size(R.RAZER_OP_GEMM_VARIANT, M, N, K), dtype=torch.uint8, device=dev)
        ms = time_graph(lambda: R.razer_gemm_variant(Xv, c0, s0, tsv, block, sfmt, V, torch.bfloat16, out=Yv, workspace=wsv), 1, stream)
        tf = 2 * M * N * K / ms / 1e9
        gmv[name] = {"ms": ms, "TFLOP/s": tf, "frac": tf / bf16}
    out["gemm_variant_4096x4096x4096"] = gmv
    out["llama3_70b_sweep"] = run_70b_sweep(R, workloads, dev, stream, hbm, bf16)
    # the tiny case the oracle checks in full (launch-bound: time only)
    Wt = workloads.weight(256, 512, seed=0).to(dev)
    xt = workloads.vectors(1, 512, seed=1).to(dev)
    ct, st_, tt = R.razer_quantize_weights(Wt)
    yt = torch.empty((1, 256), dtype=torch.float16, device=dev)
    wst = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMV, 1, 256, 512)), dtype=torch.uint8, device=dev)
    out["tiny_256x512"] = {
        "quantize_ms": time_graph(lambda: R.razer_quantize_weights(Wt, codes=ct, scales=st_, ts=tt), 1, stream),
        "gemv_b1_ms": time_graph(lambda: R.razer_gemv(xt, ct, st_, tt, "weight", torch.float16, out=yt, workspace=wst), 1, stream),
        "note": "launch-bound; parity case, no roofline fraction"}
    # cuBLAS on the decoded weights, as an outside sanity reference only (a
    # library run on bf16 operands, not a target)
    Xc = workloads.vectors(4096, 4096, seed=400, dtype=torch.bfloat16).to(dev)
    cub = {}
    for N in (4096, 14336):
        c, s, t = R.razer_quantize_weights(workloads.weight(N, 4096, seed=401).to(dev))
        Wd = R.razer_dequant(c, s, t, "weight", torch.bfloat16)
        Yc = torch.empty((4096, N), dtype=torch.bfloat16, device=dev)
        ms = time_graph(lambda: torch.matmul(Xc, Wd.t(), out=Yc), 1, stream)
        cub[f"4096x{N}x4096"] = {"ms": ms, "TFLOP/s": 2 * 4096 * N * 4096 / ms / 1e9}
        del Wd, Yc
    out["cublas_bf16_on_decoded_weights"] = cub
    return out


def _rotation(nbytes, l2=126 * 2 ** 20):
    """Operand copies for a back-to-back sequence that cannot hit L2:
    ceil(2 L2 / bytes), at least 8 below 64 MB, at least 2."""
    n = -(-2 * l2 // max(nbytes, 1))
    if nbytes < 64 * 2 ** 20:
        n = max(n, 8)
    return max(n, 2)


def run_70b_sweep(R, workloads, dev, stream, hbm, bf16):
    """Llama-3-70B projections (N(0, 0.015^2), 0.1% x10): the W4A16 GEMV at
    B = 1, 8, 32 and the prefill GEMM at M = 512, 2048, 8192, in the RaZeR
    weight format and in plain NVFP4."""
    import torch

    shapes = [(8192, 8192), (28672, 8192), (8192, 28672)]
    res = {}
    for si, (N, K) in enumerate(shapes):
        W = workloads.weight(N, K, std=0.015, seed=500 + si).to(dev)
        for fmt in ("weight", "nvfp4"):
            c, s, t = R.razer_quantize_weights(W, fmt)
            packed = c.numel() + s.numel()
            copies = [(c, s)] + [(c.clone(), s.clone()) for _ in range(_rotation(packed) - 1)]
            key = f"{N}x{K}_{'razer' if fmt == 'weight' else 'nvfp4'}"
            row = {}
            for B in (1, 8, 32):
                x = workloads.vectors(B, K, seed=510 + B).to(dev)
                y = torch.empty((B, N), dtype=torch.float16, device=dev)
                ws = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMV, B, N, K)), dtype=torch.uint8, device=dev)
                ms = time_graph(lambda: [R.razer_gemv(x, cc, ss, t, fmt, torch.float16, out=y, workspace=ws) for cc, ss in copies],
                                len(copies), stream)
                nbytes = 0.5625 * N * K + 2 * B * K + 2 * B * N
                row[f"gemv_B{B}"] = {"ms": ms, "GB/s": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm,
                                     "frac_nominal_8TBs": nbytes / ms / 1e6 / 8000.0}
            del copies
            for M in (512, 2048, 8192):
                X = workloads.vectors(M, K, seed=520 + M, dtype=torch.bfloat16).to(dev)
                Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                ws = torch.empty(max(16, R.razer_workspace_size(R.RAZER_OP_GEMM, M, N, K)), dtype=torch.uint8, device=dev)
                ms = time_graph(lambda: R.razer_gemm(X, c, s, t, fmt, torch.bfloat16, out=Y, workspace=ws), 1, stream, reps=3)
                tf = 2 * M * N * K / ms / 1e9
                row[f"gemm_M{M}"] = {"ms": ms, "TFLOP/s": tf, "frac": tf / bf16, "frac_nominal_2250": tf / 2250.0}
                del X, Y, ws
            res[key] = row
        del W
    return res


def run_e2e(R, workloads, dev, stream, args, world, pg):
    """Same step through the public API with host (pinned) buffers: the fp16
    weights are copied in, quantized, the GEMVs run, the outputs come back."""
    import torch

    Wh = [workloads.weight(N, K, seed=100 + i).pin_memory() for i, (N, K) in enumerate(SHAPES)]
    Xh = {B: [workloads.vectors(B, K, seed=10 + B).pin_memory() for _, K in SHAPES] for B in BATCHES}
    Wd = [torch.empty_like(w, device=dev) for w in Wh]
    Xd = {B: [torch.empty_like(x, device=dev) for x in Xh[B]] for B in BATCHES}
    Yh = {B: [torch.empty((B, N), dtype=torch.float16).pin_memory() for N, _ in SHAPES] for B in BATCHES}
    h2d = sum(w.numel() * 2 for w in Wh) + sum(x.numel() * 2 for B in BATCHES for x in Xh[B])
    d2h = sum(y.numel() * 2 for B in BATCHES for y in Yh[B])

    def step():
        for i in range(len(SHAPES)):
            Wd[i].copy_(Wh[i], non_blocking=True)
        codes, scales, ts = R.razer_quantize_weights_batch(Wd, "weight")
        for i in range(len(SHAPES)):
            for B in BATCHES:
                Xd[B][i].copy_(Xh[B][i], non_blocking=True)
        for B in BATCHES:
            ys = R.razer_gemv_batch([(Xd[B][i], codes[i], scales[i], ts[i:i + 1]) for i in range(len(SHAPES))], "weight",
                                    torch.float16)
            for i, y in enumerate(ys):
                Yh[B][i].copy_(y, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if pg:
        ms = max_over_ranks(ms, pg, dev)
    return {"value": step_bytes() * steps * world / (ms / 1e3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps}


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the W4A16 group-quantized linear layer on B200.

One step = one decode pass over the LLaMA-2-7B decoder-layer linear set at
M = 1 (qkv 4096->12288, o_proj 4096->4096, gate_up 4096->22016,
down 11008->4096; group 128), i.e. four awq_linear calls, each a W4A16 GEMV
that streams its packed weights from HBM once. Inputs are seeded synthetic
(weights ~ N(0, 0.02), activations ~ N(0, 1)), quantized and packed on the
GPU by awq_pack before timing. Eight rotating copies of the packed weights
(8 x 105 MB, more than the 126 MB L2) make every step read HBM. The eight
steps that use them one after another are captured in one CUDA graph, the way
a decode step of a whole model (many decoder layers) is one graph: the graph
launch boundary (about 5 us, measured) is paid once per graph. Up to 64 timed
steps run as one graph of exactly that many steps (step i on copy i mod 8);
longer runs replay the eight-step graph.

Prints ONE JSON line (rank 0): the metric (GB/s of algorithmic bytes, whole
job), the roofline of the GEMV kernel, an end-to-end figure through the
public API with host buffers, the CPU oracle baseline, the clocks seen
during the timed region, and a secondary prefill GEMM figure (TFLOP/s).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  torchrun --nproc-per-node N bench.py --gpus N ...   (N independent replicas)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import awq_synth  # noqa: E402

WORKLOAD = "llama2_7b_decode"
M_DECODE = 1
ROTATIONS = 8
PREFILL = ("prefill", "llama3_gate_up", 2048)
METRIC = "W4A16 decode GEMV GB/s (% of HBM peak); prefill GEMM TFLOP/s (% tensor peak)"
GEMV_SRC = os.path.join(ROOT, "weight_only_bit_awq_b200", "csrc", "gemv.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_llama2_7b_decode_traffic.json")


def algo_bytes(M, K, N, group=128):
    """Bytes a W4A16 linear call must move: packed weight, scales, zeros, x, y."""
    return K * N // 2 + 2 * (K // group) * N + (K // group) * N // 2 + 2 * M * K + 2 * M * N


def reduce_max(v: float, world: int, device=None) -> float:
    """Max of a per-rank value over all ranks (the process group's backend)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate_gbs(bytes_per_step: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes every rank moved over the slowest rank's time."""
    return bytes_per_step * steps * world / (ms_max * 1e-3) / 1e9


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def traffic_per_launch():
    """Mean DRAM bytes per GEMV launch from the committed ncu capture, or None
    if the GEMV source changed since it was taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    h = hashlib.sha256(open(GEMV_SRC, "rb").read()).hexdigest()
    if d.get("gemv_src_sha256") != h:
        return None
    return d.get("dram_bytes_per_step", 0) / max(1, d.get("launches_per_step", 1))


# --------------------------------------------------------------------------
# reference arm: the CPU oracle as it stands, on host cores
# --------------------------------------------------------------------------

def host_cpu():
    """(CPU model name, number of cores this process may run on)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return model, cores


def run_oracle_rows(tasks, threads):
    """Run oracle.linear over (x, packed, N, K, n0, n1) row ranges on `threads`
    host threads (the oracle's C code is reentrant and ctypes releases the
    GIL while it runs); each range is split into `threads` contiguous pieces."""
    import concurrent.futures as cf

    import oracle
    pieces = []
    for x, hp, N, K, n0, n1 in tasks:
        step = max(1, -(-(n1 - n0) // threads))
        pieces += [(x, hp, N, K, a, min(n1, a + step)) for a in range(n0, n1, step)]
    if threads == 1:
        for x, hp, N, K, a, b in pieces:
            oracle.linear(x, *hp, N, K, rows=(a, b))
        return
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda t: oracle.linear(t[0], *t[1], t[2], t[3], rows=(t[4], t[5])), pieces))


def cpu_oracle_step(layers_packed, xs, frac, threads=1):
    """One step of the workload through the oracle, on the first `frac` of
    every layer's output channels, on `threads` host threads. Returns
    (algorithmic bytes covered, seconds)."""
    tasks, tot = [], 0.0
    for (L, hp), x in zip(layers_packed, xs):
        n1 = max(16, int(L.N * frac) // 16 * 16)
        tasks.append((x, hp, L.N, L.K, 0, n1))
        tot += algo_bytes(M_DECODE, L.K, L.N) * n1 / L.N
    t0 = time.perf_counter()
    run_oracle_rows(tasks, threads)
    return tot, time.perf_counter() - t0


def host_workload(rows=None, seed=0):
    """Oracle-packed weights of the workload's layers (all rows, or the first `rows`)."""
    import oracle
    wl = awq_synth.WORKLOADS[WORKLOAD]
    out, xs = [], []
    for L in wl.layers:
        W = awq_synth.layer_weight(seed, wl, L, rows=None if rows is None else slice(0, rows))
        n = W.shape[0]
        Ls = awq_synth.Layer(L.name, L.K, n)
        out.append((Ls, oracle.quantize_pack(W), L))
        xs.append(awq_synth.layer_input(seed, wl, L, M_DECODE))
    return wl, out, xs


def run_reference(args):
    """The oracle, as it stands, timed on the host cores. Each step is a
    bounded sample of the workload: `rows_per_step` output channels taken
    round-robin from the first 64 rows of the four layers, sized so that
    warm-up plus timed steps take about --ref-budget seconds."""
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    model, cores = host_cpu()
    pool_rows = max(64, 16 * cores)  # output channels of each layer packed for the sample
    wl, pool, xs = host_workload(rows=pool_rows)
    t0 = time.perf_counter()
    for li in range(len(pool)):
        Ls, hp, L = pool[li]
        oracle.linear(xs[li], *hp, Ls.N, Ls.K, rows=(0, 1))
    t_row = (time.perf_counter() - t0) / len(pool)
    # rows of each of the four layers per step (cycling over the packed rows),
    # split over all host cores; ~ref_budget seconds in all
    per_layer = int(max(1, min(pool_rows, args.ref_budget * cores / (args.steps + args.warmup) / t_row / len(pool))))
    cursor = 0

    def one_step():
        nonlocal cursor
        tasks, b = [], 0.0
        r0 = cursor % pool_rows
        r1 = min(pool_rows, r0 + per_layer)
        cursor = r1 % pool_rows
        for li in range(len(pool)):
            Ls, hp, L = pool[li]
            tasks.append((xs[li], hp, Ls.N, Ls.K, r0, r1))
            b += algo_bytes(M_DECODE, L.K, L.N) * (r1 - r0) / L.N
        t = time.perf_counter()
        run_oracle_rows(tasks, cores)
        return b, time.perf_counter() - t

    for _ in range(args.warmup):
        one_step()
    tot_b, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        b, t = one_step()
        tot_b += b
        tot_t += t
    gbs = tot_b / tot_t / 1e9
    sample = (f"up to {per_layer} output channel(s) of each of the four layers per step, cycling over their "
              f"first {pool_rows} rows, split over {cores} host threads (fp64 C oracle: unpack, dequant, dot products; "
              f"CPU: {model})")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_DECODE, "group": 128,
                   "layers": [[L.name, L.K, L.N] for L in wl.layers]},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "cpu_model": model,
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# every workload configuration (GPU, rank 0 at N = 1)
# --------------------------------------------------------------------------

L2_BYTES = 126e6


def rotations_for(weight_bytes: float, cap: int) -> int:
    """Rotating weight copies whose total is at least 3x the L2 (every step reads HBM)."""
    return int(max(2, min(cap, -(-3 * L2_BYTES // weight_bytes))))


def timed_region(run, stream, min_seconds=0.25):
    """Replays `run` (one call = one timed unit) until about `min_seconds` of
    device time, after 3 untimed calls; CUDA events on `stream`, nvidia-smi
    clocks sampled during the region. Returns (ms per call, calls, clocks)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(3):
            run()
        e1.record(stream)
    torch.cuda.synchronize()
    calls = int(max(10, min(20000, min_seconds * 1e3 / max(e0.elapsed_time(e1) / 3, 1e-4))))
    with ClockSampler(torch.cuda.current_device()) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(calls):
                run()
            e1.record(stream)
        torch.cuda.synchronize()
    return e0.elapsed_time(e1) / calls, calls, clk.summary()


def decode_sweep(awq, dev, stream, hbm):
    """Every decode configuration: each workload's layer set as one step (one
    awq_linear per layer), R consecutive steps over R rotating packed-weight
    copies captured in one CUDA graph."""
    import torch
    out = []
    for wl_name in ("single_4096", "llama2_7b_decode", "llama3_8b_decode", "llama2_70b_decode"):
        wl = awq_synth.WORKLOADS[wl_name]
        base = []
        for L in wl.layers:
            W = torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
            base.append(awq.awq_pack(W, awq.new_workspace(0, L.K, L.N, dev)))
            del W
        wbytes = sum(algo_bytes(0, L.K, L.N) for L in wl.layers)
        R = rotations_for(wbytes, 32)
        packed = [base] + [[tuple(t.clone() for t in p) for p in base] for _ in range(R - 1)]
        for M in wl.batches:
            xs = [torch.from_numpy(awq_synth.layer_input(0, wl, L, M).view(np.uint16)).view(torch.float16).to(dev)
                  for L in wl.layers]
            ys = [torch.empty((M, L.N), dtype=torch.float16, device=dev) for L in wl.layers]
            ws = torch.zeros(max(awq.awq_workspace_bytes(M, L.K, L.N) for L in wl.layers), dtype=torch.uint8,
                             device=dev)

            def steps():
                for r in range(R):
                    for L, x, y, p in zip(wl.layers, xs, ys, packed[r]):
                        awq.awq_linear(x, *p, L.N, ws, y=y)

            with torch.cuda.stream(stream):
                steps()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                steps()
            ms, calls, clocks = timed_region(g.replay, stream)
            st = awq.awq_get_status(ws)
            if st != awq.AWQ_OK:
                raise RuntimeError(awq.awq_status_string(st))
            step_bytes = sum(algo_bytes(M, L.K, L.N) for L in wl.layers)
            us = ms * 1e3 / R
            gbs = step_bytes / (us * 1e-6) / 1e9
            out.append({"workload": wl_name, "M": M, "kind": "decode", "layers": [[L.name, L.K, L.N] for L in wl.layers],
                        "us_per_step": us, "value": gbs, "unit": "GB/s", "frac": gbs / hbm,
                        "launches_per_step": sum(awq.awq_linear_launches(M, L.K, L.N) for L in wl.layers),
                        "rotations": R, "steps_timed": calls * R, "clocks": clocks})
            del g, xs, ys, ws
        del packed, base
        torch.cuda.empty_cache()
    return out


def prefill_sweep(awq, dev, stream, tc_burst):
    """Every prefill configuration, W4A16 (awq_linear: the tcgen05 GEMM) and
    W4A8-FP8 (per-token E4M3 quantization of x + the kind::f8f6f4 GEMM), with
    rotating packed-weight copies; eager launches (each call runs 0.05-12 ms)."""
    import torch
    out = []
    wl = awq_synth.WORKLOADS["prefill"]
    for L in wl.layers:
        W = torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
        base = awq.awq_pack(W, awq.new_workspace(0, L.K, L.N, dev))
        del W
        R = rotations_for(algo_bytes(0, L.K, L.N), 16)
        packed = [base] + [tuple(t.clone() for t in base) for _ in range(R - 1)]
        e8 = awq.awq_fp8_row_exponents(base[1], L.K, L.N)
        for M in wl.batches:
            x = torch.from_numpy(awq_synth.layer_input(0, wl, L, M).view(np.uint16)).view(torch.float16).to(dev)
            y = torch.empty((M, L.N), dtype=torch.float16, device=dev)
            ws = awq.new_workspace(M, L.K, L.N, dev)
            x8 = torch.empty((M, L.K), dtype=torch.uint8, device=dev)
            sx = torch.empty(M, dtype=torch.float32, device=dev)
            flops = 2.0 * M * L.N * L.K
            cur = [0]

            def w4a16():
                awq.awq_linear(x, *packed[cur[0]], L.N, ws, y=y)
                cur[0] = (cur[0] + 1) % R

            def w4a8():
                awq.lib.awq_fp8_quantize_x(x.data_ptr(), M, L.K, x8.data_ptr(), sx.data_ptr(), stream.cuda_stream)
                awq.awq_w4a8_gemm(x8, sx, *packed[cur[0]], e8, L.N, ws, y=y)
                cur[0] = (cur[0] + 1) % R

            for name, fn, peak in (("w4a16", w4a16, tc_burst), ("w4a8_fp8", w4a8, 2 * tc_burst)):
                ms, calls, clocks = timed_region(fn, stream, min_seconds=0.2)
                st = awq.awq_get_status(ws)
                if st != awq.AWQ_OK:
                    raise RuntimeError(awq.awq_status_string(st))
                tf = flops / (ms * 1e-3) / 1e12
                out.append({"workload": f"prefill/{L.name}", "K": L.K, "N": L.N, "M": M, "kind": name,
                            "ms": ms, "value": tf, "unit": "TFLOP/s", "frac": tf / peak,
                            "launches": awq.awq_linear_launches(M, L.K, L.N) if name == "w4a16" else None,
                            "rotations": R, "calls_timed": calls, "clocks": clocks})
            del x, y, ws, x8, sx
        del packed, base, e8
        torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import weight_only_bit_awq_b200 as awq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    hbm, tc_burst, tc_sus, peak_kind = peaks()
    wl = awq_synth.WORKLOADS[WORKLOAD]
    layers = wl.layers
    ws = awq.new_workspace(M_DECODE, max(L.K for L in layers), max(L.N for L in layers), dev)
    ws_bytes = max(awq.awq_workspace_bytes(M_DECODE, L.K, L.N) for L in layers)
    if ws.numel() < ws_bytes:
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)

    # inputs: seeded weights, packed on this GPU by awq_pack (K1), R copies;
    # every layer's x (and y) is a view into one contiguous buffer, so the end
    # to end step moves all activations with one copy each way
    packed = [[] for _ in range(ROTATIONS)]
    x_all = torch.empty(sum(M_DECODE * L.K for L in layers), dtype=torch.float16, device=dev)
    y_all = torch.empty(sum(M_DECODE * L.N for L in layers), dtype=torch.float16, device=dev)
    xs, ys = [], []
    xo = yo = 0
    for L in layers:
        W = torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
        qw, sc, ze = awq.awq_pack(W, ws)
        st = awq.awq_get_status(ws)
        if st != awq.AWQ_OK:
            raise RuntimeError(awq.awq_status_string(st))
        del W
        for r in range(ROTATIONS):
            packed[r].append((qw.clone(), sc.clone(), ze.clone()) if r else (qw, sc, ze))
        x = x_all[xo:xo + M_DECODE * L.K].view(M_DECODE, L.K)
        x.copy_(torch.from_numpy(awq_synth.layer_input(0, wl, L, M_DECODE).view(np.uint16)).view(torch.float16))
        xs.append(x)
        ys.append(y_all[yo:yo + M_DECODE * L.N].view(M_DECODE, L.N))
        xo += M_DECODE * L.K
        yo += M_DECODE * L.N
    step_bytes = sum(algo_bytes(M_DECODE, L.K, L.N) for L in layers)

    def step(r):
        for L, x, y, (qw, sc, ze) in zip(layers, xs, ys, packed[r]):
            awq.awq_linear(x, qw, sc, ze, L.N, ws, y=y)

    # CUDA graphs: graphs[j] holds j consecutive steps (step i on weight copy
    # i % ROTATIONS, 4 layers each). Up to WHOLE_GRAPH_STEPS steps run as one
    # graph of exactly k steps; more replay graphs[ROTATIONS] k // ROTATIONS
    # times, then graphs[k % ROTATIONS] once
    WHOLE_GRAPH_STEPS = 64
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        for r in range(ROTATIONS):   # warm the launch paths before capture
            step(r)
    torch.cuda.synchronize()

    def plan(k):
        return [k] if k <= WHOLE_GRAPH_STEPS else [ROTATIONS] * (k // ROTATIONS) + (
            [k % ROTATIONS] if k % ROTATIONS else [])

    graphs = {}
    for j in set(plan(args.steps) + plan(args.warmup)) - {0}:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(j):
                step(i % ROTATIONS)
        graphs[j] = g
    torch.cuda.synchronize()

    def run_steps(k):  # exactly k steps
        for j in plan(k):
            if j:
                graphs[j].replay()

    # every graph the warm-up and the timed region use is replayed once first,
    # so neither region holds a graph's first launch
    with torch.cuda.stream(stream):
        for g in graphs.values():
            g.replay()
        run_steps(args.warmup)
    barrier()
    st = awq.awq_get_status(ws)
    if st != awq.AWQ_OK:
        raise RuntimeError(awq.awq_status_string(st))

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1))
    clocks = clk.summary()
    st = awq.awq_get_status(ws)
    if st != awq.AWQ_OK:
        raise RuntimeError(awq.awq_status_string(st))
    value = job_rate_gbs(step_bytes, args.steps, world, ms)
    per_gpu_gbs = job_rate_gbs(step_bytes, args.steps, 1, ms)

    # ---- end to end through the public API with pinned host buffers ----
    # one step: one H2D copy of every layer's x from pinned memory, the four
    # awq_linear calls, one D2H copy of every y into pinned memory
    xh = torch.empty_like(x_all, device="cpu").pin_memory().copy_(x_all.cpu())
    yh = torch.empty_like(y_all, device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 2000))

    def e2e_step(r):
        x_all.copy_(xh, non_blocking=True)
        for L, x, y, (qw, sc, ze) in zip(layers, xs, ys, packed[r]):
            awq.awq_linear(x, qw, sc, ze, L.N, ws, y=y)
        yh.copy_(y_all, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            e2e_step(i % ROTATIONS)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i % ROTATIONS)
        e1.record(stream)
    barrier()
    eager_ms = max_over_ranks(e0.elapsed_time(e1))
    # the same steps captured as a decode runtime would run them: a CUDA graph
    # of ROTATIONS consecutive steps (each with its own H2D and D2H copies),
    # captured from the same public-API calls and replayed
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        for r in range(ROTATIONS):
            e2e_step(r)
    replays = max(1, e2e_steps // ROTATIONS)
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup // ROTATIONS + 1)):
            e2e_graph.replay()
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g0.record(stream)
        for _ in range(replays):
            e2e_graph.replay()
        g1.record(stream)
    barrier()
    graph_ms = max_over_ranks(g0.elapsed_time(g1))
    graph_steps = replays * ROTATIONS
    del e2e_graph
    e2e = {"value": job_rate_gbs(step_bytes, graph_steps, world, graph_ms), "unit": "GB/s",
           "h2d_bytes_per_step": x_all.numel() * 2, "d2h_bytes_per_step": y_all.numel() * 2,
           "steps": graph_steps, "ms_per_step": graph_ms / graph_steps,
           "how": "public Python API calls captured in a CUDA graph of 8 consecutive steps, replayed: every step "
                  "one H2D copy of all x from pinned memory, four awq_linear calls, one D2H copy of all y to "
                  "pinned memory",
           "eager": {"value": job_rate_gbs(step_bytes, e2e_steps, world, eager_ms), "steps": e2e_steps,
                     "ms_per_step": eager_ms / e2e_steps,
                     "how": "the same calls launched from Python each step"}}

    # ---- every workload configuration (rank 0 at N = 1) ----
    sweep_decode = sweep_prefill = None
    prefill = None
    if world == 1 and not args.no_sweep:
        sweep_decode = decode_sweep(awq, dev, stream, hbm)
        if not args.no_prefill:
            sweep_prefill = prefill_sweep(awq, dev, stream, tc_burst)
            pe = {(e["workload"], e["M"], e["kind"]): e for e in sweep_prefill}
            a16, a8 = pe[(f"prefill/{PREFILL[1]}", PREFILL[2], "w4a16")], pe[(f"prefill/{PREFILL[1]}", PREFILL[2], "w4a8_fp8")]
            prefill = {"workload": f"{PREFILL[1]} K={a16['K']} N={a16['N']} M={PREFILL[2]}", "ms": a16["ms"],
                       "tflops_per_gpu": a16["value"], "peak_tflops": tc_burst, "frac": a16["frac"],
                       "peak_kind": f"{peak_kind} bf16 burst", "clocks": a16["clocks"],
                       "w4a8_fp8": {"ms": a8["ms"], "tflops_per_gpu": a8["value"], "peak_tflops": 2 * tc_burst,
                                    "frac": a8["frac"],
                                    "peak_kind": f"{peak_kind} bf16 burst x 2 (nominal dense fp8 : bf16 = 4.5 : 2.25)",
                                    "includes": "per-token E4M3 quantization of x + tcgen05 kind::f8f6f4 GEMM"}}

    # ---- comparator: the same layers as dense fp16 weights through cuBLAS ----
    # (torch.matmul; a library call, timed the same way: CUDA graphs over
    # rotating weight copies larger than L2). It gives the INT4 vs FP16
    # speedup the TinyChat README reports per token.
    fp16 = None
    if not args.no_fp16:
        rot16 = 2
        w16 = [[torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
                for L in layers] for _ in range(rot16)]

        def step16(r):
            for L, x, y, w in zip(layers, xs, ys, w16[r]):
                torch.matmul(x, w.t(), out=y)

        with torch.cuda.stream(stream):
            for r in range(rot16):
                step16(r)
        torch.cuda.synchronize()
        g16 = []
        for r in range(rot16):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step16(r)
            g16.append(g)
        steps16 = max(3, min(args.steps, 2000))
        with torch.cuda.stream(stream):
            for g in g16:
                g.replay()
            for i in range(args.warmup):
                g16[i % rot16].replay()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            f0.record(stream)
            for i in range(steps16):
                g16[i % rot16].replay()
            f1.record(stream)
        barrier()
        ms16 = max_over_ranks(f0.elapsed_time(f1)) / steps16
        fp16 = {"library": "cuBLAS through torch.matmul, dense fp16 weights", "decode_ms_per_step": ms16,
                "decode_speedup_int4_vs_fp16": ms16 / (ms / args.steps)}
        del g16, w16
        if prefill is not None:
            pwl = awq_synth.WORKLOADS[PREFILL[0]]
            PL = pwl.layer(PREFILL[1])
            Mp = PREFILL[2]
            W = torch.from_numpy(awq_synth.layer_weight(0, pwl, PL).view(np.uint16)).view(torch.float16).to(dev)
            Ws = [W] + [W.clone() for _ in range(rotations_for(2.0 * PL.K * PL.N, 8) - 1)]
            xp = torch.from_numpy(awq_synth.layer_input(0, pwl, PL, Mp).view(np.uint16)).view(torch.float16).to(dev)
            yp = torch.empty((Mp, PL.N), dtype=torch.float16, device=dev)
            cur = [0]

            def mm16():
                torch.matmul(xp, Ws[cur[0]].t(), out=yp)
                cur[0] = (cur[0] + 1) % len(Ws)

            pms16, _, _ = timed_region(mm16, stream, min_seconds=0.2)
            fp16.update({"prefill_ms": pms16, "prefill_tflops": 2.0 * Mp * PL.N * PL.K / (pms16 * 1e-3) / 1e12,
                         "prefill_speedup_int4_vs_fp16": pms16 / prefill["ms"],
                         "prefill_speedup_w4a8_vs_fp16": pms16 / prefill["w4a8_fp8"]["ms"]})
            del W, Ws, xp, yp
        torch.cuda.empty_cache()

    # ---- CPU oracle baseline on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, hl, hx = host_workload()
        model, cores = host_cpu()
        lp = [(L, hp) for L, hp, _ in hl]
        b1, t1 = cpu_oracle_step(lp, hx, args.cpu_frac / 8, threads=1)
        b, t = cpu_oracle_step(lp, hx, args.cpu_frac, threads=cores)
        cpu = {"value": b / t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle", "cpu_model": model,
               "single_thread_value": b1 / t1 / 1e9,
               "sample": f"one step on the first {args.cpu_frac:.3f} of each layer's output channels, rows split "
                         f"over {cores} threads ({t:.1f} s); single thread: the first {args.cpu_frac / 8:.3f} of "
                         f"the rows ({t1:.1f} s); fp64 C oracle"}

    traffic = traffic_per_launch()
    launches = sum(awq.awq_linear_launches(M_DECODE, L.K, L.N) for L in layers) * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_DECODE, "group": 128,
                   "layers": [[L.name, L.K, L.N] for L in layers],
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"{ROTATIONS} rotating packed-weight copies ({ROTATIONS * step_bytes / 1e6:.0f} MB > 126 MB L2)",
                   "timing": (f"one CUDA graph of all {args.steps} steps (step i on weight copy i mod "
                              f"{ROTATIONS})" if args.steps <= WHOLE_GRAPH_STEPS else
                              f"CUDA graphs of {ROTATIONS} consecutive steps (one per weight copy) and one graph "
                              f"of the remaining steps") + ", each replayed once before warm-up; CUDA events on "
                                                          "the replay stream"},
        "roofline": {"bound": "hbm", "achieved": per_gpu_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": per_gpu_gbs / hbm, "traffic": traffic,
                     "kernel": "gemv_kernel (awq_w4a16_gemv via awq_linear)",
                     "peak_kind": f"{peak_kind} HBM copy"},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "prefill_gemm": prefill,
        "fp16_comparator": fp16,
        "configs": (sweep_decode or []) + (sweep_prefill or []) if sweep_decode is not None else None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    graphs.clear()
    if world > 1:
        dist.destroy_process_group()
    return 0


SINGLE = {
    # one kernel on a layer larger than the 126 MB L2, for profiler captures
    "gemv": ("llama2_70b_decode", "gate_up", 1),     # 235 MB packed weight, M = 1
    "gemv_7b_qkv": ("llama2_7b_decode", "qkv", 1),    # 25 MB: the decode set's second-largest layer
    "gemv_7b_o": ("llama2_7b_decode", "o_proj", 1),   # 8 MB: the smallest, latency-bound
    "gemv_m8": ("llama3_8b_decode", "gate_up", 8),    # 61 MB, the lo/hi fp16 path at M = 8
    "gemv_m16": ("llama3_8b_decode", "gate_up", 16),  # two token tiles
    "gemm": ("prefill", "llama3_gate_up", 2048),     # 58 MB weight + 16 MB x + 117 MB y
    "gemm_m512": ("prefill", "llama3_gate_up", 512),  # stream-K schedule: the GEMM and its fixup kernel
    "gemm_fp8": ("prefill", "llama3_gate_up", 2048),  # the same layer through the W4A8-FP8 GEMM
}


def run_single(args):
    """Launch one kernel `--reps` times on one full-size layer (no graphs),
    then check the status word. Used as the target of ncu captures."""
    import torch

    import weight_only_bit_awq_b200 as awq
    wl_name, layer_name, M = SINGLE[args.single]
    wl = awq_synth.WORKLOADS[wl_name]
    L = wl.layer(layer_name)
    dev = torch.device("cuda", 0)
    W = torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
    ws = awq.new_workspace(M, L.K, L.N, dev)
    packed = awq.awq_pack(W, ws)
    del W
    x = torch.from_numpy(awq_synth.layer_input(0, wl, L, M).view(np.uint16)).view(torch.float16).to(dev)
    y = torch.empty((M, L.N), dtype=torch.float16, device=dev)
    fn = awq.awq_w4a16_gemv if args.single.startswith("gemv") else awq.awq_w4a16_gemm
    if args.single == "gemm_fp8":
        e8 = awq.awq_fp8_row_exponents(packed[1], L.K, L.N)
        x8, sx = awq.awq_fp8_quantize_x(x)

        def fn(x_, qw, sc, ze, N_, ws_, y=None):  # the GEMM alone: x was quantized above
            return awq.awq_w4a8_gemm(x8, sx, qw, sc, ze, e8, N_, ws_, y=y)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.reps + 1)]
    ev[0].record()
    for i in range(args.reps):
        fn(x, *packed, L.N, ws, y=y)
        ev[i + 1].record()
    torch.cuda.synchronize()
    st = awq.awq_get_status(ws)
    if st != awq.AWQ_OK:
        raise RuntimeError(awq.awq_status_string(st))
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.reps)]
    work = (algo_bytes(M, L.K, L.N) / 1e9, "GB") if args.single.startswith("gemv") else (2.0 * M * L.N * L.K / 1e12, "TFLOP")
    print(json.dumps({"single": args.single, "workload": f"{wl_name}/{layer_name} K={L.K} N={L.N} M={M}",
                      "ms": times, "rate_per_s": [work[0] / (t * 1e-3) for t in times], "unit": work[1] + "/s"}))
    return 0


def run_sharded(args):
    """N-sharded strong scaling of the decode layer set: every rank holds the
    packed weights of its slice of each layer's output channels (whole groups
    of 128), runs its GEMVs and all-gathers y (NCCL), so each step produces
    every layer's full output on every rank. No CUDA graphs (the all-gather
    is a collective), so a step also pays the host's launch time."""
    import datetime

    import torch
    import torch.distributed as dist

    import weight_only_bit_awq_b200 as awq
    from weight_only_bit_awq_b200.sharding import ShardedLinear

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    wl = awq_synth.WORKLOADS[WORKLOAD]
    shards, xs = [], []
    for L in wl.layers:
        W = torch.from_numpy(awq_synth.layer_weight(0, wl, L).view(np.uint16)).view(torch.float16).to(dev)
        shards.append(ShardedLinear(W, world, rank))
        del W
        xs.append(torch.from_numpy(awq_synth.layer_input(0, wl, L, M_DECODE).view(np.uint16))
                  .view(torch.float16).to(dev))
    step_bytes = sum(algo_bytes(M_DECODE, L.K, L.N) for L in wl.layers)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def step():
        return [sl.forward_full(x) for sl, x in zip(shards, xs)]

    for _ in range(args.warmup):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        ys = step()
    e1.record()
    barrier()
    ms = reduce_max(e0.elapsed_time(e1), world, dev)
    assert all(y.shape == (M_DECODE, L.N) for y, L in zip(ys, wl.layers))
    st = [awq.awq_get_status(sl.ws) for sl in shards]
    if any(st):
        raise RuntimeError(awq.awq_status_string(max(st)))
    launches = sum(awq.awq_linear_launches(M_DECODE, L.K, sl.n_local) for sl, L in zip(shards, wl.layers))
    line = {
        "metric": METRIC, "value": step_bytes * args.steps / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_DECODE, "group": 128,
                   "layers": [[L.name, L.K, L.N] for L in wl.layers],
                   "parallelism": f"N-sharded x{world} (whole groups of 128 channels) + all-gather of y",
                   "timing": "eager launches, CUDA events, max over ranks"},
        "gpu_launches": launches * args.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-configuration sweep (decode and prefill)")
    ap.add_argument("--no-fp16", action="store_true", help="skip the cuBLAS fp16 comparator")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-frac", type=float, default=1.0, help="share of rows in the CPU-baseline sample")
    ap.add_argument("--ref-budget", type=float, default=60.0, help="seconds of oracle work in the reference arm")
    ap.add_argument("--single", choices=sorted(SINGLE), help="launch one kernel on one layer (profiling target)")
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--shard", action="store_true",
                    help="N-shard the decode layers across the ranks (strong scaling) instead of replicas")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.single:
        return run_single(args)
    if args.shard:
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

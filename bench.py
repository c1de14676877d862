#!/usr/bin/env python3
"""Benchmark of the MBOK linear layer on B200.

Headline: packed-weight HBM GB/s (and us/layer) of the K=3 Boolean decode
GEMV on the LLaMA-7B q_proj shape (M = N = 4096, group 128, batch 1, bf16 x).
One step is one decode pass over L distinct weight copies of that shape
(L = 48 by default: 340 MB of packed weights, well above the 126 MB L2, so
every launch reads its weights from HBM).  The step is captured once in a
CUDA graph and replayed; time is taken with CUDA events on the launching
stream, max over ranks when several GPUs run replicas.

Also reported on the same JSON line: the roofline of the GEMV kernel, an
end-to-end number through the C ABI with host buffers, the CPU oracle
baseline, SM clocks sampled during the timed region, and secondary rows
(prefill GEMM, small batch, the LLaMA-13B layer sweep, residual
binarisation, packing).

`--impl reference` times the CPU oracle (the correctness reference of this
repository) on a bounded sample of the same workload, on the host cores.
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

import numpy as np  # noqa: E402

METRIC = "packed-weight HBM GB/s (% of peak) and us/layer, K-kernel Boolean GEMV/GEMM"
UNIT = "GB/s"


def args_parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["mbok", "reference"], default="mbok")
    p.add_argument("--layers", type=int, default=48, help="distinct weight copies per step")
    p.add_argument("--no-extras", action="store_true", help="skip the secondary rows")
    p.add_argument("--rows", default="gemm,small_batch,sweep,svid,residual,pack",
                   help="comma-separated secondary rows to run")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--profile-gemv", default=None, metavar="K,M,N,BATCH,KERNEL",
                   help="profiling helper: run four launches of one GEMV (KERNEL as mbok_gemv_set_kernel: "
                        "0 auto, 1 lookup, 2 tensor, 3 slab lookup, 4 whole-row lookup) with L2 flushed "
                        "between them, print nothing else, and exit")
    p.add_argument("--phase-profile", default=None, metavar="K,M,N,LAYERS[,svid]",
                   help="per-phase split of the decode GEMV chain (profiling build with phase stamps)")
    p.add_argument("--profile-svid", default=None, metavar="K,M,N",
                   help="profiling helper: run four launches of the rank-1-form GEMV (batch 1) with L2 flushed "
                        "between them, print nothing else, and exit")
    p.add_argument("--profile-convert", default=None, metavar="K,M,N",
                   help="profiling helper: run two launches each of residual binarisation (fp32 W) and bit "
                        "packing (int8 signs), then one scale refit and one successive-SVID conversion, "
                        "with L2 flushed before each, print nothing else, and exit")
    p.add_argument("--profile-gemm", default=None, metavar="K,M,N,T,PRECISION",
                   help="profiling helper: run three launches of one prefill GEMM (PRECISION as "
                        "mbok_gemm_ex: 0 auto, 1 bf16, 2 split), print nothing else, and exit")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(names) -> str:
    """sha256 (16 hex digits) of the listed csrc files, concatenated in order."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "boolean_weight_matmul_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(key: str):
    """Per-launch DRAM bytes from the committed ncu summary, or None when any
    source file of the kernel changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("source_sha256_16") != kernel_source_hash(e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() in ("active", "1"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def cpu_oracle_rate(seconds: float = 10.0):
    """The oracle as it stands: packed-weight GB/s of oracle.linear on sampled
    rows of one q_proj layer, repeated for about `seconds`."""
    from oracle import mbok_oracle as O
    from boolean_weight_matmul_b200 import workloads as wl
    K, M, N = 3, 4096, 4096
    words = wl.random_words(O.packed_bytes(K, M, N) // 4, wl.seed_of(2, 0, 0))
    a = wl.alpha_decaying(K, M, N, wl.seed_of(2, 0, 1))
    x = wl.x_normal(1, N, wl.seed_of(2, 0, 2))
    rows_per_call = 256
    bytes_per_row = K * N / 8 + 2 * K * N / 128
    t0 = time.perf_counter()
    n_rows = 0
    calls = 0
    rng = np.random.default_rng(0)
    while time.perf_counter() - t0 < seconds:
        rows = np.sort(rng.choice(M, rows_per_call, replace=False))
        O.linear(words, a, K, M, N, x, "bf16", rows=rows)
        n_rows += rows_per_call
        calls += 1
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = 1
    return {"value": n_rows * bytes_per_row / dt / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{calls} calls of oracle.linear on {rows_per_call} random rows of one K=3 "
                      f"4096x4096 layer ({n_rows} rows, {dt:.1f} s); numpy fp64"}


def replica_max_ms(ms: float, dist=None, device=None) -> float:
    """Max over ranks of a per-rank device time (replicas run the same step)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(max(0, a.warmup)):
        cpu_oracle_rate(0.5)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(a.steps):
        last = cpu_oracle_rate(1.0)
        vals.append(last["value"])
    dt = time.perf_counter() - t0
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * dt / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "llama7b_q_proj_k3_4096x4096_gemv_b1", "K": 3, "M": 4096,
                       "N": 4096, "group": 128, "batch": 1,
                       "sample": "each step: 1 s of oracle.linear on 256 random rows"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def build_layers(torch, mb, wl, K, M, N, L, dev, seed0):
    """L distinct packed weights (random words = Bernoulli(0.5) bits) with
    decaying scales, plus L activation vectors."""
    g = torch.Generator(device=dev)
    g.manual_seed(seed0)
    nb = mb.packed_bytes(K, M, N)
    packed = [torch.randint(-2 ** 31, 2 ** 31 - 1, (nb // 4,), dtype=torch.int32, device=dev, generator=g)
              for _ in range(L)]
    alphas = []
    for l in range(L):
        a = wl.alpha_decaying(K, M, N, seed0 + 10 * l + 1)
        ad = torch.from_numpy(a.view(np.int16)).to(dev).view(torch.float16)
        out = mb.empty_alpha(K, M, N, dev)
        mb.pack_alpha(ad, K, M, N, out)
        alphas.append(out)
    xs = [torch.from_numpy(wl.x_normal(1, N, seed0 + 10 * l + 2).view(np.int16)).to(dev).view(torch.bfloat16)
          for l in range(L)]
    return packed, alphas, xs


def e2e_copy_cuts(L: int):
    """Layer boundaries of the pipelined end-to-end step's host copies: inputs
    [0, 4) then [4, L); outputs [0, L - 4) then [L - 4, L).  Copy i covers
    layers cuts[i] .. cuts[i+1] - 1."""
    return sorted({0, min(4, L), L}), sorted({0, max(L - 4, 0), L})


def time_graph(torch, fn, steps, warmup, stream):
    """Capture fn() once, replay warmup + steps times; returns ms per replay."""
    with torch.cuda.stream(stream):
        fn()   # eager warm-up (sets kernel attributes outside capture)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        fn()
    # replay() launches on the current stream: make it the captured stream so
    # the events bracket the replays.
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / steps, graph


def run_gpu(a):
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    from boolean_weight_matmul_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if rank == 0:
        mbuild.build()
    if world > 1:
        dist.barrier()
    peaks, peak_src = measured_peaks()

    # CPU baseline first (rank 0, N=1 only), before any GPU work is timed.
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_oracle_rate(10.0)

    K, M, N, L = 3, 4096, 4096, a.layers
    bytes_per_layer = mb.packed_bytes(K, M, N) + 2 * mb.alpha_elems(K, M, N)
    packed, alphas, xs = build_layers(torch, mb, wl, K, M, N, L, dev, 1000 * 2 + 7919 * rank)
    ws = mb.zeros_workspace(K, M, N, 1, dev)
    ys = [torch.empty(1, M, dtype=torch.float32, device=dev) for _ in range(L)]
    stream = torch.cuda.Stream(device=dev)

    def step():
        for l in range(L):
            mb.gemv(packed[l], alphas[l], K, M, N, 128, xs[l], mb.BF16, 1, ys[l], ws, stream=stream)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms, graph = time_graph(torch, step, a.steps, a.warmup, stream)
    clocks = clk.summary()
    if world > 1:
        ms = replica_max_ms(ms, dist, dev)
        dist.barrier()
    value = replica_rate(L * bytes_per_layer, ms, world) / 1e9
    # the lookup GEMV is one launch, plus one that adds the slabs' partials
    # when N spans more than one 512-column slab
    launches_per_gemv = 2 if N > 512 else 1
    us_per_layer = 1e3 * ms / L
    achieved = bytes_per_layer / (us_per_layer * 1e-6) / 1e9
    traffic = ncu_traffic("gemv_lut8_q_proj_k3_4096x4096")

    # End to end through the C ABI with host buffers: per step, copy the L
    # activation vectors host->device, run the L GEMVs, copy the L outputs back.
    x_host = torch.stack([x.view(torch.int16).cpu() for x in xs]).pin_memory()
    x_dev = torch.empty_like(x_host, device=dev)
    y_host = torch.empty(L, M, dtype=torch.float32).pin_memory()
    y_dev = torch.empty(L, M, dtype=torch.float32, device=dev)

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        for l in range(L):
            mb.gemv(packed[l], alphas[l], K, M, N, 128, x_dev[l].view(torch.bfloat16), mb.BF16, 1,
                    y_dev[l], ws, stream=stream)
        y_host.copy_(y_dev, non_blocking=True)

    def time_e2e(replay):
        with torch.cuda.stream(stream):
            for _ in range(a.warmup):
                replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(a.steps):
                replay()
            e1.record(stream)
        e1.synchronize()
        t = e0.elapsed_time(e1) / a.steps
        return replica_max_ms(t, dist, dev) if world > 1 else t

    # Eagerly: one Python call per layer (host launch overhead included).
    eager_ms = time_e2e(e2e_step)
    # Eagerly through the C ABI itself: ctypes calls of mbok_gemv with raw
    # pointers prepared once (the binding's checks bypassed), the same copies.
    lib_gemv = mb.lib().mbok_gemv
    sp = stream.cuda_stream
    wsp, wsn = ws.data_ptr(), ws.numel()
    args = [(packed[l].data_ptr(), alphas[l].data_ptr(), x_dev[l].data_ptr(), y_dev[l].data_ptr())
            for l in range(L)]

    def e2e_abi_step():
        x_dev.copy_(x_host, non_blocking=True)
        for (pp, pa, px, py) in args:
            lib_gemv(pp, pa, K, M, N, 128, px, mb.BF16, 1, py, wsp, wsn, sp)
        y_host.copy_(y_dev, non_blocking=True)
    with torch.cuda.stream(stream):
        assert lib_gemv(args[0][0], args[0][1], K, M, N, 128, args[0][2], mb.BF16, 1, args[0][3], wsp, wsn, sp) == 0
    abi_ms = time_e2e(e2e_abi_step)
    # As a serving loop runs it: the whole step (copies and calls) captured
    # once in a CUDA graph and replayed; the copies still run every step.
    with torch.cuda.stream(stream):
        e2e_step()
    torch.cuda.synchronize()
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        e2e_step()
    serial_ms = time_e2e(e2e_graph.replay)
    del e2e_graph
    # The same copies pipelined with the layers, on a second stream: the
    # first 4 layers' inputs, then the rest (ready long before layer 4 needs
    # them); the outputs of all but the last 4 layers copied back while those
    # run, then the last 4.  One wait between layers (layer 4 on the second
    # input copy): each cross-stream wait or event between two layers costs
    # the overlap of their launches (5 chunks each way measured 258 us per
    # step, a third output copy at the halfway layer 248 us, this 246 us).
    cs = torch.cuda.Stream(device=dev)
    in_cuts, out_cuts = e2e_copy_cuts(L)
    chunks = len(in_cuts) - 1 + len(out_cuts) - 1

    def e2e_step_pipelined():
        cs.wait_stream(stream)
        ready = {}
        with torch.cuda.stream(cs):
            for a0, a1 in zip(in_cuts[:-1], in_cuts[1:]):
                x_dev[a0:a1].copy_(x_host[a0:a1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(cs)
                ready[a0] = ev
        out_at = dict(zip(out_cuts[1:], out_cuts[:-1]))   # chunk end -> chunk start
        for l in range(L):
            if l in ready:
                stream.wait_event(ready[l])
            mb.gemv(packed[l], alphas[l], K, M, N, 128, x_dev[l].view(torch.bfloat16), mb.BF16, 1,
                    y_dev[l], ws, stream=stream)
            if l + 1 in out_at:
                a0 = out_at[l + 1]
                done = torch.cuda.Event()
                done.record(stream)
                cs.wait_event(done)
                with torch.cuda.stream(cs):
                    y_host[a0:l + 1].copy_(y_dev[a0:l + 1], non_blocking=True)
        stream.wait_stream(cs)

    with torch.cuda.stream(stream):
        e2e_step_pipelined()
    torch.cuda.synchronize()
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=stream):
        e2e_step_pipelined()
    e2e_ms = time_e2e(e2e_graph.replay)
    e2e = {"value": replica_rate(L * bytes_per_layer, e2e_ms, world) / 1e9, "unit": UNIT,
           "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(y_host.numel() * 4),
           "ms_per_step": e2e_ms,
           "path": "mbok_gemv via the C ABI, pinned host x/y copied in and out every step in "
                   f"{chunks} copies on a second stream, overlapped with the layers; the step "
                   "(copies + calls) captured once in a CUDA graph and replayed",
           "serial": {"value": replica_rate(L * bytes_per_layer, serial_ms, world) / 1e9, "ms_per_step": serial_ms,
                      "path": "the same graph with all inputs copied before the first layer and all "
                              "outputs after the last"},
           "eager": {"value": replica_rate(L * bytes_per_layer, eager_ms, world) / 1e9, "ms_per_step": eager_ms,
                     "path": "the same step issued eagerly from Python, one binding call per layer"},
           "abi_direct": {"value": replica_rate(L * bytes_per_layer, abi_ms, world) / 1e9, "ms_per_step": abi_ms,
                          "us_per_call": 1e3 * abi_ms / L,
                          "path": "the same step issued eagerly as direct ctypes calls of mbok_gemv (C ABI, "
                                  "pointers prepared once), copies included"}}
    del e2e_graph

    del graph
    extras = None
    # The secondary rows are single-GPU rows: reported at N = 1 only, so a
    # replica run holds its GPUs just for the headline and end-to-end steps.
    if not a.no_extras and world == 1:
        del packed, alphas, xs, ys
        torch.cuda.empty_cache()
        extras = run_extras(torch, mb, wl, dev, peaks, a)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    # Secondary rows: one short JSON line each, printed before the headline
    # (which stays the last line); the headline carries a compact summary.
    compact = None
    if extras:
        compact = {}
        for name, row in extras.items():
            print(json.dumps({"row": name, **row}), flush=True)
            compact[name] = row_summary(row)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 x, 1-bit kernels, fp16 scales, fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": "llama7b_q_proj_k3_4096x4096_gemv_b1", "K": K, "M": M, "N": N,
                   "group": 128, "batch": 1, "layers_per_step": L,
                   "bytes_per_layer": bytes_per_layer, "us_per_layer": us_per_layer,
                   "l2": f"inputs larger than L2: {L} distinct weight copies, "
                         f"{L * bytes_per_layer / 1e6:.0f} MB per step vs 126 MB L2",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "kernel": "gemv_lut8_kernel<3,false,false> + gemv_combine_kernel (one layer = both launches)",
                     "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)" if peak_src == "measured"
                     else "fallback 6.65 TB/s"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": a.steps * L * launches_per_gemv,
        "rows": compact,
    }
    print(json.dumps(line), flush=True)


def row_summary(row: dict) -> list:
    """[time, rate, fraction of peak] of a secondary row, for the headline."""
    t = row.get("us", row.get("us_per_layer", row.get("ms_per_token", row.get("ms"))))
    rate = row.get("tflops", row.get("tokens_per_s", row.get("gbs", row.get("gbs_of_w", row.get("gbs_in")))))
    frac = row.get("frac_of_bf16_peak", row.get("frac_of_hbm"))
    return [None if v is None else round(float(v), 4) for v in (t, rate, frac)]


def run_extras(torch, mb, wl, dev, peaks, a):
    """Secondary rows, each timed with CUDA events (graph replays)."""
    out = {}
    rows = set(a.rows.split(","))
    stream = torch.cuda.Stream(device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(12345)
    if "gemm" in rows:
        run_gemm_row(torch, mb, wl, dev, peaks, stream, g, out)
    if "small_batch" in rows:
        run_small_batch_rows(torch, mb, wl, dev, peaks, stream, g, out)
    if "sweep" in rows:
        run_sweep_row(torch, mb, wl, dev, peaks, stream, g, out)
    if "svid" in rows:
        run_svid_row(torch, mb, wl, dev, peaks, stream, g, out)
    if "residual" in rows or "pack" in rows:
        run_conversion_rows(torch, mb, wl, dev, peaks, stream, g, out, rows)
    return out


def run_gemm_row(torch, mb, wl, dev, peaks, stream, g, out):
    # Prefill GEMM, K=3, 4096 x 4096, 2048 tokens: a graph of back-to-back
    # GEMMs (as a prefill runs its layers) on 20 distinct weight copies,
    # 142 MB of packed weights and scales, more than the 126 MB L2.
    K, M, N, T = 3, 4096, 4096, 2048
    L = 20
    packed = [torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                            device=dev, generator=g) for _ in range(L)]
    alphas = []
    for l in range(L):
        a = mb.empty_alpha(K, M, N, dev)
        mb.pack_alpha(torch.from_numpy(wl.alpha_decaying(K, M, N, 4001 + l).view(np.int16)).to(dev)
                      .view(torch.float16), K, M, N, a)
        alphas.append(a)
    X = torch.randn(T, N, device=dev, generator=g).to(torch.bfloat16)
    Y = torch.empty(T, M, dtype=torch.bfloat16, device=dev)
    for (suffix, prec, kern) in (("", mb.GEMM_AUTO, "gemm_tc_kernel<3,false> (one bf16 rounding per weight)"),
                                 ("_split", mb.GEMM_SPLIT, "gemm_tc_kernel<3,true> (hi + lo bf16 terms)")):
        def fn():
            for l in range(L):
                mb.gemm(packed[l], alphas[l], K, M, N, 128, X, T, Y, stream=stream, precision=prec)
        ms, gr = time_graph(torch, fn, 5, 3, stream)
        ms /= L
        tflops = 2.0 * M * N * T / (ms * 1e-3) / 1e12
        out["prefill_gemm_llama7b_q_proj_k3_t2048" + suffix] = {
            "us": 1e3 * ms, "tflops": tflops, "frac_of_bf16_peak": tflops / peaks["bf16_tflops"],
            "peak_tflops": peaks["bf16_tflops"], "kernel": kern, "gemms_per_graph": L,
            "l2": "20 distinct weight copies per graph (142 MB > 126 MB L2)"}
        del gr
    del packed, alphas, X, Y
    torch.cuda.empty_cache()


def run_small_batch_rows(torch, mb, wl, dev, peaks, stream, g, out):
    # Batch 1 / 4 / 16 on LLaMA-7B shapes (q_proj 4096x4096 K=3, gate 11008x4096
    # K=3, down 4096x11008 K=2), each on both GEMV kernels.  Enough distinct
    # weight copies per graph that they exceed L2 (>= 150 MB).
    shapes = (("q_proj", 3, 4096, 4096), ("gate", 3, 11008, 4096), ("down", 2, 4096, 11008))
    kernels = (("lookup", mb.GEMV_LOOKUP, True), ("lookup_weights_after_wait", mb.GEMV_LOOKUP, False),
               ("lookup_rows", mb.GEMV_LOOKUP_ROWS, True),
               ("tensor", mb.GEMV_TENSOR, True))
    for (name, K, M, N) in shapes:
        bpl = mb.packed_bytes(K, M, N) + 2 * mb.alpha_elems(K, M, N)
        L = max(8, -(-150_000_000 // bpl))
        packed = [torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                                device=dev, generator=g) for _ in range(L)]
        al = []
        for l in range(L):
            t = mb.empty_alpha(K, M, N, dev)
            mb.pack_alpha(torch.from_numpy(wl.alpha_decaying(K, M, N, 5000 + l).view(np.int16)).to(dev)
                          .view(torch.float16), K, M, N, t)
            al.append(t)
        ws = mb.zeros_workspace(K, M, N, 16, dev)
        for batch in (1, 4, 16):
            x = torch.randn(batch, N, device=dev, generator=g).to(torch.bfloat16)
            y = torch.empty(batch, M, dtype=torch.float32, device=dev)
            for (kname, kcode, static) in kernels:
                if batch > 1 and (kname.endswith("after_wait") or kname == "lookup_rows"
                                  or (name == "q_proj" and kname == "lookup")):
                    continue

                def fn():
                    for l in range(L):
                        mb.gemv(packed[l], al[l], K, M, N, 128, x, mb.BF16, batch, y, ws, stream=stream)
                mb.gemv_set_static_weights(static)
                with mb.gemv_kernel(kcode):
                    ms, gr = time_graph(torch, fn, 10, 3, stream)
                mb.gemv_set_static_weights(True)
                gbs = L * bpl / (ms * 1e-3) / 1e9
                out[f"gemv_llama7b_{name}_k{K}_{M}x{N}_b{batch}_{kname}"] = {
                    "us_per_layer": 1e3 * ms / L, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                    "layers": L}
                del gr
        del packed, al
        torch.cuda.empty_cache()


def run_svid_row(torch, mb, wl, dev, peaks, stream, g, out):
    # Rank-1-scaled kernels (SVID form), LLaMA-7B q_proj K=3, batch 1; distinct
    # weight copies per graph beyond L2.
    K, M, N = 3, 4096, 4096
    bpl = mb.packed_bytes(K, M, N) + 2 * K * (M + N)
    L = max(8, -(-150_000_000 // bpl))
    packed = [torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                            device=dev, generator=g) for _ in range(L)]
    s_in = [((torch.rand(K, N, device=dev, generator=g) * 0.4) + 0.8).to(torch.float16) for _ in range(L)]
    s_out = [((torch.rand(K, M, device=dev, generator=g) * 0.4) + 0.8).mul(0.016).to(torch.float16) for _ in range(L)]
    x = torch.randn(1, N, device=dev, generator=g).to(torch.bfloat16)
    y = torch.empty(1, M, dtype=torch.float32, device=dev)
    ws = mb.zeros_svid_workspace(K, M, N, 1, dev)

    def fn():
        for l in range(L):
            mb.gemv_svid(packed[l], s_in[l], s_out[l], K, M, N, x, mb.BF16, 1, y, ws, stream=stream)
    ms, gr = time_graph(torch, fn, 10, 3, stream)
    gbs = L * bpl / (ms * 1e-3) / 1e9
    out["gemv_svid_llama7b_q_proj_k3_4096x4096_b1"] = {
        "us_per_layer": 1e3 * ms / L, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"], "layers": L,
        "bytes_per_layer": bpl, "kernel": "gemv_lut8_kernel<1,false,true> (one CTA per kernel and slab)"}
    del gr, packed, s_in, s_out
    torch.cuda.empty_cache()


def run_sweep_row(torch, mb, wl, dev, peaks, stream, g, out):
    # LLaMA-13B linear sweep, K=4, 40 layers x 7 matrices, batch 1.
    K = 4
    layers = wl.LLAMA13B_LAYERS
    mats = []
    total_bytes = 0
    for _ in range(layers):
        for (name, M, N) in wl.LLAMA13B_LAYER:
            p = torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                              device=dev, generator=g)
            al = torch.empty(mb.alpha_elems(K, M, N), dtype=torch.float16, device=dev)
            al.copy_((torch.rand(al.shape, device=dev, generator=g) + 0.5) * 0.01)
            mats.append((p, al, M, N))
            total_bytes += mb.packed_bytes(K, M, N) + 2 * mb.alpha_elems(K, M, N)
    ws = mb.zeros_workspace(K, 13824, 13824, 1, dev)
    xin = {N: torch.randn(1, N, device=dev, generator=g).to(torch.bfloat16) for N in (5120, 13824)}
    yout = {M: torch.empty(1, M, dtype=torch.float32, device=dev) for M in (5120, 13824)}

    def sweep():
        for (p, al, M, N) in mats:
            mb.gemv(p, al, K, M, N, 128, xin[N], mb.BF16, 1, yout[M], ws, stream=stream)
    ms, gr = time_graph(torch, sweep, 5, 2, stream)
    gbs = total_bytes / (ms * 1e-3) / 1e9
    out["sweep_llama13b_k4_40x7_b1"] = {"ms_per_token": ms, "tokens_per_s": 1e3 / ms,
                                       "bytes_per_token": total_bytes, "gbs": gbs,
                                       "frac_of_hbm": gbs / peaks["hbm_gbs"], "launches": len(mats)}
    del gr, mats
    torch.cuda.empty_cache()

    # The same layers with the projections that share an input fused along M:
    # q, k, v (3 x 5120 rows) and gate, up (2 x 13824 rows) are one matrix each
    # (storage format 1 concatenates along M by concatenating octets), so a
    # layer is 4 launches instead of 7.  Then once more with every weight
    # read after the dependency wait.
    fused = (("qkv", 3 * 5120, 5120), ("o", 5120, 5120), ("gate_up", 2 * 13824, 5120), ("down", 5120, 13824))
    mats = []
    fused_bytes = 0
    for _ in range(layers):
        for (name, M, N) in fused:
            p = torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                              device=dev, generator=g)
            al = torch.empty(mb.alpha_elems(K, M, N), dtype=torch.float16, device=dev)
            al.copy_((torch.rand(al.shape, device=dev, generator=g) + 0.5) * 0.01)
            mats.append((p, al, M, N))
            fused_bytes += mb.packed_bytes(K, M, N) + 2 * mb.alpha_elems(K, M, N)
    ws = mb.zeros_workspace(K, 2 * 13824, 13824, 1, dev)
    yout = {M: torch.empty(1, M, dtype=torch.float32, device=dev) for (_, M, _) in fused}

    def sweep_fused():
        for (p, al, M, N) in mats:
            mb.gemv(p, al, K, M, N, 128, xin[N], mb.BF16, 1, yout[M], ws, stream=stream)
    for static in (True, False):
        mb.gemv_set_static_weights(static)
        ms, gr = time_graph(torch, sweep_fused, 5, 2, stream)
        mb.gemv_set_static_weights(True)
        gbs = fused_bytes / (ms * 1e-3) / 1e9
        out["sweep_llama13b_k4_40x4_fused_b1" + ("" if static else "_weights_after_wait")] = {
            "ms_per_token": ms, "tokens_per_s": 1e3 / ms, "bytes_per_token": fused_bytes, "gbs": gbs,
            "frac_of_hbm": gbs / peaks["hbm_gbs"], "launches": len(mats)}
        del gr
    del mats
    torch.cuda.empty_cache()

    # Each matrix with its own number of kernels (an illustrative allocation,
    # 3.14 kernels on average: q 3, k 2, v 4, o 3, gate 3, up 3, down 4), and
    # q/k/v and gate/up each one mbok_gemv_multi launch: 4 launches per layer.
    alloc = {"q": 3, "k": 2, "v": 4, "o": 3, "gate": 3, "up": 3, "down": 4}
    groups = (((("q", 5120), ("k", 5120), ("v", 5120)), 5120), ((("o", 5120),), 5120),
              ((("gate", 13824), ("up", 13824)), 5120), ((("down", 5120),), 13824))
    calls = []
    mixed_bytes = 0
    for _ in range(layers):
        for (grp, N) in groups:
            Ks = [alloc[n] for (n, _) in grp]
            Ms = [M for (_, M) in grp]
            ps, als = [], []
            for (K_, M_) in zip(Ks, Ms):
                ps.append(torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K_, M_, N) // 4,), dtype=torch.int32,
                                        device=dev, generator=g))
                al = torch.empty(mb.alpha_elems(K_, M_, N), dtype=torch.float16, device=dev)
                al.copy_((torch.rand(al.shape, device=dev, generator=g) + 0.5) * 0.01)
                als.append(al)
                mixed_bytes += mb.packed_bytes(K_, M_, N) + 2 * mb.alpha_elems(K_, M_, N)
            calls.append((ps, als, Ks, Ms, N))
    ws_m = torch.zeros(max(max(mb.gemv_multi_workspace_bytes(c[2], c[3], c[4]) for c in calls), 256),
                       dtype=torch.uint8, device=dev)
    ymix = {sum(c[3]): torch.empty(1, sum(c[3]), dtype=torch.float32, device=dev) for c in calls}

    def sweep_mixed():
        for (ps, als, Ks, Ms, N) in calls:
            mb.gemv_multi(ps, als, Ks, Ms, N, 128, xin[N], mb.BF16, 1, ymix[sum(Ms)], ws_m, stream=stream)
    ms, gr = time_graph(torch, sweep_mixed, 5, 2, stream)
    gbs = mixed_bytes / (ms * 1e-3) / 1e9
    out["sweep_llama13b_mixedk_40x4_multi_b1"] = {
        "ms_per_token": ms, "tokens_per_s": 1e3 / ms, "bytes_per_token": mixed_bytes, "gbs": gbs,
        "frac_of_hbm": gbs / peaks["hbm_gbs"], "launches": len(calls), "kernels": alloc}
    del gr, calls
    torch.cuda.empty_cache()


def run_conversion_rows(torch, mb, wl, dev, peaks, stream, g, out, rows):
    # Residual binarisation, LLaMA-7B gate 11008 x 4096, K=3.
    K, M, N = 3, 11008, 4096
    W = torch.randn(M, N, device=dev, generator=g) * 0.02
    packed = mb.empty_packed(K, M, N, dev)
    alpha = mb.empty_alpha(K, M, N, dev)
    R = torch.empty_like(W)
    ms, gr = time_graph(torch, lambda: mb.residual_binarize(W, M, N, K, 128, packed, alpha, R, stream=stream),
                        5, 2, stream)
    out["residual_binarize_llama7b_gate_k3"] = {"ms": ms, "gbs_of_w": 2 * W.numel() * 4 / (ms * 1e-3) / 1e9}
    del gr
    # Successive SVID (rank-1 scales by 6 power iterations per kernel), same shape.
    s_in = torch.empty(K, N, dtype=torch.float16, device=dev)
    s_out = torch.empty(K, M, dtype=torch.float16, device=dev)
    svws = torch.empty(int(mb.lib().mbok_svid_workspace_bytes(M, N)), dtype=torch.uint8, device=dev)
    ms, gr = time_graph(torch, lambda: mb.svid_binarize(W, M, N, K, 6, packed, s_in, s_out, R, svws, stream=stream),
                        3, 2, stream)
    out["svid_binarize_llama7b_gate_k3_iters6"] = {"ms": ms, "passes_over_w": K * (2 * 6 + 2) + 1,
                                                    "gbs_of_passes": (K * (2 * 6 + 2) + 1) * W.numel() * 4
                                                    / (ms * 1e-3) / 1e9}
    del gr
    # Least-squares scale refit for the kernels just produced, same shape.
    ms, gr = time_graph(torch, lambda: mb.refit_alpha(W, packed, K, M, N, 128, alpha, stream=stream), 5, 2, stream)
    out["refit_alpha_llama7b_gate_k3"] = {"ms": ms, "gbs_of_w": W.numel() * 4 / (ms * 1e-3) / 1e9}
    del gr
    # Packing of int8 signs, same shape.
    S = torch.randint(-1, 1, (K, M, N), dtype=torch.int8, device=dev, generator=g)
    ms, gr = time_graph(torch, lambda: mb.pack_bits(S, K, M, N, packed, stream=stream), 5, 2, stream)
    out["pack_bits_llama7b_gate_k3"] = {"ms": ms, "gbs_in": S.numel() / (ms * 1e-3) / 1e9}
    del gr


def profile_gemv(spec: str):
    """Four launches of one GEMV on random weights (for an ncu capture)."""
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    mbuild.build()
    K, M, N, batch, kern = (int(v) for v in spec.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                           device=dev, generator=g)
    alpha = (torch.rand(mb.alpha_elems(K, M, N), device=dev, generator=g) * 0.01).to(torch.float16)
    x = torch.randn(batch, N, device=dev, generator=g).to(torch.bfloat16)
    y = torch.empty(batch, M, dtype=torch.float32, device=dev)
    ws = mb.zeros_workspace(K, M, N, batch, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2
    with mb.gemv_kernel(kern):
        for _ in range(4):
            flush.zero_()
            mb.gemv(packed, alpha, K, M, N, 128, x, mb.BF16, batch, y, ws)
    torch.cuda.synchronize()


def profile_svid(spec: str):
    """Four launches of the rank-1-form GEMV on random weights and scales, with
    L2 flushed before each (for an ncu capture)."""
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    mbuild.build()
    K, M, N = (int(v) for v in spec.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                           device=dev, generator=g)
    s_in = ((torch.rand(K, N, device=dev, generator=g) * 0.4) + 0.8).to(torch.float16)
    s_out = ((torch.rand(K, M, device=dev, generator=g) * 0.4) + 0.8).mul(0.016).to(torch.float16)
    x = torch.randn(1, N, device=dev, generator=g).to(torch.bfloat16)
    y = torch.empty(1, M, dtype=torch.float32, device=dev)
    ws = mb.zeros_svid_workspace(K, M, N, 1, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2
    for _ in range(4):
        flush.zero_()
        mb.gemv_svid(packed, s_in, s_out, K, M, N, x, mb.BF16, 1, y, ws)
    torch.cuda.synchronize()


def profile_convert(spec: str):
    """Two launches each of residual binarisation and bit packing on random
    inputs, then one scale refit and one successive-SVID conversion, with L2
    flushed before each call (for an ncu capture)."""
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    mbuild.build()
    K, M, N = (int(v) for v in spec.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    W = torch.randn(M, N, device=dev, generator=g) * 0.02
    R = torch.empty_like(W)
    S = torch.randint(-1, 1, (K, M, N), dtype=torch.int8, device=dev, generator=g)
    packed = mb.empty_packed(K, M, N, dev)
    alpha = mb.empty_alpha(K, M, N, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > L2
    for _ in range(2):
        flush.zero_()
        mb.residual_binarize(W, M, N, K, 128, packed, alpha, R)
        flush.zero_()
        mb.pack_bits(S, K, M, N, packed)
    flush.zero_()
    mb.residual_binarize(W, M, N, K, 128, packed, alpha, R)
    flush.zero_()
    mb.refit_alpha(W, packed, K, M, N, 128, alpha)
    s_in = torch.empty(K, N, dtype=torch.float16, device=dev)
    s_out = torch.empty(K, M, dtype=torch.float16, device=dev)
    svws = torch.empty(int(mb.lib().mbok_svid_workspace_bytes(M, N)), dtype=torch.uint8, device=dev)
    flush.zero_()
    mb.svid_binarize(W, M, N, K, 6, packed, s_in, s_out, R, svws)
    torch.cuda.synchronize()


def profile_gemm(spec: str):
    """Three launches of one prefill GEMM on random weights (for an ncu capture)."""
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    mbuild.build()
    K, M, N, T, prec = (int(v) for v in spec.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (mb.packed_bytes(K, M, N) // 4,), dtype=torch.int32,
                           device=dev, generator=g)
    alpha = (torch.rand(mb.alpha_elems(K, M, N), device=dev, generator=g) * 0.01 + 0.005).to(torch.float16)
    X = torch.randn(T, N, device=dev, generator=g).to(torch.bfloat16)
    Y = torch.empty(T, M, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        mb.gemm(packed, alpha, K, M, N, 128, X, T, Y, precision=prec)
    torch.cuda.synchronize()


def phase_profile(spec: str):
    """Per-phase split of a chain of batch-1 decode GEMVs (slab lookup kernel +
    slab combine), from the profiling build's per-CTA globaltimer stamps.  The
    chain of LAYERS distinct weight copies is captured in a CUDA graph (as in
    the headline) and replayed; the stamps of the last replay are read back.
    Per layer l, on the critical path:
      handoff_in  = first main CTA past its dependency wait - last combine CTA of layer l-1 done
      x_tables    = last main CTA with its tables built - first main CTA past the wait
      loop        = last warp out of the streaming loop - last CTA with tables built
      drain       = last warp's copies drained - last warp out of the loop
      handoff_mid = first combine CTA past its wait - main kernel done
      combine     = last combine CTA done - first combine CTA past its wait
    (the six terms add up to the layer's period).  With a fifth field `svid` the
    chain runs the rank-1 form (mbok_gemv_svid: one CTA per kernel and slab)."""
    import ctypes
    import statistics
    import torch
    import boolean_weight_matmul_b200 as mb
    from boolean_weight_matmul_b200 import build as mbuild
    from boolean_weight_matmul_b200 import workloads as wl
    mbuild.build()
    path = mbuild.build(variant="stamps")
    S = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    S.mbok_gemv.argtypes = [vp, vp, i, i, i, i, vp, i, i, vp, vp, sz, vp]
    S.mbok_gemv.restype = i
    S.mbok_gemv_svid.argtypes = [vp, vp, vp, i, i, i, vp, i, i, vp, vp, sz, vp]
    S.mbok_gemv_svid.restype = i
    S.mbok_debug_phase_stamps.argtypes = [vp, sz, vp, sz]
    S.mbok_debug_phase_reset.argtypes = [i]
    fields = spec.split(",")
    svid = len(fields) == 5 and fields[4] == "svid"
    assert len(fields) == 4 or svid, "K,M,N,LAYERS[,svid]"
    K, M, N, L = (int(v) for v in fields[:4])
    assert 2 <= L <= 64
    dev = torch.device("cuda:0")
    packed, alphas, xs = build_layers(torch, mb, wl, K, M, N, L, dev, 4242)
    y = torch.empty(1, M, dtype=torch.float32, device=dev)
    if svid:
        g = torch.Generator(device=dev)
        g.manual_seed(4243)
        s_in = [((torch.rand(K, N, device=dev, generator=g) * 0.4) + 0.8).to(torch.float16) for _ in range(L)]
        s_out = [((torch.rand(K, M, device=dev, generator=g) * 0.4) + 0.8).mul(0.016).to(torch.float16)
                 for _ in range(L)]
        ws = mb.zeros_svid_workspace(K, M, N, 1, dev)
    else:
        ws = mb.zeros_workspace(K, M, N, 1, dev)
    stream = torch.cuda.Stream(device=dev)

    def chain():
        for l in range(L):
            if svid:
                st = S.mbok_gemv_svid(packed[l].data_ptr(), s_in[l].data_ptr(), s_out[l].data_ptr(), K, M, N,
                                      xs[l].data_ptr(), mb.BF16, 1, y.data_ptr(), ws.data_ptr(), ws.numel(),
                                      stream.cuda_stream)
            else:
                st = S.mbok_gemv(packed[l].data_ptr(), alphas[l].data_ptr(), K, M, N, 128, xs[l].data_ptr(),
                                 mb.BF16, 1, y.data_ptr(), ws.data_ptr(), ws.numel(), stream.cuda_stream)
            assert st == 0, st

    with torch.cuda.stream(stream):
        chain()   # eager: kernel attributes set outside the capture
    torch.cuda.synchronize()
    assert S.mbok_debug_phase_reset(1) == 0   # the capture takes slots 0 .. L-1
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        chain()
    with torch.cuda.stream(stream):
        for _ in range(5):
            graph.replay()
    torch.cuda.synchronize()
    assert S.mbok_debug_phase_reset(0) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    per_layer_us = e0.elapsed_time(e1) * 1e3 / L
    main = np.zeros((64, 1024, 5), dtype=np.uint64)
    comb = np.zeros((64, 1024, 3), dtype=np.uint64)
    assert S.mbok_debug_phase_stamps(main.ctypes.data, main.nbytes, comb.ctypes.data, comb.nbytes) == 0
    del graph
    nm = int((main[0, :, 0] > 0).sum())
    nc = int((comb[0, :, 0] > 0).sum())
    terms = {k: [] for k in ("handoff_in", "x_tables", "loop", "drain", "handoff_mid", "combine", "period")}
    spread = {k: [] for k in ("main_wait_spread", "main_tables_spread", "main_end_spread", "combine_start_spread",
                              "combine_wait_spread", "combine_cta_work", "combine_end_spread")}
    for l in range(1, L):
        m = main[l, :nm].astype(np.int64)
        c = comb[l, :nc].astype(np.int64)
        cp = comb[l - 1, :nc].astype(np.int64)
        prev_end = cp[:, 2].max()
        v = {"handoff_in": m[:, 1].min() - prev_end,
             "x_tables": m[:, 2].max() - m[:, 1].min(),
             "loop": m[:, 3].max() - m[:, 2].max(),
             "drain": m[:, 4].max() - m[:, 3].max(),
             "handoff_mid": c[:, 1].min() - m[:, 4].max(),
             "combine": c[:, 2].max() - c[:, 1].min(),
             "period": c[:, 2].max() - prev_end}
        for k, x in v.items():
            terms[k].append(x / 1000.0)
        d = {"main_wait_spread": m[:, 1].max() - m[:, 1].min(),
             "main_tables_spread": m[:, 2].max() - m[:, 2].min(),
             "main_end_spread": m[:, 4].max() - m[:, 4].min(),
             "combine_start_spread": c[:, 0].max() - c[:, 0].min(),
             "combine_wait_spread": c[:, 1].max() - c[:, 1].min(),
             "combine_cta_work": float(np.median(c[:, 2] - c[:, 1])),
             "combine_end_spread": c[:, 2].max() - c[:, 2].min()}
        for k, x in d.items():
            spread[k].append(x / 1000.0)
    med = {k: statistics.median(x) for k, x in terms.items()}
    out = {"phase_profile": f"K={K} {M}x{N} batch 1, {L} layers, graph replay" + (", rank-1 form" if svid else ""),
           "main_ctas": nm, "combine_ctas": nc, "layer_us_events": round(per_layer_us, 3),
           "median_us": {k: round(x, 3) for k, x in med.items()},
           "share_of_period": {k: round(med[k] / med["period"], 3) for k in med if k != "period"},
           "spread_median_us": {k: round(statistics.median(x), 3) for k, x in spread.items()}}
    print(json.dumps(out))


def main():
    a = args_parse()
    if a.phase_profile:
        phase_profile(a.phase_profile)
        return
    if a.profile_gemv:
        profile_gemv(a.profile_gemv)
        return
    if a.profile_gemm:
        profile_gemm(a.profile_gemm)
        return
    if a.profile_convert:
        profile_convert(a.profile_convert)
        return
    if a.profile_svid:
        profile_svid(a.profile_svid)
        return
    if a.impl == "reference":
        run_reference(a)
    else:
        run_gpu(a)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark: exact attention forward + backward on B200 through the C ABI.

One step = fa_fwd + fa_bwd over the whole workload (default: the causal
bf16 B=2 H=16 N=8192 d=128 workload), inputs already resident in device memory.
Prints one JSON line (rank 0).  Throughput counts 4*N^2*d flops per head
forward and 2.5x that backward, halved for causal.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
copy of the workload (a different seed), with no data-path collective; the
timed region is bracketed by barriers and the reported time is the maximum
over ranks ("weak" scaling).  --impl reference times the CPU fp64 oracle (the
only other implementation of this path) on a bounded sample of the workload,
on rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_online_b200 import workloads as W  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {  # the files each profiled kernel (and its launch configuration) is built from
    "bwd_sm100_kernel": ("bwd_sm100.cuh", "sm100_ptx.cuh", "layout.cuh", "fa_api.cu"),
    "fwd_sm100_kernel": ("fwd_sm100.cuh", "sm100_ptx.cuh", "layout.cuh", "fa_api.cu"),
    "fwd_persist_kernel": ("fwd_persist_sm100.cuh", "fwd_sm100.cuh", "sm100_ptx.cuh", "layout.cuh", "fa_api.cu"),
}


def _code_only(text: str) -> str:
    """C++ source without comments and with whitespace runs collapsed: edits to
    comments alone leave the compiled kernel, and so the hash, unchanged."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel: str | None = None) -> str:
    """Hash of the code (comments dropped) of the sources of `kernel` (of every
    CUDA source when None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_online_b200", "csrc")
    names = KERNEL_SOURCES.get(kernel) if kernel else None
    for name in sorted(names or os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if it
    was captured on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.rows = []
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mhz = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        power = [float(r[3]) for r in self.rows if r[3].replace(".", "").isdigit()]
        load = [m for m in mhz] or [0.0]
        reasons = sorted({n for r in self.rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows), "power_w_max": max(power) if power else None}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(w: W.Workload, min_seconds: float, max_heads: int):
    """Times the CPU oracle (fwd + bwd) on whole query heads of the workload until
    at least `min_seconds` have elapsed.  Returns (seconds, flops, heads)."""
    from oracle import ref
    x = W.make_inputs(w)
    g = w.H // w.Hkv
    fwd_f, bwd_f = W.flops(w)
    per_head = (fwd_f + bwd_f) / (w.B * w.H)
    spent, heads = 0.0, 0
    order = [(b, h) for h in range(w.H) for b in range(w.B)]
    for b, h in order[:max_heads]:
        kh = h // g
        q, do = x["q"][b:b + 1, h:h + 1], x["do"][b:b + 1, h:h + 1]
        k, v = x["k"][b:b + 1, kh:kh + 1], x["v"][b:b + 1, kh:kh + 1]
        t0 = time.perf_counter()
        ref.forward(q, k, v, w.scale, w.causal, w.window)
        ref.backward(q, k, v, do, w.scale, w.causal, w.window)
        spent += time.perf_counter() - t0
        heads += 1
        if spent >= min_seconds:
            break
    return spent, per_head * heads, heads


def run_reference(args, w, world, rank):
    if rank != 0:
        return 0
    fwd_f, bwd_f = W.flops(w)
    per_head = (fwd_f + bwd_f) / (w.B * w.H)
    from oracle import ref
    x = W.make_inputs(w)
    g = w.H // w.Hkv
    q, do = x["q"][0:1, 0:1], x["do"][0:1, 0:1]
    k, v = x["k"][0:1, 0:1], x["v"][0:1, 0:1]

    def step():
        ref.forward(q, k, v, w.scale, w.causal, w.window)
        ref.backward(q, k, v, do, w.scale, w.causal, w.window)

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = per_head / sec / 1e12
    sample = f"one query head (b=0, h=0; kv head 0) of {w.name}, forward+backward, every row"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "attention fwd+bwd TFLOP/s (bf16, causal N=8192 d=128) and % of BF16 tensor peak"


def algorithmic_bytes(w: W.Workload, kind: str) -> float:
    """Bytes a kernel must move between HBM and the SMs at the least: the
    forward reads Q, K, V and writes O and the logsumexp; the backward kernel
    reads Q, K, V, dO, the logsumexp and D, writes dK and dV, and moves the fp32
    dQ accumulator in and out once."""
    e = 2 if w.dtype == "bf16" else 4
    q = w.B * w.H * w.N * w.d * e
    kv = w.B * w.Hkv * w.N * w.d * e
    rows = w.B * w.H * w.N
    if kind == "fwd":
        return q + 2 * kv + q + 4 * rows
    return q + 2 * kv + q + 8 * rows + 2 * kv + 8 * rows * w.d


def config_of(w: W.Workload, world: int):
    in_bytes = (2 * w.B * w.H + 2 * w.B * w.Hkv) * w.N * w.d * (2 if w.dtype == "bf16" else 4)
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
            "window": w.window, "scale": "1/sqrt(d)", "parallelism": f"replicas{world}" if world > 1 else "single",
            "fwd_splits": getattr(config_of, "splits", 0),
            "block_density": getattr(config_of, "block_density", None),
            "l2": f"inputs larger than L2: {in_bytes / 2**20:.0f} MiB of Q,K,V,dO per step per GPU (no flush)"}


def run_ours(args, w, world, rank, local):
    import torch
    import exact_io_aware_online_b200 as fa
    from exact_io_aware_online_b200 import _build

    if rank == 0:
        _build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fa.lib()
    wr = w.with_(seed=w.seed + 1000 * rank)
    host = W.make_inputs(wr)
    x = {k: t.to(dev) for k, t in host.items()}
    B, H, N, d = x["q"].shape
    o = torch.empty_like(x["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d, fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP32),
                     dtype=torch.uint8, device=dev)
    bmask = None
    if args.block_density is not None:
        if w.window >= 0:
            raise SystemExit("--block-density: window workloads are not supported")
        m = W.block_mask(w.N, args.block_density, w.seed + 77, w.causal)
        bmask = torch.from_numpy(m).to(dev)
        flops_override = 4.0 * w.d * W.block_pairs(w.N, m, w.causal) * w.B * w.H
    ws_split = None
    if args.splits:
        ws_split = torch.empty(int(fa.lib().fa_fwd_splitkv_workspace_size(B, H, N, d, args.splits)),
                               dtype=torch.uint8, device=dev)
    K = args.steps
    ev_f = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    # the whole backward call (preprocess + main kernel + dQ conversion), on the same stream
    ev_bc = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ev_b = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    def step(i=None):
        if i is not None:
            fa.set_timing_events(*ev_f[i])
        if bmask is not None:
            fa.fwd_blocksparse(x["q"], x["k"], x["v"], bmask, w.scale, w.causal, w.window, out=o, lse=lse)
        elif args.splits:
            fa.fwd_splitkv(x["q"], x["k"], x["v"], args.splits, w.scale, w.causal, w.window, out=o, lse=lse,
                           workspace=ws_split)
        else:
            fa.fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window, out=o, lse=lse)
        if i is not None:
            fa.set_timing_events(*ev_b[i])
            ev_bc[i][0].record()
        if bmask is not None:
            fa.bwd_blocksparse(x["q"], x["k"], x["v"], o, lse, x["do"], bmask, w.scale, w.causal, w.window,
                               workspace=ws, grads=(dq, dk, dv))
        else:
            fa.bwd(x["q"], x["k"], x["v"], o, lse, x["do"], w.scale, w.causal, w.window, workspace=ws,
                   grads=(dq, dk, dv))
        if i is not None:
            ev_bc[i][1].record()
            fa.set_timing_events(None, None)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # torch creates an event's CUDA handle lazily, on its first record():
    # record each once so the library receives real handles.
    for a, b in ev_f + ev_b:
        a.record()
        b.record()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.device_status() != 0:
        raise RuntimeError("device-side timeout during warm-up")
    stream = torch.cuda.current_stream(dev)
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t_start.record(stream)
        for i in range(K):
            step(i)
        t_stop.record(stream)
        torch.cuda.synchronize()
    barrier()
    if fa.device_status() != 0:
        raise RuntimeError("device-side timeout during the timed region")
    ms = t_start.elapsed_time(t_stop)
    fwd_ms = [a.elapsed_time(b) for a, b in ev_f]
    bwd_ms = [a.elapsed_time(b) for a, b in ev_b]
    bwd_call_ms = [a.elapsed_time(b) for a, b in ev_bc]
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    fwd_f, bwd_f = W.flops(w)
    if bmask is not None:  # the kept (query, key) pairs inside the switched-on blocks
        fwd_f, bwd_f = flops_override, 2.5 * flops_override
    ms_step = ms / K
    value = world * (fwd_f + bwd_f) / (ms_step * 1e-3) / 1e12

    pk, src = peaks()
    # kernel times: median over the timed steps (the best one is reported beside it)
    fwd_k, bwd_k = statistics.median(fwd_ms), statistics.median(bwd_ms)
    if bwd_k * bwd_f >= 0 and bwd_k >= fwd_k:
        dom_name, dom_ms, dom_flops = "bwd_sm100_kernel", bwd_k, bwd_f
    else:
        dom_name, dom_ms, dom_flops = "fwd_sm100_kernel", fwd_k, fwd_f
    if w.dtype != "bf16":
        dom_name = dom_name.replace("sm100", "simt_f32")
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    # The kernels run for milliseconds inside a region of tens of milliseconds:
    # the burst matmul figure is the denominator, the sustained one is kept beside it.
    peak = float(pk["bf16_tflops"])
    sustained = float(pk["bf16_tflops_sustained"])
    dom_bytes = algorithmic_bytes(w, "bwd" if dom_name.startswith("bwd") else "fwd")
    ridge = peak * 1e12 / (float(pk["hbm_gbs"]) * 1e9)  # flop per byte where the two roofs meet
    if dom_flops / dom_bytes >= ridge:
        roof = {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_kind": f"bf16 dense, burst ({src})",
                "frac_of_sustained": achieved / sustained}
    else:  # below the ridge (narrow bands): the bytes that must move bound the kernel
        gbs = dom_bytes / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": gbs, "peak": float(pk["hbm_gbs"]), "unit": "GB/s",
                "frac": gbs / float(pk["hbm_gbs"]), "peak_kind": f"HBM copy ({src})",
                "tensor_tflops": achieved, "tensor_frac_of_burst": achieved / peak}
    roof.update({"traffic": ncu_traffic(dom_name, w.name), "algorithmic_bytes": dom_bytes,
                 "arithmetic_intensity": dom_flops / dom_bytes, "ridge": ridge,
                 "kernel_time": "median of the timed steps (CUDA events on the launching stream)",
                 "fwd_kernel_ms": fwd_k, "bwd_kernel_ms": bwd_k,
                 "fwd_kernel_ms_best": min(fwd_ms), "bwd_kernel_ms_best": min(bwd_ms),
                 "fwd_kernel_tflops": fwd_f / (fwd_k * 1e-3) / 1e12,
                 "bwd_kernel_tflops": bwd_f / (bwd_k * 1e-3) / 1e12,
                 # the backward as a whole: preprocess + main kernel + dQ conversion
                 "bwd_call_ms": statistics.median(bwd_call_ms), "bwd_call_ms_best": min(bwd_call_ms),
                 "bwd_call_tflops": bwd_f / (statistics.median(bwd_call_ms) * 1e-3) / 1e12})

    # ---- end to end: pinned host inputs -> device, fwd+bwd, results -> pinned host.
    # Every step copies its inputs in and its results out; consecutive steps are
    # double-buffered on three streams (upload, compute, download), so step i's
    # upload overlaps step i-1's compute and step i-2's download, as an input
    # pipeline would.  The timed region covers all copies of all K steps.
    e2e = None
    if not args.no_e2e:
        hin = {k: t.pin_memory() for k, t in host.items()}
        names_out = ("o", "lse", "dq", "dk", "dv")
        shapes = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
        hout = [{k_: torch.empty(t.shape, dtype=t.dtype).pin_memory() for k_, t in shapes.items()} for _ in range(2)]
        dx = [x, {k_: torch.empty_like(t) for k_, t in x.items()}]          # device inputs, two sets
        dy = [dict(shapes), {k_: torch.empty_like(t) for k_, t in shapes.items()}]  # device results, two sets
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        computed = [None, None]  # event: compute of the last step that used buffer set j finished
        downloaded = [None, None]  # event: download of the last step that used buffer set j finished

        def e2e_step(i):
            j = i % 2
            xi, yi = dx[j], dy[j]
            with torch.cuda.stream(s_up):
                if computed[j] is not None:
                    s_up.wait_event(computed[j])  # step i-2 has finished reading these inputs
                for k_ in ("q", "k", "v", "do"):
                    xi[k_].copy_(hin[k_], non_blocking=True)
                up = ev()
                up.record(s_up)
            stream.wait_event(up)
            if downloaded[j] is not None:
                stream.wait_event(downloaded[j])  # step i-2's results have left these buffers
            fa.fwd(xi["q"], xi["k"], xi["v"], w.scale, w.causal, w.window, out=yi["o"], lse=yi["lse"])
            fa.bwd(xi["q"], xi["k"], xi["v"], yi["o"], yi["lse"], xi["do"], w.scale, w.causal, w.window,
                   workspace=ws, grads=(yi["dq"], yi["dk"], yi["dv"]))
            computed[j] = ev()
            computed[j].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(computed[j])
                for k_ in names_out:
                    hout[j][k_].copy_(yi[k_], non_blocking=True)
                downloaded[j] = ev()
                downloaded[j].record(s_down)

        def join():
            stream.wait_stream(s_up)
            stream.wait_stream(s_down)

        for i in range(max(2, args.warmup)):
            e2e_step(i)
        join()
        torch.cuda.synchronize()
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_up.wait_stream(stream)
        s_down.wait_stream(stream)
        a.record(stream)
        s_up.wait_event(a)
        for i in range(K):
            e2e_step(i)
        join()
        b_.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = a.elapsed_time(b_)
        if world > 1:
            import torch.distributed as dist
            t = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in hout[0].values())
        e2e = {"value": world * (fwd_f + bwd_f) / (ems / K * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems / K,
               "pipeline": "double-buffered; upload, compute and download of consecutive steps overlap"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded sample by default; --full-oracle: every query head
        sec, flops_done, heads = oracle_sample(w, float("inf") if args.full_oracle else args.cpu_seconds, w.B * w.H)
        cpu = {"value": flops_done / sec / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{heads} whole query head(s) of {w.name} (fwd+bwd, every row), {sec:.1f} s",
               "host_cpus": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": config_of(w, world), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk.summary(), "gpu_launches": K * (1 + 3),
            "frac_of_peak": {"sustained": value / world / float(pk["bf16_tflops_sustained"]),
                             "burst": value / world / float(pk["bf16_tflops"]), "peaks": src},
        }
        print(json.dumps(line), flush=True)
    return 0


DECODE_SHAPE = dict(B=8, H=32, Hkv=8, Nk=32768, d=128)  # one new token per sequence vs a 32768-token cache


def run_decode(args, rank, local):
    """Decode forward (fa_fwd_decode): Nq new queries against a long cache,
    causal, bf16.  Memory-bound: the figure of merit is the bytes it must read
    (K and V once, plus Q) and write (O, LSE) per second, against the measured
    HBM copy bandwidth."""
    import torch
    import exact_io_aware_online_b200 as fa
    from exact_io_aware_online_b200 import _build
    if rank == 0:
        _build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    S = DECODE_SHAPE
    B, H, Hkv, Nk, d, Nq = S["B"], S["H"], S["Hkv"], S["Nk"], S["d"], args.decode
    g = torch.Generator("cpu").manual_seed(90 + rank)
    q = torch.randn((B, H, Nq, d), generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16).to(dev)
    splits = args.splits or fa.decode_splits(B, H, Hkv, Nq, Nk)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(int(fa.lib().fa_fwd_decode_workspace_size(B, H, Hkv, Nq, d, splits)), dtype=torch.uint8,
                     device=dev)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        a.record()
        b.record()
    # the cache (2 x 512 MiB) is larger than L2, so every step reads it from HBM
    for _ in range(args.warmup):
        fa.fwd_decode(q, k, v, splits, 1.0 / d ** 0.5, True, out=o, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t0.record(stream)
        for i in range(K):
            fa.set_timing_events(*ev[i])
            fa.fwd_decode(q, k, v, splits, 1.0 / d ** 0.5, True, out=o, lse=lse, workspace=ws)
        fa.set_timing_events(None, None)
        t1.record(stream)
        torch.cuda.synchronize()
    if fa.device_status() != 0:
        raise RuntimeError("device-side timeout during the timed region")
    ms = t0.elapsed_time(t1) / K
    kern = statistics.median(a.elapsed_time(b) for a, b in ev)
    algo = (2 * B * Hkv * Nk * d + 2 * B * H * Nq * d) * 2 + B * H * Nq * 4  # K, V, Q read; O written; LSE
    pk, src = peaks()
    peak = float(pk["hbm_gbs"])
    if rank == 0:
        print(json.dumps({
            "metric": "decode forward GB/s (bf16, causal, one cache read per step)", "value": algo / (ms * 1e-3) / 1e9,
            "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"decode_b{B}h{H}kv{Hkv}_nq{Nq}_nk{Nk}_d{d}", "splits": splits,
                       "l2": "cache of 1 GiB, larger than L2 (no flush)"},
            "roofline": {"bound": "hbm", "kernel": "fwd_sm100_kernel (decode, split)", "achieved":
                         algo / (kern * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": algo / (kern * 1e-3) / 1e9 / peak,
                         "traffic": ncu_traffic("fwd_sm100_kernel", f"decode_b{B}h{H}kv{Hkv}_nq{Nq}_nk{Nk}_d{d}"),
                         "peak_kind": f"HBM copy ({src})", "kernel_ms": kern},
            "clocks": clk.summary(), "gpu_launches": 2 * K}), flush=True)
    return 0


PACKED_SHAPE = dict(H=16, Hkv=16, d=128, lo=64, hi=448)  # lengths uniform in [lo, hi], mean 256


def packed_lengths(nseq: int, seed: int = 91):
    """Seeded sequence lengths of the packed workload (uniform in [lo, hi])."""
    import numpy as np
    rng = np.random.default_rng(seed)
    return rng.integers(PACKED_SHAPE["lo"], PACKED_SHAPE["hi"] + 1, size=nseq).tolist()


def run_packed(args, rank, local):
    """Packed variable lengths (fa_fwd_packed / fa_bwd_packed): args.packed
    short causal sequences concatenated along the token axis, forward +
    backward per step, every sequence in one launch per kernel.  Flops are
    counted per sequence as for the headline metric (4 L^2 d / 2 per head
    forward, 2.5 times that backward)."""
    import torch
    import exact_io_aware_online_b200 as fa
    from exact_io_aware_online_b200 import _build
    if rank == 0:
        _build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    S = PACKED_SHAPE
    H, Hkv, d = S["H"], S["Hkv"], S["d"]
    lens = packed_lengths(args.packed)
    cu = [0]
    for L in lens:
        cu.append(cu[-1] + L)
    T = cu[-1]
    g = torch.Generator("cpu").manual_seed(92 + rank)
    q = torch.randn((T, H, d), generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn((T, Hkv, d), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((T, Hkv, d), generator=g).to(torch.bfloat16).to(dev)
    do = torch.randn((T, H, d), generator=g).to(torch.bfloat16).to(dev)
    cu_dev = torch.tensor(cu, dtype=torch.int32, device=dev)
    o, lse = torch.empty_like(q), torch.empty(T * H, dtype=torch.float32, device=dev)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    ws = torch.empty(int(fa.lib().fa_bwd_packed_workspace_size((ctypes.c_int * len(cu))(*cu), len(lens), H, d, 0)),
                     dtype=torch.uint8, device=dev)
    scale = 1.0 / d ** 0.5

    def step():  # host offsets for the checks, the device copy for the kernels: no read-back per call
        fa.fwd_packed(q, k, v, cu, scale, True, out=o, lse=lse, cu_seqlens_dev=cu_dev)
        fa.bwd_packed(q, k, v, o, lse, do, cu, scale, True, workspace=ws, grads=grads, cu_seqlens_dev=cu_dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        t0.record(stream)
        for _ in range(K):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    if fa.device_status() != 0:
        raise RuntimeError("device-side timeout during the timed region")
    ms = t0.elapsed_time(t1) / K
    flops = sum(3.5 * 2.0 * L * L * d * H for L in lens)
    if rank == 0:
        print(json.dumps({
            "metric": "packed variable-length attention fwd+bwd TFLOP/s (bf16, causal, d=128)",
            "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"packed_{len(lens)}seq_len{S['lo']}to{S['hi']}_h{H}_d{d}_causal", "tokens": T,
                       "l2": f"{4 * T * H * d * 2 / 2**20:.0f} MiB of Q, K, V, dO per step (no flush)"},
            "clocks": clk.summary(), "gpu_launches": 4 * K}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE, choices=list(W.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--full-oracle", action="store_true",
                    help="time the CPU oracle on every query head of the workload (not a bounded sample)")
    ap.add_argument("--splits", type=int, default=0, help="split-KV forward with this many key chunks (0: off)")
    ap.add_argument("--block-density", type=float, default=None,
                    help="block-sparse attention with a seeded mask keeping this fraction of 128x128 blocks")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="run the workload at this sequence length instead (e.g. the DRAM-traffic sweep over N)")
    ap.add_argument("--decode", type=int, default=0,
                    help="time the decode forward instead: this many new queries per sequence against a "
                         "32768-token cache (B=8, 32 query heads on 8 kv heads, d=128, causal)")
    ap.add_argument("--packed", type=int, default=0,
                    help="time packed variable lengths instead: this many causal sequences of 64..448 tokens "
                         "(16 heads, d=128), forward + backward, one launch per kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    w = W.WORKLOADS[args.workload]
    if args.seq_len is not None:
        if args.seq_len < 1:
            ap.error("--seq-len must be >= 1")
        w = w.with_(N=args.seq_len, name=re.sub(r"_n\d+_", f"_n{args.seq_len}_", w.name))
    config_of.splits = args.splits
    config_of.block_density = args.block_density
    try:
        if args.decode:
            if world > 1 or args.impl != "ours":
                raise SystemExit("--decode: one GPU, --impl ours only")
            return run_decode(args, rank, local)
        if args.packed:
            if world > 1 or args.impl != "ours":
                raise SystemExit("--packed: one GPU, --impl ours only")
            return run_packed(args, rank, local)
        if args.impl == "reference":
            return run_reference(args, w, world, rank)
        return run_ours(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

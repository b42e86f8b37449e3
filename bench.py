#!/usr/bin/env python
"""Benchmark of the weight-only quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME|all]

Metric: effective weight GB/s -- algorithmic bytes (packed weight codes +
scales + zeros + activations in + outputs out, each counted once) per second
-- with the fraction of the HBM roofline, and TFLOP/s (2*M*K*N per call).

Default workload: the W8A16 decode GEMV, K = 5120, N = 17408, M in {1, 2, 4}.
One step = one wq_linear call per M on every one of R packed-weight copies,
R chosen so the copies span more than 5x the L2 size.  Every call therefore
streams its weights from HBM (rotation instead of an L2 flush).  The calls
of one M are captured once as a CUDA graph, back to back (as the layers of a
decode step run); a step replays the graphs of every M with CUDA events
recorded between them on the launching stream, so each M's average launch
duration comes from the timed region itself.

With --gpus N > 1 (launched by torchrun) every rank runs the same workload
on its own GPU: the layer needs no exchange step, so this is weak scaling
over replicas.  Time is the maximum over ranks, and the value is the total
over all ranks divided by it.

--impl reference times the CPU oracle (the plain fp64 implementation) on
the host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import wq_inputs as gen  # noqa: E402

DEFAULT_WORKLOAD = "all"
L2_ROTATION_FACTOR = 5
# With several workloads in one step, the copies of a small weight are capped:
# the other workloads stream gigabytes between two steps, so every copy is
# read from HBM once per step all the same.
MAX_COPIES = 64


def workload_names(spec):
    """'all' (every workload, in the order of wq_inputs.WORKLOADS) or one name."""
    if spec == "all":
        return list(gen.WORKLOADS)
    known = list(gen.WORKLOADS) + list(gen.EXTRA_WORKLOADS)
    if spec not in known:
        raise SystemExit(f"unknown workload {spec!r}; choose 'all' or one of {known}")
    return [spec]


# ---------------------------------------------------------------------------
# workload arithmetic (bytes, flops)
# ---------------------------------------------------------------------------

def weight_bytes(bits, K, N, group):
    if bits == 8:
        return N * K + 2 * N
    g = K // group
    return N * K // 2 + 2 * N * g + N * g // 2


def call_bytes(bits, K, N, group, M):
    return weight_bytes(bits, K, N, group) + 2 * M * K + 2 * M * N


def call_flops(K, N, M):
    return 2 * M * K * N


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_over_ranks(value: float, op: str, device=None) -> float:
    """max/sum of a per-rank scalar over all ranks (identity with one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(per_rank_bytes: float, per_rank_seconds: float, device=None):
    """Whole-job throughput: bytes of all ranks over the slowest rank's time."""
    total = reduce_over_ranks(per_rank_bytes, "sum", device)
    tmax = reduce_over_ranks(per_rank_seconds, "max", device)
    return total, tmax, (total / tmax if tmax > 0 else 0.0)


# ---------------------------------------------------------------------------
# measurement helpers
# ---------------------------------------------------------------------------

def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampled every 200 ms in the background while work runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx = float(parts[1]), float(parts[2])
                pw = float(parts[3])
            except ValueError:
                continue
            smax = mx
            if pw > 200:  # under load
                sm.append(clk)
                power.append(pw)
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples_under_load": len(sm), "samples": len(self.lines),
                "power_w_median": statistics.median(power) if power else None}


def profile_traffic(src_file: str, summary_name: str, M: int):
    """DRAM bytes per launch (read + write) of this kernel at this M, from the
    committed ncu summary -- only if it was captured on the current kernel
    source: the summary records a sha256 for every source file it covers
    (the kernel's own file among them), and each must match the file now."""
    path = os.path.join(ROOT, "profiles", summary_name)
    csrc = os.path.join(ROOT, "weight_only_quantized_02_b200", "csrc")
    try:
        lines = [ln.strip().lstrip("- ") for ln in open(path).read().splitlines()]
    except OSError:
        return None
    covered = {}
    for a, b in zip(lines, lines[1:]):
        if a.startswith("source_sha256:") and b.startswith("source:"):
            covered[os.path.basename(b.split(":", 1)[1].strip().strip("`"))] = a.split(":", 1)[1].strip()
    if src_file not in covered:
        return None
    for name, sha in covered.items():
        try:
            if hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest() != sha:
                return None
        except OSError:
            return None
    for line in lines:
        if line.startswith(f"traffic_bytes_per_launch M={M}:"):
            try:
                return float(line.split(":", 1)[1])
            except ValueError:
                return None
    return None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def tuned_shapes(path):
    """(M, K, N, bits, group) of every entry of a dispatcher table file."""
    out = set()
    for line in open(path):
        if line.startswith("#") or "|" not in line:
            continue
        f = line.split("|", 1)[1].split()
        if len(f) >= 6:
            out.add(tuple(int(v) for v in f[1:6]))
    return out


def build_weights(name, device, copies):
    import torch

    import weight_only_quantized_02_b200 as wq
    cfg = gen.workload(name)
    K, N, bits = cfg["K"], cfg["N"], cfg["bits"]
    if cfg.get("direct"):
        q, s = gen.direct_int8(K, N)
        pw0 = wq.wq_pack_int8(torch.from_numpy(q).to(device), torch.from_numpy(s.view(np.int16)).to(device))
    else:
        W = torch.from_numpy(gen.W_f32(0, N, K)).to(device)
        if bits == 8:
            q, s = wq.wq_quantize_int8(W)
            pw0 = wq.wq_pack_int8(q, s)
        else:
            q, s, z = wq.wq_quantize_int4(W)
            pw0 = wq.wq_pack_int4(q, s, z)
        del W, q, s
    pws = [pw0]
    for _ in range(copies - 1):
        pws.append(wq.PackedWeight(pw0.wq.clone(), pw0.scales.clone(),
                                   None if pw0.zeros is None else pw0.zeros.clone(), pw0.bits, pw0.K, pw0.N,
                                   pw0.group))
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return cfg, pws


KERNELS = {0: ("gemv_sk", "wq_gemv_sk.cu"), 1: ("gemm", "wq_gemm.cu"), 2: ("gemv_rb", "wq_gemv.cu"),
           3: ("gemm_sk", "wq_gemm_sk.cu"), 4: ("gemm_i8", "wq_gemm_i8.cu"), 5: ("gemv_i8", "wq_gemv_i8.cu"),
           6: ("gemm_w4", "wq_gemm_w4.cu")}


def kernel_name(variant, bits):
    return KERNELS[variant][0] + f"_w{bits}"


def kernel_file(variant, bits):
    """Source file of a variant's kernel (the integer path has one per format)."""
    if variant == 4 and bits == 4:
        return "wq_gemm_i4.cu"
    return KERNELS[variant][1]


def bench_ours(args, device, rank, world):
    """Every (workload, M) of the run in one timed region: a step replays,
    for each workload and each M, one CUDA graph of that M's calls on every
    weight copy, with CUDA events between the graphs."""
    import torch

    import weight_only_quantized_02_b200 as wq
    names = workload_names(args.workload)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    works = []  # one dict per workload
    for name in names:
        cfg0 = gen.workload(name)
        K, N, bits, group = cfg0["K"], cfg0["N"], cfg0["bits"], cfg0["group"]
        Ms = list(args.ms) if args.ms else list(cfg0["Ms"])
        wbytes = weight_bytes(bits, K, N, group)
        copies = max(2, math.ceil(L2_ROTATION_FACTOR * l2 / wbytes))
        if len(names) > 1:
            copies = min(copies, MAX_COPIES)
        cfg, pws = build_weights(name, device, copies)
        works.append(dict(name=name, K=K, N=N, bits=bits, group=group, Ms=Ms, copies=copies, pws=pws))
    ws_need = max(wq.wq_workspace_bytes(max(w["Ms"]), w["K"], w["N"], 32) for w in works)
    ws = torch.zeros(ws_need, dtype=torch.uint8, device=device)
    wq.wq_set_workspace(ws)
    for w in works:
        w["xs"] = {M: torch.from_numpy(gen.x_bf16(M, w["K"]).view(np.int16)).view(torch.bfloat16).to(device)
                   for M in w["Ms"]}
        w["ys"] = {M: torch.empty((M, w["N"]), dtype=torch.bfloat16, device=device) for M in w["Ms"]}

    # the dispatcher's measured choice (the load-time tuning of the split_k
    # auto-tune in Mit han lab Llm awq Kernel Selection Thresholds), untimed;
    # shapes the tuning file already holds are loaded, the others tuned
    have = set()
    if args.tuning_file and os.path.exists(args.tuning_file):
        if wq.wq_load_tuning(args.tuning_file) != 0:
            raise RuntimeError("unreadable tuning file " + args.tuning_file)
        have = tuned_shapes(args.tuning_file)
    tuned_any = False
    for w in works:
        K, N, bits, group = w["K"], w["N"], w["bits"], w["group"]
        for M in w["Ms"]:
            key = (M, K, N, bits, group)
            if args.choice is not None:
                # one fixed (variant, split): a single kernel to profile
                wq.wq_set_choice(M, K, N, bits, group, args.choice[0], args.choice[1])
            elif args.tune and key not in have:
                wq.wq_tune(w["xs"][M], w["pws"][0], w["ys"][M], warmup=2, iters=7)
                tuned_any = True
        w["choices"] = {M: wq.wq_get_choice(M, K, N, bits, group) for M in w["Ms"]}
    if tuned_any and args.tuning_file:
        wq.wq_save_tuning(args.tuning_file)

    stream = torch.cuda.Stream(device)
    P = max(1, min(args.steps, 64))  # event sets: per-launch times of the last P steps

    # warm the launch path before capture (attributes, tensor maps)
    with torch.cuda.stream(stream):
        for w in works:
            for M in w["Ms"]:
                for c in range(w["copies"]):
                    wq.wq_linear(w["xs"][M], w["pws"][c], y=w["ys"][M], stream=stream)
    torch.cuda.synchronize(device)

    # one CUDA graph per (workload, M): its calls on every weight copy back to
    # back (as the layers of a decode step run, the next launch may start
    # while the previous one drains); events recorded on the stream between
    # the graphs give each one's average launch duration inside the timed
    # region
    graphs, points = [], []
    for w in works:
        for M in w["Ms"]:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for c in range(w["copies"]):
                    wq.wq_linear(w["xs"][M], w["pws"][c], y=w["ys"][M], stream=stream)
            graphs.append(g)
            points.append((w, M))
    torch.cuda.synchronize(device)
    evsets = [[torch.cuda.Event(enable_timing=True) for _ in range(len(graphs) + 1)] for _ in range(P)]

    def run_step(s):
        evs = evsets[s % P] if s is not None else None
        if evs is not None:
            evs[0].record(stream)
        for i, g in enumerate(graphs):
            g.replay()
            if evs is not None:
                evs[i + 1].record(stream)

    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(vis.split(",")[device.index] if vis else device.index)
    sampler.start()
    with torch.cuda.stream(stream):
        # device warm-up before measuring (as the page's timing protocol does)
        t0 = time.time()
        i = 0
        while time.time() - t0 < args.soak:
            run_step(None)
            i += 1
            if i % 4 == 0:
                torch.cuda.synchronize(device)
        for s in range(args.warmup):
            run_step(s)
    torch.cuda.synchronize(device)

    barrier(device)
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for s in range(args.steps):
            run_step(s)
        end.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop()
    elapsed_s = start.elapsed_time(end) / 1000.0

    # per-launch durations from the timed region (its last P steps): each
    # graph's time over its launches
    per_call_us = [[] for _ in points]
    for evs in evsets[:min(P, args.steps)]:
        for i, (w, M) in enumerate(points):
            per_call_us[i].append(evs[i].elapsed_time(evs[i + 1]) * 1000.0 / w["copies"])

    def pbytes(w, M):
        return call_bytes(w["bits"], w["K"], w["N"], w["group"], M)

    step_bytes = sum(pbytes(w, M) * w["copies"] for w, M in points)
    step_flops = sum(call_flops(w["K"], w["N"], M) * w["copies"] for w, M in points)
    total_bytes, tmax, value_bps = aggregate(step_bytes * args.steps, elapsed_s, device)
    peaks = read_peaks()

    per_shape = []
    for i, (w, M) in enumerate(points):
        us = statistics.mean(per_call_us[i])
        b, f = pbytes(w, M), call_flops(w["K"], w["N"], M)
        v, sp = w["choices"][M]
        t_roof = max(b / (peaks["hbm_gbs"] * 1e3), f / (peaks["bf16_tflops"] * 1e6))
        per_shape.append({
            "workload": w["name"], "M": M, "K": w["K"], "N": w["N"], "bits": w["bits"], "group": w["group"],
            "variant": kernel_name(v, w["bits"]), "split": sp, "calls_per_step": w["copies"],
            "us_per_call": round(us, 3), "gbs": round(b / us / 1e3, 1),
            "hbm_frac_of_measured": round(b / us / 1e3 / peaks["hbm_gbs"], 4),
            "hbm_frac_of_8tbs": round(b / us / 1e3 / 8000.0, 4),
            "tflops": round(f / us / 1e6, 3),
            "bound": "tensor" if f / (peaks["bf16_tflops"] * 1e6) > b / (peaks["hbm_gbs"] * 1e3) else "hbm",
            "roofline_us": round(t_roof, 3), "roofline_frac": round(t_roof / us, 4),
        })

    # dominant kernel: the (workload, M) with the largest share of device time
    shares = [statistics.mean(per_call_us[i]) * w["copies"] for i, (w, M) in enumerate(points)]
    idom = max(range(len(points)), key=lambda i: shares[i])
    wdom, Mdom = points[idom]
    dom = per_shape[idom]
    vdom = wdom["choices"][Mdom][0]
    kfile = kernel_file(vdom, wdom["bits"])
    summary = f"{dom['variant']}_{wdom['name']}.md"
    traffic = profile_traffic(kfile, summary, Mdom)
    b_dom, f_dom = pbytes(wdom, Mdom), call_flops(wdom["K"], wdom["N"], Mdom)
    us_dom = statistics.mean(per_call_us[idom])
    if dom["bound"] == "tensor":
        achieved = f_dom / (us_dom * 1e-6) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": traffic,
                    "algorithmic_flops_per_launch": f_dom,
                    "peak_source": peaks["source"] + " (MEASURED_PEAKS.json bf16_tflops, burst)"}
    else:
        achieved = b_dom / (us_dom * 1e-6) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                    "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)",
                    "frac_of_8tbs": round(achieved / 8000.0, 4)}
    roofline.update({"kernel": f"{dom['variant']} {wdom['name']} M={Mdom} split={dom['split']}",
                     "share_of_step": round(shares[idom] / sum(shares), 4),
                     "traffic_source": f"profiles/{summary}" if traffic is not None else None,
                     "algorithmic_bytes_per_launch": b_dom})

    topk = bench_topk(args, device, works, stream, per_call_us, points)
    e2e = bench_e2e(args, device, works, stream)
    wq.wq_set_workspace(None)
    return {
        "value": value_bps / 1e9, "ms_per_step": tmax / args.steps * 1e3, "per_shape": per_shape,
        "roofline": roofline, "clocks": clocks, "e2e": e2e, "works": works, "topk": topk,
        "gpu_launches": args.steps * sum(w["copies"] for w, _ in points),
        "tflops": step_flops * args.steps * world / tmax / 1e12, "l2_bytes": l2,
    }


TOPK_K = 64


def bench_topk(args, device, works, stream, per_call_us, points):
    """The vocabulary head's top-k (wq_linear_topk, k = 64) on every
    vocabulary-sized workload: the per-call time of the logits plus the
    selection, beside the plain layer's time from the timed region."""
    import torch

    import weight_only_quantized_02_b200 as wq
    out = []
    for w in works:
        if w["N"] < 100000:
            continue
        for M in w["Ms"]:
            ws = torch.zeros(wq.wq_topk_workspace_bytes(M, w["N"], TOPK_K), dtype=torch.uint8, device=device)
            with torch.cuda.stream(stream):
                for c in range(w["copies"]):
                    wq.wq_linear_topk(w["xs"][M], w["pws"][c], TOPK_K, ws, stream=stream)
            torch.cuda.synchronize(device)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for c in range(w["copies"]):
                    wq.wq_linear_topk(w["xs"][M], w["pws"][c], TOPK_K, ws, stream=stream)
            reps = max(3, min(args.steps, 20))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                g.replay()
                a.record(stream)
                for _ in range(reps):
                    g.replay()
                b.record(stream)
            torch.cuda.synchronize(device)
            us = a.elapsed_time(b) * 1000.0 / (reps * w["copies"])
            i = next(j for j, (pw_, pm) in enumerate(points) if pw_ is w and pm == M)
            plain = statistics.mean(per_call_us[i])
            out.append({"workload": w["name"], "M": M, "k": TOPK_K, "us_per_call": round(us, 3),
                        "layer_us_per_call": round(plain, 3), "selection_us": round(us - plain, 3)})
            del g, ws
    return out


def bench_e2e(args, device, works, stream):
    """Same metric through the public call with host buffers.  Every step
    copies its inputs (the activations of every workload and M) in from
    pinned host memory, runs its calls, and copies every call's output back
    to pinned host memory: each output on a side stream as soon as its call
    is done, so the copies overlap the following calls, as a decode runtime
    overlaps them.  The step is captured once as a CUDA graph (fork and join
    included); every replay performs every copy."""
    import torch

    import weight_only_quantized_02_b200 as wq
    calls = [(wi, M, c) for wi, w in enumerate(works) for M in w["Ms"] for c in range(w["copies"])]
    hx = {(wi, M): works[wi]["xs"][M].cpu().pin_memory() for wi, w in enumerate(works) for M in w["Ms"]}
    dx = {k: torch.empty_like(works[k[0]]["xs"][k[1]]) for k in hx}
    hy = {k: torch.empty((k[1], works[k[0]]["N"]), dtype=torch.bfloat16).pin_memory() for k in calls}
    dy = {k: torch.empty((k[1], works[k[0]]["N"]), dtype=torch.bfloat16, device=device) for k in calls}
    side = torch.cuda.Stream(device)
    steps = max(1, min(args.steps, args.e2e_steps))

    def step():
        for k in hx:
            dx[k].copy_(hx[k], non_blocking=True)
        for k in calls:
            wi, M, c = k
            wq.wq_linear(dx[(wi, M)], works[wi]["pws"][c], y=dy[k], stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            side.wait_event(done)
            with torch.cuda.stream(side):
                hy[k].copy_(dy[k], non_blocking=True)
        stream.wait_stream(side)

    with torch.cuda.stream(stream):
        step()  # eager once: attributes, tensor maps
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        for _ in range(max(1, min(args.warmup, 5))):
            g.replay()
    torch.cuda.synchronize(device)
    barrier(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(steps):
            g.replay()
        b.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    t = a.elapsed_time(b) / 1000.0
    # the outputs that came back match the device results of the last replay
    for k in (calls[0], calls[-1]):
        if not torch.equal(hy[k].view(torch.int16), dy[k].cpu().view(torch.int16)):
            raise RuntimeError("end-to-end outputs differ from the device results")
    step_bytes = sum(call_bytes(works[wi]["bits"], works[wi]["K"], works[wi]["N"], works[wi]["group"], M)
                     for wi, M, _ in calls)
    total, tmax, v = aggregate(step_bytes * steps, t, device)
    return {"value": round(v / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": sum(2 * k[1] * works[k[0]]["K"] for k in hx),
            "d2h_bytes_per_step": sum(2 * M * works[wi]["N"] for wi, M, _ in calls), "steps": steps,
            "note": "wq_linear with pinned host buffers: the step's activations copied in, every call's output "
                    "copied out on a side stream overlapping the next calls; the step replayed as one CUDA graph"}


class OracleSample:
    """The CPU oracle as it stands on a bounded sample of one workload: every
    M of one step on the first `rows` output channels."""

    def __init__(self, name, rows=None):
        import oracle
        self.oracle = oracle
        cfg = gen.workload(name)
        self.name = name
        self.K, self.N, self.bits, self.group = cfg["K"], cfg["N"], cfg["bits"], cfg["group"]
        self.Ms = list(cfg["Ms"])
        self.direct = cfg.get("direct", False)
        self.xs = {M: gen.x_bf16(M, self.K) for M in self.Ms}
        self.set_rows(rows or min(self.N, 256))

    def set_rows(self, rows):
        rows = max(16, min(self.N, int(rows)) // 16 * 16)
        self.rows = rows
        if self.direct:
            q, s = gen.direct_int8(self.K, self.N)
            self.c = (q[:rows], s[:rows])
        else:
            W = gen.W_f32(0, rows, self.K)
            self.c = self.oracle.quant_int8(W) if self.bits == 8 else self.oracle.quant_int4(W)

    def run(self):
        for M in self.Ms:
            if self.bits == 8:
                self.oracle.linear_int8(self.xs[M], self.c[0], self.c[1])
            else:
                self.oracle.linear_int4(self.xs[M], self.c[0], self.c[1], self.c[2])

    def bytes(self):
        """Algorithmic bytes of one pass, scaled to the sampled channels."""
        return sum(call_bytes(self.bits, self.K, self.N, self.group, M) for M in self.Ms) * self.rows / self.N

    def describe(self):
        return f"{self.name}: {self.rows} of {self.N} output channels, M in {self.Ms}"


def sized_samples(names, budget_s):
    """One OracleSample per workload, each sized to about budget_s / len(names)
    seconds of oracle work per pass (at most the whole layer)."""
    each = budget_s / max(1, len(names))
    out = []
    for name in names:
        smp = OracleSample(name)
        t0 = time.perf_counter()
        smp.run()
        tp = time.perf_counter() - t0
        smp.set_rows(smp.rows * each / max(tp, 1e-6))
        out.append(smp)
    return out


def cpu_baseline(names, budget_s=16.0):
    """The CPU oracle as it stands, on the host cores, over a bounded sample
    of the run's workloads: every M of each workload on a contiguous block of
    output channels sized to about budget_s seconds of work in all, passed
    over again until about budget_s / 2 seconds have gone."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    smps = sized_samples(names, budget_s)
    reps, t = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or (t < budget_s / 2 and reps < 10000):
        for smp in smps:
            smp.run()
        reps += 1
        t = time.perf_counter() - t0
    b = sum(smp.bytes() for smp in smps) * reps
    return {"value": round(b / t / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": round(t, 3),
            "sample": "; ".join(smp.describe() for smp in smps) + f"; one weight copy, {reps} pass(es); "
                      "bytes scaled to the sampled channels"}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def bench_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    names = workload_names(args.workload)
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    # size each step so the whole run stays within about 90 s of CPU time
    smps = sized_samples(names, 90.0 / max(1, args.steps + args.warmup))

    def step():
        for smp in smps:
            smp.run()

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    t = time.perf_counter() - t0
    value = sum(smp.bytes() for smp in smps) * args.steps / t / 1e9
    sample = "; ".join(smp.describe() for smp in smps) + " per step"
    return {
        "metric": METRIC, "impl": "reference",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(run_config(names), parallelism="cpu oracle, rank 0 only"),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


METRIC = "effective weight GB/s (W8A16/W4A16 linear, algorithmic bytes)"


def run_config(names):
    """The run's workloads, named by what they are."""
    ws = []
    for name in names:
        c = gen.workload(name)
        ws.append({"name": name, "bits": c["bits"], "group": c["group"], "K": c["K"], "N": c["N"],
                   "Ms": list(c["Ms"])})
    label = ("all five workloads: " if len(names) == len(gen.WORKLOADS) else "") + ", ".join(names)
    return {"workload": label, "workloads": ws}


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed device warm-up")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-tune", dest="tune", action="store_false",
                    help="time the dispatcher's untuned default instead of its tuned choice")
    ap.add_argument("--tuning-file", default=None,
                    help="load this dispatcher table instead of tuning (saved there after tuning if absent)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ms", type=lambda v: [int(t) for t in v.split(",")], default=None,
                    help="comma-separated subset of the workload's M values")
    ap.add_argument("--choice", type=lambda v: tuple(int(t) for t in v.split(":")), default=None,
                    help="VARIANT:SPLIT used for every M instead of tuning (e.g. to profile one kernel)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        line = bench_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    names = workload_names(args.workload)
    r = bench_ours(args, device, rank, world)
    if rank == 0:
        conf = run_config(names)
        conf.update({
            "weight_copies": {w["name"]: w["copies"] for w in r["works"]},
            "l2": f"inputs larger than L2: each workload's weights rotated over copies spanning > "
                  f"{L2_ROTATION_FACTOR}x the {r['l2_bytes'] // 2**20} MiB L2 (at most {MAX_COPIES} copies of a "
                  f"small weight when other workloads stream between steps); no flush",
            "parallelism": "replicas" if world > 1 else "single GPU",
            "timing": "one CUDA graph per (workload, M) of its calls back to back, CUDA events between the "
                      "graphs, max over ranks"})
        line = {
            "metric": METRIC,
            "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02^2) weights quantized on device; the direct "
                    "W8A16 case draws its codes and scales)",
            "config": conf,
            "tflops": round(r["tflops"], 2), "per_shape": r["per_shape"], "roofline": r["roofline"],
            "clocks": r["clocks"], "e2e": r["e2e"], "gpu_launches": r["gpu_launches"], "topk": r["topk"],
            "dispatch": {f"{w['name']} M={M}": list(w["choices"][M]) for w in r["works"] for M in w["Ms"]},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(names)
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

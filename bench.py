#!/usr/bin/env python
"""Benchmark of the any4 linear layer on B200.

Workload: the linear stack of Llama-3-8B (32 decoder layers x {q 4096x4096,
k 1024x4096, v 1024x4096, o 4096x4096, gate 14336x4096, up 14336x4096,
down 4096x14336}), any4 with group 128, run back to back at M = 1 and then at
M = 16. One step = both passes = 448 any4_linear calls. Weights are synthetic
any4 tensors (one drawn set per distinct shape, packed once, copied to 32
distinct device buffers: 3.76 GB, far above the 126 MB L2, so every call
streams its weights from HBM). Activations are per call.

Output: one JSON line (rank 0). ``value`` is the aggregate algorithmic HBM
throughput in GB/s (packed indices, LUTs, alpha/beta, x and y bytes of every
call of every rank / the max over ranks of the step time).

``--impl reference`` times the CPU oracle on the same workload and metric,
each step a bounded sample of the stack.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

GROUP = 128
# DRAM bytes per algorithmic byte of the linear kernel, from an ncu capture of
# one 14336x4096, M=1, G=128 launch of the current kernel (--set full,
# --clock-control none): dram__bytes_read.sum 31,696,384 B +
# dram__bytes_write.sum 0 B for 31,690,752 algorithmic bytes.
DRAM_PER_ALGO_BYTE = 31_696_384 / 31_690_752
LAST_CAPTURE_NOTE = ("null: no capture of the current kernel")
LAYERS = 32
MS = (1, 16)
FALLBACK_HBM_GBS = 6650.0


def algorithmic_bytes(m: int, n: int, k: int, g: int) -> int:
    return n * k // 2 + n * (k // g) * 4 + n * 32 + m * k * 2 + m * n * 2


def stack_calls():
    """(m, layer, shape) for one step, in execution order."""
    return [(m, layer, sh) for m in MS for layer in range(LAYERS) for sh in synth.LLAMA3_8B_LAYER]


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period: float = 0.02):
        self.index, self.period = index, period
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()
        self.ok = True
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.ok = False
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml_unavailable"],
                    "samples": 0}
        names = [v for b, v in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float, calls=None, threads: int | None = None):
    """Time the oracle (as it stands) on the stack's calls, in order, for about
    ``budget_s`` seconds of work, with its BLAS limited to ``threads`` (all the
    cores this process may run on when None). The bit-exact fp64 dequant is
    single-threaded NumPy; the fp64 matmul uses the BLAS threads."""
    import oracle
    from threadpoolctl import threadpool_limits
    cores = host_cores() if threads is None else threads
    calls = calls or stack_calls()
    cache = {}
    done_bytes, t_total, count = 0, 0.0, 0
    with threadpool_limits(limits=cores):
        for (m, layer, sh) in calls:
            key = (sh.n, sh.k)
            if key not in cache:
                idx, lut, a, b = synth.random_any4(sh.n, sh.k, GROUP, 0, layer=sh.name)
                cache[key] = oracle.Any4Tensors(idx, lut, a, b, GROUP)
            s = synth.channel_scale(sh.k, 0, layer=sh.name)
            x = synth.activations_bf16(m, s, layer, layer=sh.name)
            t0 = time.perf_counter()
            oracle.linear(x, cache[key])
            t_total += time.perf_counter() - t0
            done_bytes += algorithmic_bytes(m, sh.n, sh.k, GROUP)
            count += 1
            if t_total >= budget_s:
                break
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": int(cores),
            "kind": "oracle", "seconds": t_total, "calls": count,
            "sample": f"first {count} of {len(calls)} calls of one step (M=1 pass first), "
                      f"{t_total:.1f} s: fp64 bit-exact dequant (single-threaded numpy) + "
                      f"fp64 matmul ({cores} BLAS threads)"}


def cpu_baselines(budget_s: float) -> dict:
    """The oracle on all host cores, plus the same on one core."""
    full = cpu_baseline(budget_s)
    one = cpu_baseline(budget_s / 2, threads=1)
    return {**full, "one_core": {k: one[k] for k in ("value", "unit", "cores", "sample")}}


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take part; NCCL on GPUs, gloo on CPU)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_config(world: int) -> dict:
    """The workload of the JSON line (both arms)."""
    return {"workload": "llama3_8b_linear_stack", "layers": LAYERS,
            "linears_per_layer": len(synth.LLAMA3_8B_LAYER), "ms": list(MS),
            "group": GROUP, "calls_per_step": len(stack_calls()),
            "l2": "inputs larger than L2: 3.76 GB of distinct packed weights per step",
            "parallelism": f"replicas x{world}"}


def result_line(world: int, steps: int, warmup: int, ms_step: float, step_bytes: int, n_calls: int,
                per_m: dict, peak: float, peak_kind: str, clocks, e2e, cpu, dominant: dict | None = None) -> dict:
    """The JSON line of one run: whole-job throughput over all ranks (weak
    scaling: every rank runs the full step) and the roofline of the dominant
    kernel. ``dominant`` = {"bytes", "ms", "launches"}: that kernel's calls of
    one step timed on their own (algorithmic bytes, device ms, launches);
    without it the whole step stands in for it."""
    if dominant is None:
        dominant = {"bytes": step_bytes, "ms": ms_step, "launches": n_calls}
    achieved = dominant["bytes"] / (dominant["ms"] * 1e6)
    per_launch = dominant["bytes"] / dominant["launches"]
    return {
        "metric": "any4_linear achieved HBM GB/s (algorithmic bytes)",
        "value": step_bytes * world / (ms_step * 1e6), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(world),
        "us_per_call": ms_step * 1e3 / n_calls,
        "by_m": per_m,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": (DRAM_PER_ALGO_BYTE * per_launch if DRAM_PER_ALGO_BYTE is not None else None),
                     "traffic_note": ("dram bytes per launch: ncu dram__bytes_read+write of one "
                                      "14336x4096 M=1 launch over its algorithmic bytes, times "
                                      "this kernel's mean algorithmic bytes per launch"
                                      if DRAM_PER_ALGO_BYTE is not None else LAST_CAPTURE_NOTE),
                     "peak_source": f"{peak_kind} hbm_gbs", "kernel": "linear_kernel",
                     "launches_per_step": dominant["launches"],
                     "note": ("achieved = the kernel's algorithmic bytes per launch over its mean launch "
                              "time, from its own calls of the step replayed back to back; the k/v calls "
                              "and the M=1 q/o calls run linear_small_kernel (M=1) or "
                              "linear_regt_kernel (M=16)")},
        "gpu_launches": n_calls * steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }


def run_reference(args, rank: int, world: int):
    """The oracle on the host cores, rank 0 only: each step is a bounded
    sample of the stack's calls (in order); ``value`` is the algorithmic bytes
    of the sampled calls over the time they took, ``ms_per_step`` the measured
    time of one sampled step."""
    if rank != 0:
        return
    calls = stack_calls()
    per_step_budget = max(0.5, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(per_step_budget, calls)
        if i >= args.warmup:
            vals.append(r)
    seconds = sum(v["seconds"] for v in vals)
    value = sum(v["value"] * v["seconds"] for v in vals) / seconds
    line = {"impl": "reference", "metric": "any4_linear achieved HBM GB/s (algorithmic bytes)",
            "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": seconds * 1e3 / len(vals), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(1),
            "step": (f"a bounded sample of the stack: the first {vals[-1]['calls']} of {len(calls)} "
                     f"calls, about {per_step_budget:.1f} s of oracle work per step"),
            "cpu_baseline": {**vals[-1], "value": value},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# Shapes of the per-shape lines: the Llama-3-8B MLP shapes the 70 % target is
# set on, then the attention projections.
BY_SHAPE = (("gate/up", 14336, 4096), ("down", 4096, 14336), ("q/o", 4096, 4096), ("k/v", 1024, 4096))
L2_BYTES = 126 * 2 ** 20


def time_by_shape(a4, dev, peak: float, calls: int = 200) -> dict:
    """µs per call of each shape at M = 1 and 16: ``calls`` back-to-back
    any4_linear launches replayed from one CUDA graph, rotating over enough
    distinct copies of the packed weight (>= 3x the L2 size) that every call
    reads its weight from HBM; CUDA events around the replay."""
    import torch
    out = {}
    for name, n, k in BY_SHAPE:
        idx, lut, al, be = synth.random_any4(n, k, GROUP, 0, layer="shape_" + name)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)
        base = a4.any4_pack(t(idx), t(lut), t(al), t(be), GROUP)
        wbytes = algorithmic_bytes(1, n, k, GROUP)
        copies = max(2, -(-3 * L2_BYTES // wbytes))
        packs = [base] + [base.clone() for _ in range(copies - 1)]
        for m in MS:
            s = synth.channel_scale(k, 0, layer="shape_" + name)
            x = torch.from_numpy(synth.activations_bf16(m, s, 7, layer="shape_" + name).view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            ws = torch.zeros(a4.any4_linear_workspace_bytes(m, n, k, GROUP), dtype=torch.uint8, device=dev)
            side = torch.cuda.Stream(dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                for i in range(4):
                    a4.any4_linear(x, packs[i % copies], n, k, GROUP, out=y, workspace=ws)
            torch.cuda.current_stream(dev).wait_stream(side)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(calls):
                    a4.any4_linear(x, packs[i % copies], n, k, GROUP, out=y, workspace=ws)
            g.replay()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            us = e0.elapsed_time(e1) * 1e3 / calls
            b = algorithmic_bytes(m, n, k, GROUP)
            out[f"{name} {n}x{k} M={m}"] = {"us_per_call": us, "GB/s": b / (us * 1e3),
                                             "frac": b / (us * 1e3) / peak, "weight_copies": copies}
            del g
        del packs, base
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import learned_bit_lut_b200 as a4

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)

    calls = stack_calls()
    # packed weights: one drawn set per distinct shape, copied to 32 layers
    packed = {}
    for sh in synth.LLAMA3_8B_LAYER:
        idx, lut, al, be = synth.random_any4(sh.n, sh.k, GROUP, 0, layer=sh.name)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)
        base = a4.any4_pack(t(idx), t(lut), t(al), t(be), GROUP)
        for layer in range(LAYERS):
            packed[(layer, sh.name)] = base if layer == 0 else base.clone()
    del base
    # activations and outputs per call (one flat device buffer each)
    xoff, yoff, xo, yo = [], [], 0, 0
    for (m, layer, sh) in calls:
        xoff.append(xo); yoff.append(yo)
        xo += m * sh.k
        yo += m * sh.n
    x_host = np.empty(xo, dtype=np.uint16)
    for i, (m, layer, sh) in enumerate(calls):
        s = synth.channel_scale(sh.k, 0, layer=sh.name)
        x_host[xoff[i]:xoff[i] + m * sh.k] = synth.activations_bf16(m, s, 1000 + layer, layer=sh.name).ravel()
    x_dev = torch.from_numpy(x_host.view(np.int16)).to(dev).view(torch.bfloat16)
    y_dev = torch.empty(yo, dtype=torch.bfloat16, device=dev)
    ws_need = max(a4.any4_linear_workspace_bytes(m, sh.n, sh.k, GROUP) for m, _, sh in calls)
    ws = torch.zeros(ws_need, dtype=torch.uint8, device=dev)

    def issue(sel):
        for i in sel:
            m, layer, sh = calls[i]
            a4.any4_linear(x_dev[xoff[i]:xoff[i] + m * sh.k].view(m, sh.k),
                           packed[(layer, sh.name)], sh.n, sh.k, GROUP,
                           out=y_dev[yoff[i]:yoff[i] + m * sh.n].view(m, sh.n), workspace=ws)

    sel = {mm: [i for i, c in enumerate(calls) if c[0] == mm] for mm in MS}
    graphs = {}
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        issue(range(len(calls)))          # eager warm-up before capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    for mm in MS:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            issue(sel[mm])
        graphs[mm] = g

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, steps):
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    def step():
        for mm in MS:
            graphs[mm].replay()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    with sampler:
        ms_total = timed(step, args.steps)
    ms_step = ms_total / args.steps
    per_m = {}
    for mm in MS:
        for _ in range(2):
            graphs[mm].replay()
        ms_m = timed(graphs[mm].replay, args.steps) / args.steps
        b = sum(algorithmic_bytes(mm, sh.n, sh.k, GROUP) for m, _, sh in calls if m == mm)
        per_m[str(mm)] = {"us_per_call": ms_m * 1e3 / len(sel[mm]), "GB/s": b / (ms_m * 1e6)}

    # the dominant kernel (the shared-table decode, linear_kernel) on its own:
    # its calls of the step, replayed back to back from their own graphs
    kern = [a4.any4_linear_kernel(m, sh.n, sh.k, GROUP) for m, _, sh in calls]
    dom = {"bytes": 0, "ms": 0.0, "launches": 0}
    for mm in MS:
        ids = [i for i in sel[mm] if kern[i] == "shared_tables"]
        if not ids:
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            issue(ids)
        for _ in range(2):
            g.replay()
        dom["ms"] += timed(g.replay, args.steps) / args.steps
        dom["bytes"] += sum(algorithmic_bytes(calls[i][0], calls[i][2].n, calls[i][2].k, GROUP) for i in ids)
        dom["launches"] += len(ids)
        del g
    if dom["launches"] == 0:
        dom = None

    step_bytes = sum(algorithmic_bytes(m, sh.n, sh.k, GROUP) for m, _, sh in calls)
    peak, peak_kind = read_peaks()
    by_shape = None if args.no_shapes else time_by_shape(a4, dev, peak)

    # end to end through the Python API: pinned host x in, y out, every step.
    # Per group of 4 layers (28 calls), x goes in on one copy stream and y
    # comes out on another, so the transfers overlap the other groups' calls
    # (few groups: the stream and event bookkeeping costs host time per group).
    e2e = None
    if not args.no_e2e:
        x_pin = torch.from_numpy(x_host.view(np.int16)).pin_memory()
        y_pin = torch.empty(yo, dtype=torch.int16).pin_memory()
        x_in = torch.empty_like(x_dev)
        y_out = torch.empty_like(y_dev)
        per_group = 4 * len(synth.LLAMA3_8B_LAYER)
        groups = [(a, min(a + per_group, len(calls))) for a in range(0, len(calls), per_group)]
        span = lambda off, i: off[i] + calls[i][0] * (calls[i][2].k if off is xoff else calls[i][2].n)
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        # each call's activation and output views, held like a model's buffers
        views = [(x_in[xoff[i]:xoff[i] + m * sh.k].view(m, sh.k), packed[(layer, sh.name)], sh.n, sh.k,
                  y_out[yoff[i]:yoff[i] + m * sh.n].view(m, sh.n)) for i, (m, layer, sh) in enumerate(calls)]

        def e2e_step():
            cur = torch.cuda.current_stream(dev)
            h2d.wait_stream(cur)
            d2h.wait_stream(cur)
            ready = []
            with torch.cuda.stream(h2d):
                for a, b in groups:
                    x_in.view(torch.int16)[xoff[a]:span(xoff, b - 1)].copy_(
                        x_pin[xoff[a]:span(xoff, b - 1)], non_blocking=True)
                    ready.append(torch.cuda.Event())
                    ready[-1].record(h2d)
            for (a, b), ev in zip(groups, ready):
                cur.wait_event(ev)
                for xv, pk, n, k, yv in views[a:b]:
                    a4.any4_linear(xv, pk, n, k, GROUP, out=yv, workspace=ws)
                done = torch.cuda.Event()
                done.record(cur)
                d2h.wait_event(done)
                with torch.cuda.stream(d2h):
                    y_pin[yoff[a]:span(yoff, b - 1)].copy_(
                        y_out.view(torch.int16)[yoff[a]:span(yoff, b - 1)], non_blocking=True)
            cur.wait_stream(h2d)
            cur.wait_stream(d2h)

        for _ in range(2):
            e2e_step()
        e2e_steps = max(3, min(args.steps, 20))
        ms_e2e = timed(e2e_step, e2e_steps) / e2e_steps
        e2e = {"value": step_bytes * world / (ms_e2e * 1e6), "unit": "GB/s",
               "h2d_bytes_per_step": int(x_host.nbytes), "d2h_bytes_per_step": int(yo * 2),
               "ms_per_step": ms_e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baselines(args.cpu_seconds)

    if rank == 0:
        line = result_line(world, args.steps, args.warmup, ms_step, step_bytes, len(calls), per_m,
                           peak, peak_kind, sampler.summary(), e2e, cpu, dom)
        line["by_shape"] = by_shape
        print(json.dumps(line), flush=True)
    for g in graphs.values():
        del g


def run_one(n: int, k: int, m: int, g: int, calls: int = 8):
    """A few any4_linear calls of one shape (4 weight copies in rotation), for
    profiler captures of a single launch."""
    import torch

    import learned_bit_lut_b200 as a4
    dev = torch.device("cuda:0")
    idx, lut, al, be = synth.random_any4(n, k, g, 0, layer="one")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)
    ws = [a4.any4_pack(t(idx), t(lut), t(al), t(be), g) for _ in range(4)]
    s = synth.channel_scale(k, 0, layer="one")
    x = torch.from_numpy(synth.activations_bf16(m, s, 0, layer="one").view(np.int16)).to(dev).view(torch.bfloat16)
    for i in range(calls):
        a4.any4_linear(x, ws[i % 4], n, k, g)
    torch.cuda.synchronize()
    print(f"ran {calls} calls of N={n} K={k} M={m} G={g}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-shapes", action="store_true", help="skip the per-shape lines")
    ap.add_argument("--shapes", action="store_true", help="only the per-shape lines (1 GPU)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--one", type=int, nargs=4, metavar=("N", "K", "M", "G"),
                    help="only run a few calls of one shape (profiler captures)")
    args = ap.parse_args()
    if args.one:
        run_one(*args.one)
        return
    if args.shapes:
        import torch

        import learned_bit_lut_b200 as a4
        peak, _ = read_peaks()
        print(json.dumps(time_by_shape(a4, torch.device("cuda:0"), peak)), flush=True)
        return
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

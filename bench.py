#!/usr/bin/env python
"""Throughput of the fused Invariant Point Attention core on B200.

One step = one pass of the whole hot path over one batch element of the
long-context workload (L = 4096 residues, 12 heads, 16 scalar channels,
4 query / 8 value points, rank-2 x 128-channel factorised pair
representation): frames applied and augmented operands built (prologue), then
the fused attention pass (core).  Metric: algorithmic TFLOP/s of the fused
core, 2 L^2 H (Dqk + Dv) flops per batch element with Dqk = C + 3 Pq + 1 + R Cz
and Dv = C + 3 Pv + R Cz.

Launch: `python bench.py --gpus N --steps K --warmup W` (N > 1 under
torchrun; every rank runs its own batch element -- weak scaling, no
collective on the data path).  Rank 0 prints one JSON line.
`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from rna_structure_models_b200.synth import GeoDims, IpaDims, geo_inputs, ipa_inputs  # noqa: E402

H, C, PQ, PV, R, CZ = 12, 16, 4, 8, 2, 128
METRIC = "fused IPA attention TFLOP/s and % bf16 tensor-pipe peak at L=4096 (1xB200)"
UNIT = "TFLOP/s"
REF_BUDGET_S = 90.0

# DRAM traffic of one launch of the core kernel (the CTA-pair kernel at this
# workload's R Cz = 256) from an ncu capture, valid only for the kernel source
# it was taken on (sha256 over the sources listed in CORE_SOURCES).
CORE_KERNEL = "ipa_attention_pair_kernel"
CORE_SOURCES = ("ipa_attention_pair.cu", "ipa_epilogue.cuh", "sm100.cuh", "bounds.cuh")
NCU_TRAFFIC = {"kernel_sha256": "e39af46f7b0d460e83ad3fd90dead1e64a41ae5bd9b55cdbea6b70388c2426dd",
               "bytes_per_launch": 29.86e6}


def ipa_flops(B, L, n_valid=None, heads=H, rcz=R * CZ):
    """Algorithmic flops of the fused core (2 per multiply-add)."""
    dqk = C + 3 * PQ + 1 + rcz
    dv = C + 3 * PV + rcz
    pairs = B * L * L if n_valid is None else float(np.sum(np.asarray(n_valid, float) ** 2))
    return 2.0 * pairs * heads * (dqk + dv)


def ipa_bwd_flops(B, L, heads=H, rcz=R * CZ):
    """Algorithmic flops of the gradient pass: the logits again (Dqk), dP
    (Dv), dQ (Dqk), dK (Dqk) and dV (Dv) per (query, key, head)."""
    dqk = C + 3 * PQ + 1 + rcz
    dv = C + 3 * PV + rcz
    return 2.0 * B * L * L * heads * (3 * dqk + 2 * dv)


def host_threads():
    """Cores this process may run on and the BLAS pool size (reported beside
    the CPU oracle timings; the oracle's einsums themselves run on one)."""
    cores = len(os.sched_getaffinity(0))
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=None)
    except Exception:  # noqa: BLE001 -- reported as unknown
        pass
    return cores, blas


def rank_inputs(rank, L):
    """Each rank times its own batch element of the workload (weak scaling):
    same shapes, seed = rank."""
    return ipa_inputs(IpaDims(B=1, L=L, H=H, C=C, Pq=PQ, Pv=PV, R=R, Cz=CZ), seed=rank)


def max_over_ranks(ms, world, dist=None, device="cpu"):
    """The job's time is the slowest rank's (every rank calls this, in the
    same order, also when it has nothing to report)."""
    if world == 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_rank_step, steps, total_ms):
    """Whole-job throughput: all ranks' work over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (total_ms / 1e3) / 1e12


def kernel_sha():
    h = hashlib.sha256()
    for f in CORE_SOURCES:
        h.update(open(os.path.join(ROOT, "rna_structure_models_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x2: "applications_clocks_setting", 0x1: "gpu_idle",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, torch_device):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
            self.ok = True
        except Exception:  # noqa: BLE001 -- clocks are reported as unavailable
            pass

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.001)   # >= 5 samples even in a short (20-step) timed region

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def cpu_oracle_sample(L, seconds, max_rows, seed=0, inp=None):
    """Time the float64 oracle on query-row blocks of the same workload
    (input generation is outside the timed part)."""
    from oracle import ipa_dense
    if inp is None:
        inp = ipa_inputs(IpaDims(B=1, L=L, H=H, C=C, Pq=PQ, Pv=PV, R=R, Cz=CZ), seed)
    rows_done, t_total = 0, 0.0
    while rows_done < max_rows and t_total < seconds:
        rows = np.arange(rows_done, min(rows_done + 64, L, max_rows))
        t0 = time.perf_counter()
        ipa_dense(inp, rows=rows)
        t_total += time.perf_counter() - t0
        rows_done += len(rows)
    flops = 2.0 * rows_done * L * H * (C + 3 * PQ + 1 + R * CZ + C + 3 * PV + R * CZ)
    return flops / t_total / 1e12, rows_done, t_total


def timed_graph(torch, fn, flush, n=20):
    """Mean CUDA-event time (ms) of `fn` replayed as a CUDA graph, L2 flushed
    (untimed) before each replay; direct launches if capture fails."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    run = fn
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        torch.cuda.synchronize()
        run = gr.replay
    except Exception:  # noqa: BLE001 -- fall back to direct launches
        torch.cuda.synchronize()
    ts = []
    for _ in range(n):
        flush.zero_()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        run()
        a1.record()
        torch.cuda.synchronize()
        ts.append(a0.elapsed_time(a1))
    return statistics.mean(ts)


def fig2a_mb(L):
    """The FlashIPA page's Fig. 2A memory fits (MB) at length L, as printed:
    IPA 2.4e-3 L^2 + 1.4e-2 L, FlashIPA -7e-12 L^2 + 7.5e-2 L (context only;
    their hardware and precision are not stated)."""
    return {"ipa_MB": 2.4e-3 * L * L + 1.4e-2 * L, "flashipa_MB": -7e-12 * L * L + 7.5e-2 * L}


def bench_configs(api, torch, dev, flush):
    """Each configuration of the fused core on its own: step (prologue +
    core) and core alone as CUDA-graph replays, algorithmic TFLOP/s of the
    core (valid pairs only), fraction of the measured peak, and the device
    bytes one call needs (inputs + output + workspace)."""
    from rna_structure_models_b200.synth import IpaDims, ipa_inputs, ipa_preset
    peaks, kind = measured_peaks()
    peak = float(peaks["bf16_tflops"])
    cases = [("AF2-sized, last 10% masked", ipa_preset("af2")),
             ("batched generation-shaped, ragged 64..128", ipa_preset("batched"))]
    cases += [(f"long-context L={Lc}", ipa_inputs(IpaDims(B=1, L=Lc, H=12), 0)) for Lc in (2048, 8192, 16384)]
    res = []
    for name, inp in cases:
        Bc, Lc, Hc, _ = inp["q"].shape
        Rc, Czc = inp["z1"].shape[2], inp["z1"].shape[3]
        d = {n: torch.from_numpy(inp[n]).to(dev) for n in api.IPA_INPUTS}
        plan = api.IpaPlan(Bc, Lc, Hc, C, PQ, PV, Rc, Czc, device=dev)
        out = torch.empty((Bc, Lc, Hc, plan.F), dtype=torch.float32, device=dev)
        args_in = [d[n] for n in api.IPA_INPUTS]

        def step():
            plan.prologue(*args_in)
            plan.core(out)

        ms_step = timed_graph(torch, step, flush)
        ms_core = timed_graph(torch, lambda: plan.core(out), flush)
        plan.check()
        n_valid = inp["mask"].sum(axis=1)
        flops = ipa_flops(Bc, Lc, n_valid=n_valid, heads=Hc, rcz=Rc * Czc)
        in_bytes = sum(t.numel() * t.element_size() for t in args_in)
        dbytes = in_bytes + out.numel() * 4 + plan.workspace.numel()
        entry = {"config": name, "B": Bc, "L": Lc, "H": Hc, "R_Cz": Rc * Czc,
                 "valid_pairs_per_head": float(np.sum(n_valid.astype(float) ** 2)),
                 "gflop_algorithmic": flops / 1e9, "core_us": ms_core * 1e3, "step_us": ms_step * 1e3,
                 "core_tflops": flops / (ms_core / 1e3) / 1e12, "step_tflops": flops / (ms_step / 1e3) / 1e12,
                 "frac": flops / (ms_core / 1e3) / 1e12 / peak, "peak_source": f"{kind} bf16 dense (burst)",
                 "device_bytes": dbytes, "workspace_bytes": plan.workspace.numel()}
        if Bc == 1:
            entry["fig2a_context"] = fig2a_mb(Lc)
        res.append(entry)
        del d, plan, out
        torch.cuda.empty_cache()
    return res


def bench_backward(api, torch, dev, flush, L, dvc, names):
    """Training forward and gradient pass at the headline workload."""
    peaks, kind = measured_peaks()
    peak = float(peaks["bf16_tflops"])
    plan = api.IpaPlan(1, L, H, C, PQ, PV, R, CZ, device=dev)
    gplan = api.IpaGradPlan(1, L, H, C, PQ, PV, R, CZ, device=dev)
    args_in = [dvc[n] for n in names]
    out, lse, U = plan.train(*args_in)
    g = torch.randn(out.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(1))
    grads = gplan(dvc, out, lse, U, g)
    torch.cuda.synchronize()
    plan.check()
    gplan.check()
    ms_train = timed_graph(torch, lambda: plan.train(*args_in, out=out, lse=lse, u_agg=U), flush)
    ms_bwd = timed_graph(torch, lambda: gplan(dvc, out, lse, U, g, grads=grads), flush, n=10)
    gplan.check()
    fb = ipa_bwd_flops(1, L)
    return {"workload": f"IPA core gradients B=1 L={L} H={H} C={C} Pq={PQ} Pv={PV} R={R} Cz={CZ}",
            "train_forward_ms": ms_train, "backward_ms": ms_bwd,
            "backward_gflop_algorithmic": fb / 1e9,
            "backward_tflops": fb / (ms_bwd / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "achieved": fb / (ms_bwd / 1e3) / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": fb / (ms_bwd / 1e3) / 1e12 / peak,
                         "peak_source": f"{kind} bf16 dense (burst)",
                         "note": "whole gradient call (prologue again, rows, query pass, key pass, mapping)"},
            "issued_flops_per_triple": 4480, "algorithmic_flops_per_triple": 2 * (3 * 285 + 2 * 296),
            "workspace_bytes": gplan.workspace.numel()}


def cpu_oracle_configs(seconds):
    """The float64 oracle on each configuration of the core: tiny, AF2 and
    batched in full; the long-context lengths on 64-row blocks within a time
    budget, extrapolated linearly in rows to the whole sequence."""
    from oracle import ipa_dense
    from rna_structure_models_b200.synth import IpaDims, ipa_inputs, ipa_preset
    res = []
    for name in ("tiny", "af2", "batched"):
        inp = ipa_preset(name)
        t0 = time.perf_counter()
        if name == "batched":
            for b in range(inp["q"].shape[0]):
                ipa_dense({k: (v[b:b + 1] if isinstance(v, np.ndarray) and v.ndim >= 2 and k not in ("w_bias",)
                               else v) for k, v in inp.items()})
        else:
            ipa_dense(inp)
        res.append({"config": name, "seconds": time.perf_counter() - t0, "extrapolated": False})
    for Lc in (2048, 4096, 8192, 16384):
        inp = ipa_inputs(IpaDims(B=1, L=Lc, H=12), 0)
        rows, t = 0, 0.0
        while rows < Lc and t < seconds / 4:
            r = np.arange(rows, min(rows + 64, Lc))
            t0 = time.perf_counter()
            ipa_dense(inp, rows=r)
            t += time.perf_counter() - t0
            rows += len(r)
        res.append({"config": f"long-context L={Lc}", "seconds": t * Lc / rows, "extrapolated": rows < Lc,
                    "rows_timed": rows})
    # the direction/distance variant (B=2, N=2048): 64-row blocks, extrapolated in rows
    from oracle import geo_dense_blocked
    g = geo_inputs(GeoDims(B=2, N=2048, H=8, M=4, Cout=256), 0)
    rows, t = 0, 0.0
    while rows < 2048 and t < seconds / 4:
        r = np.arange(rows, min(rows + 64, 2048))
        t0 = time.perf_counter()
        geo_dense_blocked(g, rows=r, block=64)
        t += time.perf_counter() - t0
        rows += len(r)
    res.append({"config": "geometric variant B=2 N=2048", "seconds": t * 2048 / rows, "extrapolated": rows < 2048,
                "rows_timed": rows})
    return res


def run_reference(args, rank, world):
    if rank != 0:
        return
    L = args.L
    ms = []
    inp = ipa_inputs(IpaDims(B=1, L=L, H=H, C=C, Pq=PQ, Pv=PV, R=R, Cz=CZ), 0)
    rows_per_step = args.ref_rows
    if rows_per_step is None:
        # size each step so that the whole --steps K --warmup W run takes about
        # REF_BUDGET_S seconds of oracle time (calibrated on 8 rows, untimed)
        _, _, t8 = cpu_oracle_sample(L, 1e9, 8, inp=inp)
        per_row = t8 / 8
        rows_per_step = int(max(1, min(64, REF_BUDGET_S / max(1, args.steps + args.warmup) / per_row)))
    for s in range(args.warmup + args.steps):
        _, nrows, dt = cpu_oracle_sample(L, 1e9, rows_per_step, inp=inp)
        if s >= args.warmup:
            ms.append(dt * 1e3)
    flops_step = 2.0 * rows_per_step * L * H * (C + 3 * PQ + 1 + R * CZ + C + 3 * PV + R * CZ)
    value = flops_step * len(ms) / (sum(ms) / 1e3) / 1e12
    sample = f"{rows_per_step} query rows x all {L} keys x {H} heads of the L={L} workload per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"IPA core B=1 L={L} H={H} C={C} Pq={PQ} Pv={PV} R={R} Cz={CZ}",
                       "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--L", type=int, default=4096)
    ap.add_argument("--ref-rows", type=int, default=None,
                    help="query rows per reference step (default: sized to ~90 s for the whole run)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variant", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration timings")
    ap.add_argument("--no-backward", action="store_true", help="skip the gradient-pass timing")
    ap.add_argument("--core-only", action="store_true", help="profiling aid: time only, print nothing else")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels directly instead of replaying a CUDA graph")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    from rna_structure_models_b200 import api

    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    L = args.L
    inp = rank_inputs(rank, L)                             # each rank its own batch element
    names = api.IPA_INPUTS
    host = {n: torch.from_numpy(inp[n]) for n in names}
    dvc = {n: host[n].to(dev) for n in names}
    plan = api.IpaPlan(1, L, H, C, PQ, PV, R, CZ, device=dev)
    out = torch.empty((1, L, H, plan.F), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    args_in = [dvc[n] for n in names]

    def step():
        plan.prologue(*args_in)
        plan.core(out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    plan.check()

    # the step as a CUDA graph (tile, rows and core kernels replayed without
    # host launch gaps), and the core alone for its roofline time
    graphs = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g_step, g_core = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step):
            step()
        with torch.cuda.graph(g_core):
            plan.core(out)
        torch.cuda.synchronize()
        graphs = (g_step, g_core)
        for _ in range(3):
            g_step.replay()
        torch.cuda.synchronize()
        plan.check()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    evc = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for k in range(K):
            flush.zero_()                                  # L2 flushed between steps (untimed)
            ev[k][0].record()
            if graphs:
                graphs[0].replay()
            else:
                plan.prologue(*args_in)
                ev[k][1].record()
                plan.core(out)
            ev[k][2].record()
        torch.cuda.synchronize()
        if graphs:                                         # the core alone, same flush between runs
            for k in range(K):
                flush.zero_()
                evc[k][0].record()
                graphs[1].replay()
                evc[k][1].record()
            torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    plan.check()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    if graphs:
        core_ms = [e[0].elapsed_time(e[1]) for e in evc]
        pro_ms = [max(0.0, sm - cm) for sm, cm in zip(step_ms, core_ms)]
    else:
        core_ms = [e[1].elapsed_time(e[2]) for e in ev]
        pro_ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dist, dev)
    if args.core_only:
        if world > 1:
            dist.destroy_process_group()
        return

    flops = ipa_flops(1, L)
    value = aggregate_tflops(world, flops, K, total_ms)
    peaks, peak_kind = measured_peaks()
    core_mean = statistics.mean(core_ms)
    achieved = flops / (core_mean / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])        # fp16 and bf16 share the dense tensor rate
    traffic = NCU_TRAFFIC["bytes_per_launch"] if NCU_TRAFFIC["kernel_sha256"] == kernel_sha() else None

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": f"IPA core B=1 L={L} H={H} C={C} Pq={PQ} Pv={PV} R={R} Cz={CZ} per GPU",
                   "global_batch": world, "seq_len": L, "parallelism": f"dp{world}",
                   "l2": "flushed between steps (256 MB write, untimed)",
                   "step": "prologue (frames, augmented fp16 operands) + fused attention core",
                   "launch": "direct launches" if args.no_graph else
                             "CUDA graph replay of the step's 3 kernels; core time from a core-only graph"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": CORE_KERNEL,
                     "peak_source": f"{peak_kind} bf16 dense (burst); fp16 has the same nominal rate",
                     "core_ms": core_mean,
                     "prologue_ms": statistics.mean(pro_ms),   # step minus core with graphs
                     "issued_frac": achieved * 640.0 / 581.0 / peak},
        "gpu_launches": 3 * K,                             # tile, rows, core
        "clocks": clk.summary(),
    }

    # end to end through the public API with host buffers
    if not args.no_e2e:
        pinned = {n: host[n].pin_memory() for n in names}
        res = torch.empty((1, L, H, plan.F), dtype=torch.float32, pin_memory=True)
        d2h = res.numel() * res.element_size()
        ke = max(3, min(K, 50))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hc = api.IpaHostCalls(1, L, H, C, PQ, PV, R, CZ, slots=3, device=dev)
        # the inputs in the packed host layout (filled once, like any host input)
        packed = hc.pack(pinned)
        h2d = hc.packed_layout()[0]
        outs = [res] + [torch.empty_like(res).pin_memory() for _ in range(2)]
        for _ in range(max(1, min(args.warmup, 3))):
            for k in range(3):
                hc.call_packed(packed, outs[k], k)
            hc.run([pinned] * 3, outs)
        hc.check()

        def timed_calls(call, serial):
            # serial: one call at a time on one stream (copies, kernels and
            # the copy back in series); else calls k on stream k mod 3
            s0 = hc.streams[0]
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0.record(s0)
            for st in hc.streams[1:]:
                st.wait_event(e0)
            for k in range(ke):
                call(0 if serial else k % 3, res if serial else outs[k % 3])
            for st in hc.streams[1:]:
                done = torch.cuda.Event()
                done.record(st)
                s0.wait_event(done)
            e1.record(s0)
            torch.cuda.synchronize()
            hc.check()
            return max_over_ranks(e0.elapsed_time(e1), world, dist, dev)

        t_serial = timed_calls(lambda k, o: hc.call_packed(packed, o, k), True)
        te = timed_calls(lambda k, o: hc.call_packed(packed, o, k), False)
        t_per_input = timed_calls(lambda k, o: hc.call(pinned, o, k), False)
        line["e2e"] = {"value": aggregate_tflops(world, flops, ke, te), "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ke,
                       "ms_per_step": te / ke,
                       "api": "C entry point ipa_attn_fwd_host_packed (the 13 inputs in one page-locked "
                              "buffer: one upload, one download per call), three streams",
                       "serial_ms_per_step": t_serial / ke,
                       "per_input_uploads_ms_per_step": t_per_input / ke}

    # second hot-path row: direction/distance geometric attention (B=2, N=2048)
    if not args.no_variant and rank == 0:
        g = geo_inputs(GeoDims(B=2, N=2048, H=8, M=4, Cout=256), 0)
        gd = {k: (torch.from_numpy(v).to(dev) if isinstance(v, np.ndarray) else None) for k, v in g.items()
              if k != "dims"}
        gp = api.GeoPlan(2, 2048, 8, 4, 256, device=dev)
        outs = {"vectors": torch.empty((2, 2048, 8, 4, 3), device=dev),
                "output": torch.empty((2, 2048, 256), device=dev),
                "attention": torch.empty((2, 8, 2048, 2048), device=dev)}
        res, resg = {}, {}
        for with_att in (False, True):
            o2 = dict(outs)
            if not with_att:
                o2["attention"] = None
            # device time of the call's kernels (CUDA-graph replay), next to the direct call
            resg[with_att] = timed_graph(torch, lambda o2=o2: gp(gd, out=o2), flush)
            for _ in range(3):
                gp(gd, out=o2)
            torch.cuda.synchronize()
            times = []
            for _ in range(20):
                flush.zero_()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                gp(gd, out=o2)
                a1.record()
                torch.cuda.synchronize()
                times.append(a0.elapsed_time(a1))
            res[with_att] = statistics.mean(times)
        gp.check()
        pairs = 2 * 8 * 2048 * 2048
        att_bytes = pairs * 4 + pairs * 1          # attention map written + pair mask read
        map_gbs = att_bytes / ((resg[True] - resg[False]) / 1e3) / 1e9 if resg[True] > resg[False] else None
        peaks, psrc = measured_peaks()
        # scores and aggregation: per (i, j, h) 27 fp32-pipe operations (the
        # direction dot product 3, displacement 3, squared distance 3, score
        # 4, subtraction of the running maximum 1, row sum 1, 3 M = 12 value
        # products) and 2 MUFU (square root, exp2); the fp32 pipe bounds it
        # at 148 SMs x 128 lanes x 1.965 GHz
        alu_ops = 27
        alu_peak = 148 * 128 * 1.965e9 / 1e12
        alu_achieved = pairs * alu_ops / (resg[False] / 1e3) / 1e12
        line["variant"] = {
            "workload": "geometric attention B=2 N=2048 H=8 M=4 Cout=256, 20% pair mask, 5% invalid frames",
            "ms_no_attention_map": resg[False], "ms_with_attention_map": resg[True],
            "direct_call_ms": {"no_attention_map": res[False], "with_attention_map": res[True]},
            "timing": "ms_*: CUDA-graph replay of the call's kernels (device time); direct_call_ms: one "
                      "call from Python per step, host work included",
            "pair_heads_per_s": pairs / (resg[False] / 1e3),
            "attention_map_GBps": map_gbs,
            "roofline": [
                {"kernel": "geo_attn_kernel", "bound": "alu", "achieved": alu_achieved, "peak": alu_peak,
                 "unit": "Top/s (fp32 pipe)", "frac": alu_achieved / alu_peak,
                 "note": f"{alu_ops} fp32 operations per (query, key, head), 2 MUFU; timed as the whole call "
                         "without the map (weights, prep and readout kernels included), CUDA-graph replay"},
                {"kernel": "geo_map_kernel", "bound": "hbm", "achieved": map_gbs, "peak": peaks["hbm_gbs"],
                 "unit": "GB/s", "frac": map_gbs / peaks["hbm_gbs"] if map_gbs else None,
                 "peak_source": psrc,
                 "note": "268 MB map written + 67 MB pair mask read, over the time the map adds to the call"},
            ],
        }
        # gradients of the variant (forward statistics recomputed inside the call)
        from rna_structure_models_b200.synth import geo_upstream
        ug = {k: (torch.from_numpy(v).to(dev) if v is not None else None)
              for k, v in geo_upstream(g["dims"], 1).items()}
        gg = api.GeoGradPlan(2, 2048, 8, 4, 256, device=dev)
        gout = {n: torch.empty(tuple(gd[n].shape), device=dev) for n in api.GEO_GRADS}
        bres, bresg = {}, {}
        for with_ga in (False, True):
            ga = ug["g_attention"] if with_ga else None
            bresg[with_ga] = timed_graph(torch, lambda ga=ga: gg(gd, ug["g_output"], ga, ug["g_vectors"], out=gout),
                                         flush, n=10)
            for _ in range(3):
                gg(gd, ug["g_output"], ga, ug["g_vectors"], out=gout)
            torch.cuda.synchronize()
            times = []
            for _ in range(10):
                flush.zero_()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                gg(gd, ug["g_output"], ga, ug["g_vectors"], out=gout)
                a1.record()
                torch.cuda.synchronize()
                times.append(a0.elapsed_time(a1))
            bres[with_ga] = statistics.mean(times)
        line["variant"].update({
            "backward_ms": bresg[False], "backward_ms_with_attention_grad": bresg[True],
            "backward_direct_call_ms": {"no_attention_grad": bres[False], "with_attention_grad": bres[True]},
            "backward_pair_heads_per_s": pairs / (bresg[False] / 1e3),
        })

    # distance-aware attention of MEET (§2.2) on the same core (B=1, L=4096, H=8)
    if not args.no_variant and rank == 0:
        from rna_structure_models_b200.synth import MeetDims, meet_inputs
        mi = meet_inputs(MeetDims(B=1, L=L, H=8, C=16), 0)
        md = {n: torch.from_numpy(mi[n]).to(dev) for n in api.MEET_INPUTS}
        mp = api.MeetPlan(1, L, 8, 16, device=dev)
        mout = torch.empty((1, L, 8, 16), device=dev)
        for _ in range(3):
            mp(*[md[n] for n in api.MEET_INPUTS], out=mout)
        torch.cuda.synchronize()
        mt = []
        for _ in range(20):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            mp(*[md[n] for n in api.MEET_INPUTS], out=mout)
            a1.record()
            torch.cuda.synchronize()
            mt.append(a0.elapsed_time(a1))
        mp.check()
        ms_meet_direct = statistics.mean(mt)
        ms_meet = timed_graph(torch, lambda: mp(*[md[n] for n in api.MEET_INPUTS], out=mout), flush)
        mp.check()
        triples = L * L * 8
        line["meet"] = {
            "workload": f"MEET distance-aware attention B=1 L={L} H=8 C=16 (all four kernels of a call)",
            "ms": ms_meet, "direct_call_ms": ms_meet_direct,
            "timing": "ms: CUDA-graph replay of the call's kernels; direct_call_ms: one call from Python per step",
            "pair_heads_per_s": triples / (ms_meet / 1e3),
            "tflops_algorithmic": triples * 2 * (2 * 16 + 9) / (ms_meet / 1e3) / 1e12,
        }

    # the IPA layer around the core (projections + core), same sizes, c_s = 384
    if not args.no_variant and rank == 0:
        from rna_structure_models_b200.synth import ModuleDims, module_inputs
        md_ = ModuleDims(B=1, L=L, H=12, Cz=128, c_s=384)
        mi_ = module_inputs(md_, 0)
        mdev = {k: torch.from_numpy(mi_[k]).to(dev) for k in api.MODULE_INPUTS}
        mplan = api.ModulePlan(1, L, 12, 16, 4, 8, 2, 128, 384, device=dev)
        mo = torch.empty((1, L, 384), device=dev)

        def timed(fn, n=20):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(n):
                flush.zero_()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                fn()
                a1.record()
                torch.cuda.synchronize()
                ts.append(a0.elapsed_time(a1))
            return statistics.mean(ts)

        ms_layer_direct = timed(lambda: mplan(mdev, out=mo))
        ms_layer = timed_graph(torch, lambda: mplan(mdev, out=mo), flush)
        mplan.check()
        width = 12 * (3 * 16 + 3 * (2 * 4 + 8))
        HF = 12 * (16 + 32 + 128)
        lin_in = api.LinearPlan(L, 384, width, device=dev)
        lin_out = api.LinearPlan(L, HF, 384, device=dev)
        xo = torch.randn((L, HF), device=dev)
        wo = torch.randn((HF, 384), device=dev)
        ms_in_direct = timed(lambda: lin_in(mdev["s"].view(L, 384), mdev["w_in"], mdev["b_in"]))
        ms_out_direct = timed(lambda: lin_out(xo, wo, mdev["b_out"]))
        ms_in = timed_graph(torch, lambda: lin_in(mdev["s"].view(L, 384), mdev["w_in"], mdev["b_in"]), flush)
        ms_out = timed_graph(torch, lambda: lin_out(xo, wo, mdev["b_out"]), flush)
        lin_in.check()
        lin_out.check()
        f_in, f_out = 2.0 * L * 384 * width, 2.0 * L * HF * 384
        line["layer"] = {
            "workload": f"IPA layer B=1 L={L} H=12 Cz=128 c_s=384: input projection, core, output projection",
            "ms": ms_layer,
            "direct_call_ms": {"layer": ms_layer_direct, "linear_in": ms_in_direct, "linear_out": ms_out_direct},
            "timing": "ms and linear_*_ms: CUDA-graph replay of the calls' kernels (device time); "
                      "direct_call_ms: one call from Python per step, host work (tensor-map encoding) included",
            "linear_in_ms": ms_in, "linear_in_tflops": f_in / (ms_in / 1e3) / 1e12,
            "linear_out_ms": ms_out, "linear_out_tflops": f_out / (ms_out / 1e3) / 1e12,
            "linear_note": "tf32 tcgen05 GEMM on the caller's fp32 x (TMA); each call transposes W to fp32 W^T "
                           "(one small kernel) first",
        }

    # secondary sections: a failure there is reported in the line and does not
    # take the headline with it
    for key, enabled, fn in (("configs", not args.no_configs, lambda: bench_configs(api, torch, dev, flush)),
                             ("backward", not args.no_backward,
                              lambda: bench_backward(api, torch, dev, flush, L, dvc, names))):
        if enabled and rank == 0:
            try:
                line[key] = fn()
            except Exception as exc:  # noqa: BLE001
                torch.cuda.synchronize()
                line[key] = {"error": f"{type(exc).__name__}: {exc}"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, nrows, secs = cpu_oracle_sample(L, args.cpu_seconds, 4096)
        cores, blas = host_threads()
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                "host_cores": cores, "blas_threads": blas,
                                "sample": f"{nrows} query rows x {L} keys x {H} heads of the same workload, "
                                          f"{secs:.1f} s of numpy float64 (einsum on one thread; "
                                          f"{cores} host cores available)"}
        if not args.no_configs:
            line["cpu_configs"] = cpu_oracle_configs(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

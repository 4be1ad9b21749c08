#!/usr/bin/env python
"""Benchmark: one Muon step (momentum, Gram Newton-Schulz x5, update) over a
projection-matrix set, on N GPUs of one node.

A "step" is one dmuon_step call over the whole set (224 bf16 matrices of the
Llama-7B projection shapes by default).  Inputs are resident in HBM when the
timed region starts; they total far more than the 126 MB L2 per step, so no
L2 flush is done between steps.  Per-kernel times come from CUDA events that
the library records around each of its launches on the launching stream,
inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 oracle on the host cores

Multi-GPU (torchrun): every rank runs its own replica of the set (weak
scaling, no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "Muon steps/sec (matrices/s) and NS TFLOP/s as % of B200 BF16 peak, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama_7b_bf16")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--e2e-group", type=int, default=16,
                    help="matrices per dmuon_step call in the end-to-end pipeline")
    ap.add_argument("--cpu-budget-s", type=float, default=30.0,
                    help="bound on the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and time its replays")
    ap.add_argument("--ns-steps", type=int, default=None,
                    help="override the workload's Newton-Schulz iteration count")
    ap.add_argument("--stage", choices=["gram", "poly", "apply", "momentum", "update", "step", "clip",
                                        "lib_chain", "lib_apply"],
                    help="time one kernel through its stage call instead of the whole step")
    ap.add_argument("--clip-norm", type=float, default=None,
                    help="time dmuon_step_clipped: global 2-norm clipping of the gradients to this bound")
    ap.add_argument("--lib", choices=["torch", "quack"], default="torch",
                    help="--stage lib_chain / lib_apply: the library whose GEMMs run the comparison")
    ap.add_argument("--owners", action="store_true",
                    help="dedicated ownership over the ranks: every rank holds the whole set, steps the "
                         "matrices it owns and broadcasts them (strong scaling); default: one replica per rank")
    ap.add_argument("--launch-detail", default=None, metavar="PATH",
                    help="after the timed region, write every launch of one more step (kind, start, "
                         "duration, work) to PATH as JSON")
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--n", type=int, default=4096)
    return ap.parse_args(argv)


# ------------------------------------------------------------------- peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def roofline_peak(kind: str, has_flops: bool, peaks: dict, sms: int, sm_max_mhz):
    """(bound, unit, peak, basis) of the step's dominant kernel.  The FFMA
    kernels (fp32 products on the CUDA cores: `*_ffma`, and the clustered
    thin-matrix chain `chain_small`) are bound by the FMA issue rate: SMs x 128
    fp32 lanes (4 schedulers x 32) x 2 flop per cycle at the maximum SM clock;
    tensor-core kernels by the measured sustained bf16 peak; kernels counted
    in bytes by the measured copy bandwidth.  basis is None unless derived here."""
    if has_flops and (kind.endswith("_ffma") or kind == "chain_small"):
        mhz = float(sm_max_mhz or 1965.0)
        peak = sms * 128 * 2 * mhz * 1e6 / 1e12
        return "alu", "TFLOP/s", round(peak, 1), f"{sms} SMs x 128 fp32 lanes x 2 flop x {mhz:.0f} MHz"
    if has_flops:
        return "tensor", "TFLOP/s", float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))), None
    return "hbm", "GB/s", float(peaks["hbm_gbs"]), None


def launches_per_matrix(kernel: str, m: int, n: int, dtype: str, steps: int):
    """How many launches of `kernel` one matrix of oriented shape m x n sees in
    a step (the library's default schedule: bf16 matrices with m <= 64, or
    m < 256 and n < 3 m, run FFMA chains; wide bf16 matrices on the tensor path,
    n >= 2 m or n >= 1.25 m with m >= 512, run their last two iterations as one
    Gram-space block)."""
    if kernel != "apply_tc" or dtype != "bf16" or m <= 64 or (m < 256 and n < 3 * m):
        return None  # FFMA paths
    mode = os.environ.get("DMUON_GRAM_BLOCKS", "1")[:1]
    wide = n >= 2 * m or (m >= 512 and 4 * n >= 5 * m)
    blocked = mode != "0" and wide and steps >= 2
    if blocked and mode == "2":
        return None
    applies = steps - 1 if blocked else steps
    # the last apply updates the parameters itself (apply_update_tc) unless disabled
    fused = os.environ.get("DMUON_FUSED_UPDATE", "1")[:1] != "0" and steps >= 1
    return applies - 1 if fused else applies


def traffic_record(kernel: str, w, launches: int):
    """Average DRAM bytes per launch of `kernel` in one step of workload w, from
    the committed per-matrix ncu figures, or None if they do not cover it or
    the kernel source changed since they were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            ent = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not ent or launches <= 0:
        return None
    src = os.path.join(ROOT, "newton_schulz_grad_b200", "csrc", ent.get("source", ""))
    try:
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != ent.get("sha256"):
                return None
    except OSError:
        return None
    per = ent.get("bytes_per_matrix", {})
    total = 0.0
    for r, c in w.shapes:
        m, n = min(r, c), max(r, c)
        k = launches_per_matrix(kernel, m, n, w.dtype, w.ns_steps)
        if k is None or f"{m}x{n}" not in per:
            return None
        total += k * per[f"{m}x{n}"]
    return total / launches


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def _gpu_id(self) -> str:
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = getattr(p, "pci_bus_id", None)
            dom = getattr(p, "pci_domain_id", 0)
            devid = getattr(p, "pci_device_id", 0)
            if bus is not None:
                return f"{dom:08X}:{bus:02X}:{devid:02X}.0"
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[self.dev].strip()
        return str(self.dev)

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= len(self.FIELDS):
                    rows.append([c.strip() for c in r])
        os.unlink(self.path)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for k, nm in enumerate(names):
                if r[5 + k].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def reduce_max(value: float, device) -> float:
    """Max over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(count_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job matrices/s: all ranks' matrices over the slowest rank's time."""
    return world * count_per_rank / (ms_max / 1e3)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def class_samples(w):
    """One matrix index per launch class (oriented shape), with class sizes."""
    classes = {}
    for i, (r, c) in enumerate(w.shapes):
        key = (min(r, c), max(r, c))
        classes.setdefault(key, []).append(i)
    return [(key, idx[0], len(idx)) for key, idx in classes.items()]


def oracle_matrix_seconds(w, idx: int) -> float:
    """Time the oracle's Muon step on matrix idx of w (host fp64)."""
    from oracle import muon as om
    p, g, b = workloads.make_matrix(w, idx, "cpu", workloads.skewed_indices(w))
    p64, g64, b64 = (t.to(torch.float64).numpy() for t in (p, g, b))
    t0 = time.perf_counter()
    om.muon_step([p64], [g64], [b64], w.lr, w.momentum, w.nesterov, w.ns_steps, None, w.wd)
    return time.perf_counter() - t0


def cpu_baseline(w, budget_s: float):
    """Oracle matrices/s extrapolated from one timed matrix per launch class."""
    per_class = []
    spent = 0.0
    for key, idx, cnt in sorted(class_samples(w), key=lambda e: e[0][0] ** 2 * e[0][1]):
        if spent > budget_s and per_class:
            # out of budget: extrapolate by flops from the cheapest measured class
            (k0, t0, _) = per_class[0]
            f0 = 3 * k0[0] ** 2 * k0[1] + k0[0] ** 3
            f = 3 * key[0] ** 2 * key[1] + key[0] ** 3
            per_class.append((key, t0 * f / f0, cnt))
            continue
        t = oracle_matrix_seconds(w, idx)
        spent += t
        per_class.append((key, t, cnt))
    total = sum(t * cnt for _, t, cnt in per_class)
    sample = "; ".join(f"1 x {k[0]}x{k[1]} ({t:.2f} s, class of {c})" for k, t, c in per_class)
    return {"value": w.count / total, "unit": "matrices/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle, one matrix per launch class, extrapolated to the "
                      f"{w.count}-matrix set by class counts: {sample}"}


# ---------------------------------------------------------------- our arm
def run_ours(args):
    import newton_schulz_grad_b200 as nsg

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist
    w = workloads.get(args.workload)
    if args.ns_steps is not None:
        import dataclasses
        w = dataclasses.replace(w, ns_steps=args.ns_steps)
    ps, gs, bs = workloads.make_all(w, dev)
    code = 1 if w.dtype == "bf16" else 0
    shapes = [(r, c, code) for r, c in w.shapes]
    pp = [t.data_ptr() for t in ps]
    gp = [t.data_ptr() for t in gs]
    bp = [t.data_ptr() for t in bs]
    stream = torch.cuda.current_stream(dev)
    # graph capture needs a non-default stream; the library keeps one
    # workspace per stream, so warm-up and capture use the same one
    run_stream = torch.cuda.Stream(dev) if args.graph else stream
    if args.owners:  # this rank launches the step of the matrices it owns
        own = nsg.dmuon_assign_owners(shapes, world)[0]
        launches_per_step = nsg.dmuon_step_launches([s for s, o in zip(shapes, own) if o == rank], w.ns_steps)
    else:
        launches_per_step = nsg.dmuon_step_launches(shapes, w.ns_steps)
    if args.clip_norm is not None:
        # one norm launch per table of <= 256 matrices of one shape, plus the coefficient
        groups = {}
        for sh in shapes:
            groups[sh] = groups.get(sh, 0) + 1
        launches_per_step += sum((c + 255) // 256 for c in groups.values()) + 1

    def step():
        nsg.dmuon_step_ptrs(pp, gp, bp, shapes, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                            ns_steps=w.ns_steps, wd=w.wd, stream=run_stream, max_norm=args.clip_norm)

    if args.owners:
        if args.graph or args.clip_norm is not None:
            raise SystemExit("--owners runs without --graph and --clip-norm")
        from newton_schulz_grad_b200.distributed import owned_step

        def step():  # noqa: F811
            owned_step(ps, gs, bs, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov, ns_steps=w.ns_steps,
                       wd=w.wd)

    for _ in range(max(args.warmup, 0)):
        step()
    # one more warm-up step with the per-launch events on: the library keeps
    # those events for reuse, so the timed region below only records them
    nsg.dmuon_profile_start()
    step()
    nsg.dmuon_profile_stop()
    st = nsg.dmuon_stream_status(run_stream)
    if st != nsg.DMUON_OK:
        raise RuntimeError(f"warm-up failed: {nsg.STATUS_NAMES[st]} {nsg.dmuon_get_last_error()}")
    eager_step = step
    if args.graph:
        # one step captured once (after the warm-up allocated the workspace);
        # the timed loop replays it on the timing stream
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=run_stream):
            eager_step()

        def step():  # noqa: F811
            graph.replay()
        step()
        torch.cuda.synchronize(dev)

    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    nsg.dmuon_profile_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    e1.synchronize()
    kstats = nsg.dmuon_profile_stop()
    if args.graph:
        # replays bypass the library's event timing: break the kernels down on
        # eager steps right after the timed region
        torch.cuda.synchronize(dev)
        nsg.dmuon_profile_start()
        for _ in range(args.steps):
            eager_step()
        kstats = nsg.dmuon_profile_stop()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    clk = clocks.stop()
    st = nsg.dmuon_stream_status(stream)
    if st != nsg.DMUON_OK:
        raise RuntimeError(f"timed steps failed: {nsg.STATUS_NAMES[st]}")
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = reduce_max(ms_local, dev)
    # replicas: every rank steps the whole set; owners: the ranks share one set
    value = aggregate_value(w.count, 1 if args.owners else world, ms)

    peaks, peak_src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    chain = {k: v for k, v in kstats.items() if k.endswith("_tc") or k.endswith("_ffma") or k == "chain_small"}
    chain_ms = sum(v["total_ms"] for v in chain.values()) / args.steps
    ns_flops = w.ns_flops()
    ns_tflops_step = ns_flops / (ms / 1e3) / 1e12
    ns_tflops_chain = ns_flops / (chain_ms / 1e3) / 1e12 if chain_ms > 0 else None
    executed = sum(v["flops"] for v in chain.values()) / args.steps
    # dominant kernel: largest share of the timed region among the kernels of
    # the chain stream (aux-stream event windows include queueing, see below)
    timed_kinds = {k: v for k, v in kstats.items() if k not in ("momentum", "norm", "update")} or kstats
    dom = max(timed_kinds.items(), key=lambda kv: kv[1]["total_ms"])
    dname, d = dom
    avg_ms = d["total_ms"] / d["launches"]
    bound, unit, peak, peak_basis = roofline_peak(dname, d["flops"] > 0, peaks,
                                                  torch.cuda.get_device_properties(dev).multi_processor_count,
                                                  (clk or {}).get("sm_max_mhz"))
    if d["flops"] > 0:
        achieved = (d["flops"] / d["launches"]) / (avg_ms / 1e3) / 1e12
    else:
        achieved = (d["bytes"] / d["launches"]) / (avg_ms / 1e3) / 1e9
    # kernels of the auxiliary stream (momentum, norm, separate update) run
    # underneath the chain: their event windows include time spent queued
    # behind it, so they carry no bandwidth figure here (see elementwise_isolated)
    aux_kinds = ("momentum", "norm", "update")
    kernels = {k: {"launches_per_step": v["launches"] // args.steps,
                   "ms_per_step": round(v["total_ms"] / args.steps, 3),
                   **({"window": "aux stream, includes queueing behind the chain"} if k in aux_kinds else
                      {"share_of_chain": round(v["total_ms"] / sum(x["total_ms"] for x in chain.values()), 4)}
                      if k in chain else {})}
               for k, v in kstats.items()}

    if args.launch_detail:
        nsg.dmuon_profile_start()
        eager_step()
        recs = nsg.dmuon_profile_stop_launches()
        with open(args.launch_detail, "w") as f:
            json.dump({"workload": w.name, "launches": recs}, f)

    # the elementwise kernels run underneath the chain in the step above; their
    # own bandwidth comes from a few momentum + update-only steps (no iterations)
    elem_iso = {}
    if w.ns_steps > 0:
        nsg.dmuon_profile_start()
        for _ in range(3):
            nsg.dmuon_step_ptrs(pp, gp, bp, shapes, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                                ns_steps=0, wd=w.wd, stream=stream)
        iso = nsg.dmuon_profile_stop()
        for k in ("momentum", "update"):
            if k in iso:
                gbs = iso[k]["bytes"] / (iso[k]["total_ms"] / 1e3) / 1e9
                elem_iso[k] = {"GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / float(peaks["hbm_gbs"]), 3)}

    e2e = None
    if not args.no_e2e and not args.owners:  # the e2e pipeline steps whole replicas
        e2e = run_e2e(args, w, ps, gs, bs, shapes, stream, dev, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_budget_s)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "matrices/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "strong" if args.owners else "weak", "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded low-rank + noise gradients, random-init parameters)",
        "config": workload_config(w, args, world),
        "ns_tflops": round(executed / (ms / 1e3) / 1e12, 1),
        "ns_frac_of_peak": round(executed / (ms / 1e3) / 1e12 / sustained, 4),
        "ns_tflops_per_iteration_count": round(ns_tflops_step, 1),
        "ns_frac_of_peak_per_iteration_count": round(ns_tflops_step / sustained, 4),
        "ns_chain_tflops_per_iteration_count": round(ns_tflops_chain, 1) if ns_tflops_chain else None,
        "ns_flops_note": "ns_tflops counts the products the chain executes (one triangle of each "
                         "symmetric product; the last two iterations of wide matrices run in Gram space) "
                         "over the whole step time, against the measured sustained bf16 peak; the "
                         "*_per_iteration_count keys count 3m^2n+m^3 per matrix and iteration of the "
                         "per-iteration form instead (the figure the 60 % target is stated in)",
        "peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback",
        "roofline": {"kernel": dname, "bound": bound, "achieved": round(achieved, 1), "peak": peak,
                     "unit": unit, "frac": round(achieved / peak, 4),
                     **({"peak_basis": peak_basis} if peak_basis else {}),
                     "traffic": traffic_record(dname, w, d["launches"] // max(1, args.steps)),
                     "per_launch": {"flops": d["flops"] / d["launches"],
                                    "bytes": d["bytes"] / d["launches"], "avg_ms": avg_ms}},
        "elementwise_isolated": elem_iso,
        "elementwise_note": "in the step the momentum kernels of one chunk run on a second stream "
                            "underneath the Newton-Schulz chain of another; their bandwidth is measured "
                            "in momentum+update-only steps (elementwise_isolated)",
        "kernels": kernels,
        "gpu_launches": launches_per_step * args.steps,
        "cuda_graph": bool(args.graph),
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


def workload_config(w, args, world: int) -> dict:
    """The `config` of the JSON line: the workload, the same for both arms."""
    return {"workload": w.name, "matrices": w.count,
            "shapes": sorted({f"{r}x{c}" for r, c in w.shapes}),
            "ns_steps": w.ns_steps, "nesterov": w.nesterov, "lr": w.lr, "wd": w.wd,
            **({"clip": {"max_norm": args.clip_norm, "norm_type": 2.0, "fused": "dmuon_step_clipped"}}
               if getattr(args, "clip_norm", None) is not None else {}),
            "parallelism": (f"dedicated owners x{world}" if getattr(args, "owners", False) else f"replicas x{world}")
            if world > 1 else "single GPU",
            "l2": f"no flush: each step touches {w.elements() * 2 * 7 / 1e9:.1f} GB "
                  f"(inputs alone {w.elements() * 2 * 3 / 1e9:.1f} GB) >> 126 MB L2"}


def e2e_groups(w, size: int = 16, edge: int = 2):
    """Matrix indices in groups of one oriented shape, at most `size` each.

    The first group's host-to-device copy and the last group's read-back
    overlap no compute, so both are `edge` matrices of the class with the
    smallest matrices (when it has enough members); the rest follow in groups
    of `size`."""
    by_class = {}
    for i, (r, c) in enumerate(w.shapes):
        by_class.setdefault((min(r, c), max(r, c)), []).append(i)
    small = min(by_class, key=lambda k: k[0] * k[1])
    head, tail = [], []
    if len(by_class[small]) > 2 * edge:
        head, tail = by_class[small][:edge], by_class[small][-edge:]
        by_class[small] = by_class[small][edge:-edge]
    groups = [head] if head else []
    for idx in by_class.values():
        for k in range(0, len(idx), size):
            groups.append(idx[k:k + size])
    if tail:
        groups.append(tail)
    return groups


def run_e2e(args, w, ps, gs, bs, shapes, stream, dev, world):
    """Same metric through the public API with host buffers.

    Every step copies all gradients host->device from pinned memory and reads
    all updated parameters back.  The set is split into groups of one shape;
    group j's gradients travel on a copy stream while earlier groups compute,
    its dmuon_step call runs on the compute stream, and its parameters return
    on a second copy stream, so PCIe traffic in both directions overlaps the
    tensor-core work (only the small first group's copy in and the small last
    group's copy out overlap nothing).
    """
    import newton_schulz_grad_b200 as nsg
    try:
        g_host = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in gs]
        p_host = [torch.empty(p.shape, dtype=p.dtype, pin_memory=True) for p in ps]
    except RuntimeError as exc:
        return {"value": None, "unit": "matrices/s", "unavailable": f"pinned allocation failed: {exc}"}
    for gh, g in zip(g_host, gs):
        gh.copy_(g)
    h2d = sum(g.numel() * g.element_size() for g in gs)
    d2h = sum(p.numel() * p.element_size() for p in ps)
    groups = e2e_groups(w, size=args.e2e_group)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    done_compute = [None] * len(groups)  # last step's compute of group j (frees its gradients)
    done_copy_out = [None] * len(groups)  # last step's read-back of group j (frees its params)

    def e2e_step():
        for j, idx in enumerate(groups):
            ev_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if done_compute[j] is not None:
                    s_in.wait_event(done_compute[j])
                for i in idx:
                    gs[i].copy_(g_host[i], non_blocking=True)
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if done_copy_out[j] is not None:
                stream.wait_event(done_copy_out[j])
            nsg.dmuon_step([ps[i] for i in idx], [gs[i] for i in idx], [bs[i] for i in idx], lr=w.lr,
                           momentum=w.momentum, nesterov=w.nesterov, ns_steps=w.ns_steps, wd=w.wd,
                           stream=stream)
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            done_compute[j] = ev_c
            ev_o = torch.cuda.Event()
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                for i in idx:
                    p_host[i].copy_(ps[i], non_blocking=True)
                ev_o.record(s_out)
            done_copy_out[j] = ev_o

    e2e_step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(max(1, args.e2e_steps)):
        e2e_step()
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    e1.synchronize()
    wall = (time.perf_counter() - t0) / max(1, args.e2e_steps)
    ms = reduce_max(e0.elapsed_time(e1) / max(1, args.e2e_steps), dev)
    return {"value": round(aggregate_value(w.count, world, ms), 3), "unit": "matrices/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "wall_ms_per_step": round(wall * 1e3, 3), "steps": max(1, args.e2e_steps),
            "api": "newton_schulz_grad_b200.dmuon_step (C ABI dmuon_step) per group of one shape, "
                   "pinned host buffers, copies on two side streams overlapping compute",
            "groups": len(groups)}


# ---------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 oracle on the host cores: each step one sampled matrix, the
    samples rotating through the launch classes; extrapolated to the set."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = workloads.get(args.workload)
    samples = class_samples(w)
    for i in range(max(args.warmup, 0)):
        oracle_matrix_seconds(w, samples[i % len(samples)][1])
    times = {}
    for i in range(args.steps):
        key, idx, cnt = samples[i % len(samples)]
        times.setdefault(key, []).append(oracle_matrix_seconds(w, idx))
    # classes not reached in K steps: extrapolate by flops from the measured ones
    rate = statistics.mean(t / (3 * k[0] ** 2 * k[1] + k[0] ** 3)
                           for k, ts in times.items() for t in ts)
    total = 0.0
    for key, idx, cnt in samples:
        t = statistics.mean(times[key]) if key in times else rate * (3 * key[0] ** 2 * key[1] + key[0] ** 3)
        total += t * cnt
    value = w.count / total
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "matrices/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total * 1e3, 1), "extrapolated": True,
            "seconds_per_matrix": {f"{k[0]}x{k[1]}": round(statistics.mean(ts), 4) for k, ts in times.items()},
            "extrapolation": "ms_per_step is the oracle's time for the whole set, summed from the measured "
                             "seconds per matrix of each launch class (classes not sampled: by flops), "
                             "not a timed region",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args, world),
            "cpu_baseline": {"value": round(value, 5), "unit": "matrices/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": "each step one matrix, rotating over the launch classes; "
                                       f"extrapolated to the {w.count}-matrix set by class counts"},
            "e2e": {"value": round(value, 5), "unit": "matrices/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_lib_chain(args):
    """Comparison only: the workload's Newton-Schulz chain (5 iterations of
    G = X X^T, P = b G + c G G, X <- a X + P X on the oriented, normalised
    matrices, batches of 16 per shape) through a library's bf16 GEMMs, timed
    with CUDA events.  `torch`: torch.bmm / baddbmm (cuBLAS); `quack`: quack's
    symmetric and add GEMMs (the kernels the DMuon pages name for SM90 and
    later).  Nothing here is on the library's path and nothing is checked for
    parity; the line sets the chain's time beside this library's chain
    (the `ns_chain_tflops` of the default run counts the same flops)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    steps = w.ns_steps if args.ns_steps is None else args.ns_steps
    a, b, c = 3.4445, -4.7750, 2.0315
    gen = torch.Generator(device=dev).manual_seed(11)
    by_class = {}
    for r, cc in w.shapes:
        key = (min(r, cc), max(r, cc))
        by_class[key] = by_class.get(key, 0) + 1
    batches = []
    for (m, n), cnt in by_class.items():
        for k in range(0, cnt, 16):
            X = torch.randn(min(16, cnt - k), m, n, generator=gen, device=dev)
            X = (X / X.flatten(1).norm(dim=1).view(-1, 1, 1)).to(torch.bfloat16)
            batches.append(X)
    if args.lib == "quack":
        from quack.gemm_interface import gemm_add, gemm_symmetric

        def chain(X):
            for _ in range(steps):
                G = gemm_symmetric(X, X.mT)
                P = gemm_symmetric(G, G, C=G, alpha=c, beta=b)
                X = gemm_add(P, X, C=X, alpha=1.0, beta=a, tuned=False)
            return X
    else:
        def chain(X):
            for _ in range(steps):
                G = torch.bmm(X, X.mT)
                P = torch.baddbmm(G, G, G, beta=b, alpha=c)
                X = torch.baddbmm(X, P, X, beta=a, alpha=1.0)
            return X
    for X in batches:                 # warm-up (and compilation, for quack)
        chain(X)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = max(1, args.steps)
    clocks = ClockSampler(0)
    clocks.start()
    e0.record()
    for _ in range(reps):
        for X in batches:
            chain(X)
    e1.record()
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / reps
    flops = w.ns_flops() * steps / max(1, w.ns_steps)
    print(json.dumps({"stage": "lib_chain", "lib": args.lib, "workload": w.name, "ns_steps": steps,
                      "chain_ms": round(ms, 3), "matrices_per_s": round(w.count / (ms / 1e3), 2),
                      "ns_tflops": round(flops / (ms / 1e3) / 1e12, 1), "reps": reps, "clocks": clk,
                      "note": "Newton-Schulz chain only (no momentum, normalisation or update); "
                              "flops counted as 3 m^2 n + m^3 per matrix and iteration"}), flush=True)


def run_stage(args):
    """One kernel through its stage call (bf16), e.g. for an ncu capture of a small case."""
    import newton_schulz_grad_b200 as nsg
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    b, m, n = args.batch, args.m, args.n
    gen = torch.Generator(device=dev).manual_seed(7)
    bf = torch.bfloat16
    if args.stage == "gram":
        X = torch.randn(b, m, n, generator=gen, device=dev).to(bf)
        out = torch.empty(b, m, m, dtype=bf, device=dev)
        run = lambda: nsg.dmuon_gram(X, out)  # noqa: E731
        flops, nbytes = b * m * m * n, 2 * b * (m * n + m * m)
    elif args.stage == "poly":
        G = torch.randn(b, m, m, generator=gen, device=dev)
        G = ((G + G.transpose(1, 2)) / (2 * math.sqrt(m))).to(bf).contiguous()
        out = torch.empty_like(G)
        run = lambda: nsg.dmuon_gram_poly(G, out, -4.775, 2.0315)  # noqa: E731
        flops, nbytes = b * m ** 3, 2 * b * 2 * m * m
    elif args.stage in ("apply", "lib_apply"):
        P = (torch.randn(b, m, m, generator=gen, device=dev) / math.sqrt(m)).to(bf)
        X = torch.randn(b, m, n, generator=gen, device=dev).to(bf)
        out = torch.empty_like(X)
        if args.stage == "apply":
            # as in the step: the tensor path's p(G) carries a I, so its applies add no a X
            run = lambda: nsg.dmuon_poly_apply(P, X, out, 0.0)  # noqa: E731
        elif args.lib == "quack":  # comparison only: the same product through quack
            from quack.gemm_interface import gemm_add
            run = lambda: gemm_add(P, X, C=X, out=out, alpha=1.0, beta=3.4445, tuned=False)  # noqa: E731
        else:  # comparison only: the same product through torch (cuBLAS)
            run = lambda: torch.baddbmm(X, P, X, beta=3.4445, alpha=1.0, out=out)  # noqa: E731
        flops, nbytes = 2 * b * m * m * n, 2 * b * (m * m + 2 * m * n)
    elif args.stage == "step":
        # a whole step over `batch` m x n matrices (rows x cols as given): the
        # way to reach the apply with the fused update (its last launch)
        steps = 1 if args.ns_steps is None else args.ns_steps
        ps = [(torch.randn(m, n, generator=gen, device=dev) * 0.02).to(bf) for _ in range(b)]
        gs = [torch.randn(m, n, generator=gen, device=dev).to(bf) for _ in range(b)]
        bs = [torch.zeros(m, n, dtype=bf, device=dev) for _ in range(b)]
        run = lambda: nsg.dmuon_step(ps, gs, bs, ns_steps=steps)  # noqa: E731
        lo, hi = min(m, n), max(m, n)
        flops, nbytes = b * steps * (3 * lo * lo * hi + lo ** 3), 0
    elif args.stage == "clip":
        # standalone clipping of `batch` m x n gradients: norm pass + in-place scale
        gs = [torch.randn(m, n, generator=gen, device=dev).to(bf) for _ in range(b)]
        run = lambda: nsg.dmuon_clip_grad_norm(gs, 1.0)  # noqa: E731
        flops, nbytes = 0, 2 * b * m * n * 3
    elif args.stage == "momentum":
        g = torch.randn(m, n, generator=gen, device=dev).to(bf)
        buf = torch.randn(m, n, generator=gen, device=dev).to(bf)
        x0 = torch.empty_like(g)
        run = lambda: nsg.dmuon_momentum(buf, g, x0, 0.95, True)  # noqa: E731
        flops, nbytes = 0, 8 * m * n
    else:
        p = torch.randn(m, n, generator=gen, device=dev).to(bf)
        o = torch.randn(m, n, generator=gen, device=dev).to(bf)
        run = lambda: nsg.dmuon_update(p, o, 0.02, 0.0)  # noqa: E731
        flops, nbytes = 0, 6 * m * n
    for _ in range(max(args.warmup, 0)):
        run()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    nsg.dmuon_profile_start()
    e0.record()
    for _ in range(args.steps):
        run()
    e1.record()
    e1.synchronize()
    kstats = nsg.dmuon_profile_stop()
    ms = e0.elapsed_time(e1) / args.steps
    if nsg.dmuon_stream_status() != nsg.DMUON_OK:
        raise RuntimeError("stage call failed")
    kernels = {k: {"ms": round(v["total_ms"] / args.steps, 4),
                   "GB/s": round(v["bytes"] / (v["total_ms"] / 1e3) / 1e9, 1) if v["bytes"] else None}
               for k, v in kstats.items()}
    print(json.dumps({"stage": args.stage, "batch": b, "m": m, "n": n, "ms": round(ms, 4), "kernels": kernels,
                      "tflops": round(flops / (ms / 1e3) / 1e12, 1) if flops else None,
                      "GB/s": round(nbytes / (ms / 1e3) / 1e9, 1) if nbytes else None}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.stage == "lib_chain":
        run_lib_chain(args)
        return
    if args.stage:
        run_stage(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

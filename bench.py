#!/usr/bin/env python
"""Benchmark of the fused attention-KL forward + recompute backward on B200.

One step = one pass of the whole path over one batch of synthetic input:
streamkl_fwd (L, LSE1, LSE2) then streamkl_bwd (dQ1, dK1, dQ2, dK2).  The
default workload is the forward+backward configuration B1 H32 N=16384
d1=d2=128 causal with dL = 1/(B*H*NQ).  Inputs (537 MB) are larger than the
126 MB L2, so no flush is needed between steps.

Prints one JSON line (rank 0).  With torchrun (N > 1) every rank runs an
independent replica of the workload (weak scaling: the path has no data
exchange), or with ``--shard heads`` a contiguous range of the workload's
B*H heads (strong scaling: the heads are independent problems); the timed
region is bracketed by barriers and the max over ranks is taken.

``--impl reference`` times the fp64 CPU oracle on the host cores on a
bounded sample of the same workload (the only other place this file runs the
oracle is the ``cpu_baseline`` leg).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

from attention_kl_distillation_b200.inputs import WORKLOADS, Workload, bf16_bits, make_inputs  # noqa: E402

METRIC = "fused attn-KL fwd / fwd+bwd TFLOP/s and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_TFLOPS = 1590.0
FALLBACK_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="fwdbwd16k")
    ap.add_argument("--phase", choices=["auto", "fwd", "fwdbwd"], default="auto")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (smaller cases for profiling; not a bench line)")
    ap.add_argument("--nq", type=int, default=None,
                    help="override NQ (small-NQ forward cases; not a bench line)")
    ap.add_argument("--splitk", action="store_true",
                    help="run the forward through streamkl_fwd_splitk with the suggested split")
    ap.add_argument("--table", action="store_true",
                    help="instead of the bench line, one JSON line per recipe (median of >= 10 "
                         "timed calls, >= 5 for long64k, after 3 warm-ups)")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: every rank runs the whole workload (replicas, weak scaling) or "
                         "a contiguous range of its B*H heads (heads, strong scaling)")
    ap.add_argument("--bwd-algo", default="auto",
                    choices=["auto", "fused", "split", "fused_key_tiles", "fused_query_tiles",
                             "fused_sides"],
                    help="streamkl_bwd algorithm (process-wide setting of the library)")
    ap.add_argument("--compare-bwd", action="store_true",
                    help="instead of the bench line, one JSON line per backward algorithm on the "
                         "workload (median of --steps calls after --warmup): the measurement the "
                         "library's AUTO selection rests on")
    ap.add_argument("--need", default="1111",
                    help="which of dQ1 dK1 dQ2 dK2 the backward returns (e.g. 0101 = dK only)")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- helpers
def peaks():
    f = ROOT / "MEASURED_PEAKS.json"
    try:
        d = json.loads(f.read_text())
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_TFLOPS, FALLBACK_GBS, "fallback"


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def workload_desc(w: Workload, phase: str) -> dict:
    return {
        "workload": (f"{w.name}: B{w.B} H{w.H} NQ={w.NQ} NK={w.NK} d1={w.d1} d2={w.d2} "
                     f"{'causal' if w.causal else 'non-causal'}, "
                     f"{'forward+backward' if phase == 'fwdbwd' else 'forward'}"),
        "B": w.B, "H": w.H, "NQ": w.NQ, "NK": w.NK, "d1": w.d1, "d2": w.d2,
        "causal": w.causal, "phase": phase,
        "student": w.student + (f" sigma={w.sigma}" if w.student == "perturb" else ""),
        "l2": f"inputs {w.input_bytes() / 1e6:.0f} MB vs 126 MB L2; "
              + ("no flush (inputs larger than L2)" if w.input_bytes() > 126e6
                 else "L2 flushed between steps"),
    }


def run_config(args, w: Workload, phase: str, world: int, nsplit=None) -> dict:
    """The `config` object of a bench line; the reference arm prints the same one."""
    if args.shard == "heads":
        par = f"heads{world} (contiguous ranges of the B*H heads per GPU, no collective)"
    else:
        par = f"dp{world} (independent replicas, no collective)"
    return {**workload_desc(w, phase), **({"need": args.need} if args.need != "1111" else {}),
            **({"splitk": nsplit} if nsplit else {}), "parallelism": par}


# The sources a profiled kernel is built from: its own file and the two shared headers.
PROFILED_SOURCES = {
    "fwd_kernel": "fwd_sm100.cu",
    "fwd_t_kernel": "fwd_t_sm100.cu",
    "bwd_fused_key_tiles_kernel": "bwd_sm100.cu",
    "bwd_fused_query_tiles_kernel": "bwd_qt_sm100.cu",
    "bwd_split_kernel": "bwd_split_sm100.cu",
    "bwd_fused_sides_kernel": "bwd_side_sm100.cu",
}


def kernel_sources_sha1(kernel_file: str) -> str:
    import hashlib
    h = hashlib.sha1()
    csrc = ROOT / "attention_kl_distillation_b200" / "csrc"
    for name in (kernel_file, "kernels.h", "sm100.cuh"):
        f = csrc / name
        h.update(f.name.encode())
        h.update(f.read_bytes())
    return h.hexdigest()


def profiled_traffic(profile: str):
    """DRAM bytes per full launch recorded in profiles/<profile>, or None when the
    kernel's sources changed since that ncu capture."""
    import re
    f = ROOT / "profiles" / profile
    if not f.exists():
        return None
    kernel = next((k for k in sorted(PROFILED_SOURCES, key=len, reverse=True)
                   if profile.startswith(k + "_")), None)
    if kernel is None:
        return None
    text = f.read_text()
    m1 = re.search(r"source-sha1: ([0-9a-f]{40})", text)
    m2 = re.search(r"dram-bytes-per-full-launch: (\d+)", text)
    if not (m1 and m2) or m1.group(1) != kernel_sources_sha1(PROFILED_SOURCES[kernel]):
        return None
    return int(m2.group(1))


DATASHEET_BF16_TFLOPS = 2250.0  # dense (not 2:4 sparse) bf16 per GPU


def peak_ratios(step_tf: float, fwd_tf: float, clk: dict, dev) -> dict:
    """The per-GPU step and forward rates against three denominators: the dense bf16
    datasheet figure, the measured cuBLAS figure, and the clock-normalised tensor peak
    (SMs x 8192 FLOP/clk x the median SM clock sampled during the timed region)."""
    peak, _, _ = peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clk or {}).get("sm_mhz")
    clock_peak = sms * 8192 * mhz * 1e6 / 1e12 if mhz else None
    out = {}
    for name, v in (("step", step_tf), ("fwd", fwd_tf)):
        out[name] = {"datasheet_dense_bf16": v / DATASHEET_BF16_TFLOPS, "measured_bf16": v / peak,
                     "clock_normalised": (v / clock_peak) if clock_peak else None}
    out["clock_peak_tflops"] = clock_peak
    return out


def step_flops(w: Workload, phase: str) -> int:
    return w.fwd_flops() + (w.bwd_flops() if phase == "fwdbwd" else 0)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def finish(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) != 8:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except Exception:
                continue
        inside = [r for r in rows if self.t0 - 0.05 <= r[0] <= self.t1 + 0.05] or rows[-3:]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in inside for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {
            "sm_mhz": statistics.median(r[1] for r in inside) if inside else None,
            "sm_max_mhz": max(r[2] for r in inside) if inside else None,
            "reasons": reasons,
            "samples": len(inside),
        }


# --------------------------------------------------------------------------- oracle legs
def oracle_sample_run(w: Workload, phase: str, R: int, nthreads: int, seed: int):
    """Run the oracle on a bounded sample of the workload: the first R query rows of head 0
    with the keys they can see (for a causal square problem that prefix is itself the problem
    NQ = NK = R; otherwise R rows against all keys).  Returns (seconds, algorithmic FLOPs)."""
    from oracle import oracle as O
    orc = O.default()
    sub = w.with_(B=1, H=1, NQ=R, NK=R if (w.causal and w.NQ == w.NK) else w.NK)
    Q1, K1, Q2, K2 = (bf16_bits(t) for t in make_inputs(sub, seed=seed))
    t0 = time.perf_counter()
    if phase == "fwdbwd":
        orc.fwd_all(Q1, K1, Q2, K2, causal=sub.causal, nthreads=nthreads)
        g = np.full((1, sub.NQ), 1.0 / (w.B * w.H * w.NQ))
        orc.bwd_heads(Q1, K1, Q2, K2, [0], g, causal=sub.causal, nthreads=nthreads)
    else:
        orc.fwd_all(Q1, K1, Q2, K2, causal=sub.causal, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return dt, step_flops(sub, phase), sub


def cpu_baseline(w: Workload, phase: str, target_s: float) -> dict:
    nthreads = host_threads()
    R = 512
    dt, fl, sub = oracle_sample_run(w, phase, R, nthreads, w.seed)
    if dt < target_s / 4:
        scale = (target_s / max(dt, 1e-3)) ** (0.5 if sub.NK == sub.NQ else 1.0)
        R = int(min(w.NQ, max(R, R * scale * 0.9)) // 64 * 64)
        dt, fl, sub = oracle_sample_run(w, phase, R, nthreads, w.seed)
    pps = sub.visible_pairs() / dt
    # one thread, on a smaller prefix (about a tenth of the threaded sample's time)
    R1 = max(64, int(sub.NQ * (0.1 / nthreads) ** (0.5 if sub.NK == sub.NQ else 1.0)) // 64 * 64)
    dt1, _, sub1 = oracle_sample_run(w, phase, min(R1, sub.NQ), 1, w.seed)
    return {
        "value": fl / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
        "seconds": dt,
        "sample": (f"first {sub.NQ} query rows of one head ({sub.NK} keys, "
                   f"{'causal' if sub.causal else 'non-causal'}) of the {w.name} recipe, "
                   f"{'forward+backward' if phase == 'fwdbwd' else 'forward'}; "
                   f"{fl / 1e9:.1f} GFLOP algorithmic"),
        # rows are independent and the oracle's cost is linear in the visible pairs
        "pairs_per_s": pps,
        "full_config_s_extrapolated": w.visible_pairs() / pps,
        "single_thread": {"pairs_per_s": sub1.visible_pairs() / dt1, "sample_rows": sub1.NQ,
                          "seconds": dt1},
    }


def run_reference(args, w: Workload, phase: str):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    nthreads = host_threads()
    budget = 150.0 / max(1, args.steps + args.warmup)  # seconds of oracle work per step
    R = 512
    dt, fl, sub = oracle_sample_run(w, phase, R, nthreads, w.seed)
    if dt < budget / 2:
        scale = (budget / max(dt, 1e-3)) ** (0.5 if sub.NK == sub.NQ else 1.0)
        R = int(min(w.NQ, max(R, R * scale * 0.8)) // 64 * 64)
    times = []
    for s in range(args.warmup + args.steps):
        dt, fl, sub = oracle_sample_run(w, phase, R, nthreads, w.seed + s)
        if s >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = fl * len(times) / total / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference", "config": run_config(args, w, phase, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"first {sub.NQ} query rows of one head per step "
                                   f"({sub.NK} keys), {fl / 1e9:.1f} GFLOP algorithmic"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- per-recipe table
def run_table(args):
    """Per recipe and phase: median CUDA-event time of the library calls, TFLOP/s, rows/s and
    the fraction of the measured bf16 peak (the reporting the measurement plan asks for)."""
    import attention_kl_distillation_b200 as skl
    from attention_kl_distillation_b200 import binding
    peak, _, _ = peaks()
    dev = torch.device("cuda", 0)
    for name in ("tiny", "causal4k", "sparse_student", "long64k", "fwdbwd16k"):
        w = WORKLOADS[name]
        Q1, K1, Q2, K2 = (t.to(dev) for t in make_inputs(w))
        L, A, B = (torch.empty((w.B, w.H, w.NQ), device=dev) for _ in range(3))
        dL = torch.full((w.B, w.H, w.NQ), 1.0 / (w.B * w.H * w.NQ), device=dev)
        grads = tuple(torch.empty_like(t) for t in (Q1, K1, Q2, K2)) if w.backward else None
        ws = (torch.empty(binding.workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal),
                          dtype=torch.uint8, device=dev) if w.backward else None)
        calls = [("fwd", None, lambda: skl.fwd(Q1, K1, Q2, K2, causal=w.causal, out=(L, A, B)),
                  w.fwd_flops())]
        ns = binding.splitk_suggest(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal)
        if ns > 1 and name != "tiny":
            fws = torch.empty(max(256, binding.splitk_workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, ns)),
                              dtype=torch.uint8, device=dev)
            calls.append((f"fwd_splitk{ns}", None,
                          lambda: skl.fwd_splitk(Q1, K1, Q2, K2, causal=w.causal, nsplit=ns,
                                                 workspace=fws, out=(L, A, B)), w.fwd_flops()))
        if w.backward:
            for algo in ("fused_key_tiles", "fused_query_tiles", "fused_sides", "split"):
                calls.append((f"bwd_{algo}", algo,
                              lambda: skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal,
                                              workspace=ws, out=grads), w.bwd_flops()))
            # one gradient side (teacher fixed: dQ2, dK2; student fixed: dQ1, dK1): both S
            # products are recomputed, the contractions of the other side are not done
            pairs = w.bwd_flops() / (6 * (w.d1 + w.d2))
            for side, keep, d in (("student", (2, 3), w.d2), ("teacher", (0, 1), w.d1)):
                outs = tuple(g if i in keep else None for i, g in enumerate(grads))
                calls.append((f"bwd_{side}_side", None,
                              lambda outs=outs: skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal,
                                                        workspace=ws, out=outs),
                              pairs * (2 * (w.d1 + w.d2) + 4 * d)))
        n = 5 if name == "long64k" else 10
        for phase, algo, fn, fl in calls:
            binding.set_bwd_algorithm(algo or args.bwd_algo)
            for _ in range(3):
                fn()
            times = []
            for _ in range(n):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            tf = fl / (ms * 1e-3) / 1e12
            print(json.dumps({"recipe": name, "phase": phase, "calls": n, "median_ms": ms,
                              "tflops": tf, "frac_of_measured_bf16": tf / peak,
                              "rows_per_s": w.BH * w.NQ / (ms * 1e-3),
                              "mufu_ceiling_frac_of_clock_peak": (w.d1 + w.d2) / 512}), flush=True)
        if skl.query_device_status() != 0:
            raise RuntimeError("device status reported an error")
        del Q1, K1, Q2, K2, L, A, B, dL, grads, ws, calls
        torch.cuda.empty_cache()


def run_compare_bwd(args, w: Workload):
    """Times streamkl_bwd with each algorithm on one workload (same inputs, same saved
    state), so that the fused/split choice can be set from a measurement."""
    import attention_kl_distillation_b200 as skl
    from attention_kl_distillation_b200 import binding
    peak, _, _ = peaks()
    dev = torch.device("cuda", 0)
    Q1, K1, Q2, K2 = (t.to(dev) for t in make_inputs(w))
    L, A, B = skl.fwd(Q1, K1, Q2, K2, causal=w.causal)
    dL = torch.full((w.B, w.H, w.NQ), 1.0 / (w.B * w.H * w.NQ), device=dev)
    grads = tuple(torch.empty_like(t) for t in (Q1, K1, Q2, K2))
    ws = torch.empty(binding.workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal),
                     dtype=torch.uint8, device=dev)
    acc_bytes = w.BH * w.NQ * (w.d1 + w.d2) * 4
    for algo in ("fused_query_tiles", "fused_sides", "fused_key_tiles", "split"):
        binding.set_bwd_algorithm(algo)
        for _ in range(max(1, args.warmup)):
            skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal, workspace=ws, out=grads)
        times = []
        for _ in range(max(1, args.steps)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal, workspace=ws, out=grads)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        if skl.query_device_status() != 0:
            raise RuntimeError("device status reported an error")
        ms = statistics.median(times)
        tf = w.bwd_flops() / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": workload_desc(w, "fwdbwd")["workload"], "algorithm": algo,
                          "calls": len(times), "median_ms": ms, "tflops": tf,
                          "frac_of_measured_bf16": tf / peak,
                          "fp32_accumulator_bytes": acc_bytes}), flush=True)
    binding.set_bwd_algorithm("auto")
    print(json.dumps({"auto_selects": binding.bwd_algorithm_for(w.B, w.H, w.NQ, w.NK, w.d1, w.d2,
                                                                w.causal)}), flush=True)


# --------------------------------------------------------------------------- our path
def main(argv=None):
    args = parse_args(argv)
    if args.table:
        return run_table(args)
    w = WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    if args.nq:
        w = w.with_(NQ=args.nq)
    phase = args.phase if args.phase != "auto" else ("fwdbwd" if w.backward else "fwd")
    if args.impl == "reference":
        return run_reference(args, w, phase)
    if args.compare_bwd:
        return run_compare_bwd(args, w)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import attention_kl_distillation_b200 as skl
    from attention_kl_distillation_b200 import binding
    from attention_kl_distillation_b200.parallel import max_over_ranks
    binding.set_bwd_algorithm(args.bwd_algo)

    dev = torch.device("cuda", local)
    full_w = w
    if args.shard == "heads":
        # strong scaling: this rank's contiguous range of the B*H heads, as a B = 1 problem
        from attention_kl_distillation_b200.parallel import head_shard, shard_heads
        if world > w.BH:
            raise SystemExit(f"--shard heads needs at most {w.BH} ranks")
        a, b = head_shard(w.BH, world, rank)
        cpu_ins = [shard_heads(t, world, rank) for t in make_inputs(w)]
        w = w.with_(B=1, H=b - a)
    else:
        cpu_ins = make_inputs(w, seed=w.seed + rank)  # independent replica per rank
    Q1, K1, Q2, K2 = (t.to(dev) for t in cpu_ins)
    g = 1.0 / (full_w.B * full_w.H * full_w.NQ)  # the mean over the whole job's rows
    dL = torch.full((w.B, w.H, w.NQ), g, device=dev)
    L, A, B = (torch.empty((w.B, w.H, w.NQ), device=dev) for _ in range(3))
    need = tuple(c == "1" for c in args.need)
    grads = tuple(torch.empty_like(t) if n else None for t, n in zip((Q1, K1, Q2, K2), need))
    ws = torch.empty(binding.workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal),
                     dtype=torch.uint8, device=dev)
    nsplit = None
    if args.splitk:
        nsplit = binding.splitk_suggest(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal)
        fws = torch.empty(max(256, binding.splitk_workspace_size(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, nsplit)),
                          dtype=torch.uint8, device=dev)

    def fwd_call():
        if nsplit is None:
            skl.fwd(Q1, K1, Q2, K2, causal=w.causal, out=(L, A, B))
        else:
            skl.fwd_splitk(Q1, K1, Q2, K2, causal=w.causal, nsplit=nsplit, workspace=fws, out=(L, A, B))

    def step():
        fwd_call()
        if phase == "fwdbwd":
            skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal, workspace=ws, out=grads)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if skl.query_device_status() != 0:
        raise RuntimeError("device status reported an error after warm-up")

    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    launches0 = skl.launch_count()
    clocks.mark_start()
    t_start.record(stream)
    for k in range(args.steps):
        ev[k][0].record(stream)
        fwd_call()
        ev[k][1].record(stream)
        if phase == "fwdbwd":
            skl.bwd(dL, Q1, K1, Q2, K2, L, A, B, causal=w.causal, workspace=ws, out=grads)
        ev[k][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier()
    launches = skl.launch_count() - launches0
    clk = clocks.finish()
    if skl.query_device_status() != 0:
        raise RuntimeError("device status reported an error in the timed region")

    total_ms = max_over_ranks(t_start.elapsed_time(t_end), device=dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) if phase == "fwdbwd" else 0.0
    fl_step = step_flops(w, phase)
    # whole-job work per step: every rank's replica, or the whole workload once when sharded
    job_fl_step = step_flops(full_w, phase) if args.shard == "heads" else world * fl_step
    value = job_fl_step * args.steps / (total_ms * 1e-3) / 1e12
    peak, hbm, src = peaks()
    fwd_tf = w.fwd_flops() / (fwd_ms * 1e-3) / 1e12
    bwd_tf = w.bwd_flops() / (bwd_ms * 1e-3) / 1e12 if bwd_ms > 0 else None
    full_size = w == WORKLOADS[args.workload] and args.need == "1111" and not args.heads
    algo = binding.bwd_algorithm_for(w.B, w.H, w.NQ, w.NK, w.d1, w.d2, w.causal)
    if phase == "fwdbwd" and bwd_ms >= fwd_ms:
        dom = {"kernel": f"streamkl_bwd, {algo} (prep + main + convert kernels)",
               "achieved": bwd_tf, "flops_per_launch": w.bwd_flops(), "ms": bwd_ms,
               "traffic": profiled_traffic(f"bwd_{algo}_kernel_{w.name}_h8.md") if full_size else None}
    else:
        dom = {"kernel": "streamkl_fwd_kernel", "achieved": fwd_tf,
               "flops_per_launch": w.fwd_flops(), "ms": fwd_ms,
               "traffic": profiled_traffic(f"fwd_kernel_{w.name}_h8.md") if full_size else None}
    roofline = {"bound": "tensor", "achieved": dom["achieved"], "peak": peak, "unit": UNIT,
                "frac": dom["achieved"] / peak, "traffic": dom["traffic"], "kernel": dom["kernel"],
                "flops_per_launch": dom["flops_per_launch"], "ms_per_launch": dom["ms"],
                "peak_source": f"{src} dense bf16 (burst)"}
    if phase == "fwd" and w.NQ <= 32:
        # few query rows: the transposed kernel streams K1 and K2 once per head; the
        # algorithmic bytes are the inputs read once plus the three fp32 row vectors
        alg = w.input_bytes() + 3 * w.BH * w.NQ * 4
        gbs = alg / (fwd_ms * 1e-3) / 1e9
        captured = args.workload == "long64k" and w.NQ == 1 and nsplit is not None and not args.heads
        roofline = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                    "traffic": profiled_traffic("fwd_t_kernel_long64k_nq1.md") if captured else None,
                    "kernel": "streamkl_fwd_t_kernel" + (" + streamkl_fwd_merge_kernel" if nsplit else ""),
                    "bytes_per_launch": alg, "ms_per_launch": fwd_ms, "peak_source": f"{src} HBM copy"}

    # End to end through the public API: every step copies its inputs from pinned
    # host memory and reads its result (the per-row KL) back to the host.  The copy
    # of step k+1's inputs runs on a side stream into the other of two device
    # buffers while step k computes (the loader prefetch a training loop has); the
    # gradients stay on the device, where an optimizer would consume them.
    e2e = None
    if not args.no_e2e:
        h_in = [t.pin_memory() for t in cpu_ins]
        h_dL = dL.cpu().pin_memory()
        h_L = torch.empty((w.B, w.H, w.NQ), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in) + h_dL.numel() * 4
        d2h = h_L.numel() * 4
        bufs = [[torch.empty_like(t, device=dev) for t in cpu_ins] + [torch.empty_like(dL)]
                for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n, start=None):
            """n steps; returns nothing.  Copies for step k go to buffer k % 2."""
            def issue_copy(k):
                b = k % 2
                with torch.cuda.stream(copy_stream):
                    if k >= 2:
                        copy_stream.wait_event(used[b])  # step k-2 is done with the buffer
                    for dst, src in zip(bufs[b], h_in + [h_dL]):
                        dst.copy_(src, non_blocking=True)
                    copied[b].record(copy_stream)
            if start is not None:
                copy_stream.wait_event(start)
            issue_copy(0)
            for k in range(n):
                if k + 1 < n:
                    issue_copy(k + 1)
                b = k % 2
                stream.wait_event(copied[b])
                d_in = [t.detach().requires_grad_(phase == "fwdbwd") for t in bufs[b][:4]]
                if phase == "fwdbwd":
                    Lx = skl.streamkl(*d_in, causal=w.causal)
                    Lx.backward(bufs[b][4])
                else:
                    Lx, _, _ = skl.fwd(*d_in, causal=w.causal)
                h_L.copy_(Lx.detach(), non_blocking=True)
                used[b].record(stream)

        e2e_run(2)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ke = max(3, args.steps)  # every timed step copies its inputs in and its result out
        e0.record(stream)
        e2e_run(ke, start=e0)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
        e2e = {"value": job_fl_step * ke / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / ke, "api": "attention_kl_distillation_b200.streamkl",
               "pipeline": "inputs of step k+1 copied on a side stream during step k (step 0's copy is not overlapped); result L read back every step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(full_w, phase, args.cpu_seconds)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) teacher, student = teacher + noise; bf16)",
        "config": run_config(args, full_w, phase, world, nsplit),
        "pct_of_peak": value / world / peak,
        "peak_ratios": peak_ratios(value / world, fwd_tf, clk, dev),
        **({"heads_per_rank": [head_shard(full_w.BH, world, r)[1] - head_shard(full_w.BH, world, r)[0]
                               for r in range(world)]} if args.shard == "heads" else {}),
        "fwd": {"ms": fwd_ms, "tflops": fwd_tf, "frac_of_peak": fwd_tf / peak,
                "rows_per_s": w.BH * w.NQ / (fwd_ms * 1e-3)},
        "bwd": ({"ms": bwd_ms, "tflops": bwd_tf, "frac_of_peak": bwd_tf / peak}
                if bwd_tf else None),
        "roofline": roofline,
        "mufu_ceiling_frac_of_clock_peak": (w.d1 + w.d2) / 512,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

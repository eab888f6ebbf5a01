#!/usr/bin/env python
"""Benchmark of the block-confined bidirectional selective scan on B200.

One step = one full-block (all-block) training pass of the mixer over one batch
of synthetic input: the forward scan over every token, the reverse scan inside
every block, the fused softplus / exp / skip / combine, and the block-boundary
cache states (every row of the hot path). The default workload is the training
configuration: batch 8, L 4096, D 1536, N 16, block 16, bf16 I/O, fp32 state.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun every rank runs its own batch
(independent sequences, no data-path collective: weak scaling); the timing is
the max over ranks. `--impl reference` times the fp64 CPU oracle instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_ssm_scan_mamba_b200 import inputs as I  # noqa: E402

WORKLOAD = "train"
METRIC = "bidirectional block-scan tokens/s and achieved HBM GB/s vs B200 peak"
SM_COUNT = 148
EX2_PER_CLK_SM = 16          # MUFU.EX2 results per clock per SM (measured 15.9 on this machine)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "train_traffic.json")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "selective_ssm_scan_mamba_b200", "csrc", "*"))):
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def algorithmic_bytes(w, boundary=True, h_out=True) -> int:
    s = 2 if w.io == "bf16" else 4
    n = w.batch * w.L * w.D * s * 3            # x, dt in; y out
    n += w.batch * w.L * w.N * s * 2           # B, C
    n += w.D * w.N * 4 + w.D * 4               # A, Dskip
    if boundary:
        n += w.batch * (w.L // w.K) * w.D * w.N * 4
    if h_out:
        n += w.batch * w.D * w.N * 4
    return n


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = sorted(sm)[len(sm) // 4:] or sm   # drop idle samples at the edges
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- data parallel
def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank scans its own independent batch of sequences (weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(values, device=None):
    """Elementwise max of per-rank timings (the job time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_step(w, world: int) -> int:
    return w.batch * w.L * world


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w, seed, n_seq):
    """Time the fp64 oracle on n_seq of the workload's sequences (all channels)."""
    import oracle
    s = I.make_sequence(seed, n_seq, w.L, w.D, w.N, w.io)
    p = I.make_params(seed, w.D, w.N)
    t0 = time.perf_counter()
    oracle.train_blocks(s["x"], s["dt"], p["A"], s["B"], s["C"], p["Dskip"], w.K)
    dt = time.perf_counter() - t0
    tokens = n_seq * w.L
    return tokens / dt, dt, tokens


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = I.WORKLOADS[WORKLOAD]
    n_seq = 1
    for _ in range(args.warmup):
        oracle_sample(w, w.seed, n_seq)
    times = [oracle_sample(w, w.seed, n_seq)[1] for _ in range(args.steps)]
    per_step = statistics.mean(times)
    value = n_seq * w.L / per_step
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD, "batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N,
                   "block": w.K, "io_dtype": w.io, "parallelism": f"dp{args.gpus}",
                   "sample": f"{n_seq} of {w.batch} sequences per step"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{n_seq} sequence x {w.L} tokens x {w.D} channels per step, single thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU path
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from selective_ssm_scan_mamba_b200 import bdscan

    w = I.WORKLOADS[WORKLOAD]
    seed = rank_seed(w.seed, rank)
    s = I.make_sequence(seed, w.batch, w.L, w.D, w.N, w.io)
    p = I.make_params(w.seed, w.D, w.N)

    def up(a, pin=False):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.pin_memory() if pin else t.to(dev)

    g = {k: up(v) for k, v in s.items()}
    A, Dk = up(p["A"]), up(p["Dskip"])
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device=dev)
    bnd = torch.empty((w.batch, w.L // w.K, w.D, w.N), dtype=torch.float32, device=dev)
    hout = torch.empty((w.batch, w.D, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        bdscan.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, w.K, y=y, boundary=bnd, h_out=hout)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    # timed region: device time with CUDA events on the launching stream; one
    # event pair per launch gives the per-launch duration for the roofline.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    elapsed_ms, launch_ms = max_over_ranks(
        [start.elapsed_time(stop), statistics.mean(a.elapsed_time(b) for a, b in ev)], device=dev)
    ms_per_step = elapsed_ms / args.steps
    tokens_per_step = job_tokens_per_step(w, world)
    value = tokens_per_step / (ms_per_step * 1e-3)

    # end to end through the public call with host buffers: pinned H2D of the
    # step's inputs, the pass, D2H of its outputs (y, boundary states, final state)
    hx = {k: up(v, pin=True) for k, v in s.items()}
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    hb = torch.empty(bnd.shape, dtype=bnd.dtype).pin_memory()
    hh = torch.empty(hout.shape, dtype=hout.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = hy.numel() * hy.element_size() + hb.numel() * hb.element_size() + hh.numel() * hh.element_size()
    dx = {k: torch.empty_like(v, device=dev) for k, v in hx.items()}

    def e2e_step():
        for k in hx:
            dx[k].copy_(hx[k], non_blocking=True)
        bdscan.train_blocks(dx["x"], dx["dt"], A, dx["B"], dx["C"], Dk, w.K, y=y, boundary=bnd, h_out=hout)
        hy.copy_(y, non_blocking=True)
        hb.copy_(bnd, non_blocking=True)
        hh.copy_(hout, non_blocking=True)

    e2e_value = None
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 5))
        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        (te,) = max_over_ranks([e0.elapsed_time(e1)], device=dev)
        e2e_value = tokens_per_step / (te / e2e_steps * 1e-3)

    peaks = load_peaks()
    nbytes = algorithmic_bytes(w)
    hbm_gbs = nbytes / (launch_ms * 1e-3) / 1e9
    ex2 = w.batch * w.L * w.D * w.N
    ex2_rate = ex2 / (launch_ms * 1e-3) / 1e9
    ex2_peak = EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e6 / 1e9
    traffic = None
    if os.path.exists(PROFILE_TRAFFIC):
        pt = json.load(open(PROFILE_TRAFFIC))
        if pt.get("kernel_source_hash") == kernel_source_hash():
            traffic = pt.get("traffic_bytes_per_launch")
    clocks = clk.summary()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_seq = 1
        v, secs, toks = oracle_sample(w, w.seed, n_seq)
        cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{n_seq} of {w.batch} sequences ({toks} tokens, all {w.D} channels), "
                         f"single thread, {secs:.1f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N,
                   "block": w.K, "io_dtype": w.io, "state_dtype": "f32", "outputs": "y + all block-boundary states + final state",
                   "parallelism": f"dp{world}", "l2": "working set 506 MB per step > 126 MB L2 (no flush)"},
        "roofline": {"bound": "alu", "achieved": ex2_rate, "peak": ex2_peak, "unit": "Gex2/s",
                     "frac": ex2_rate / ex2_peak, "traffic": traffic,
                     "peak_source": f"16 MUFU.EX2/clk/SM x {SM_COUNT} SMs x {peaks['sm_max_mhz']:.0f} MHz",
                     "hbm": {"achieved": hbm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": hbm_gbs / peaks["hbm_gbs"], "peak_source": peaks["source"],
                             "algorithmic_bytes_per_launch": nbytes},
                     "kernel_ms": launch_ms},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg (profiling runs)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

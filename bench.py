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
    """Hash of the code the forward scan kernel is compiled from (its device
    sources, with comments and whitespace removed: host-side launch code,
    other kernels and comment edits do not change it)."""
    import re
    h = hashlib.sha256()
    for name in ("bdscan_device.cuh", "bdscan_kernels.cuh"):
        src = open(os.path.join(ROOT, "selective_ssm_scan_mamba_b200", "csrc", name)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update("".join(src.split()).encode())
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
def _oracle_worker(conn, name, seed, n_seq, c0, c1):
    """One process of OraclePool: regenerates its channel slice of the workload
    once, then runs the oracle on it whenever asked."""
    import oracle
    w = I.WORKLOADS[name]
    chans = list(range(c0, c1))
    s = I.make_sequence(seed, n_seq, w.L, w.D, w.N, w.io, channels=chans)
    p = I.make_params(seed, w.D, w.N)
    A, Dk = p["A"][c0:c1].copy(), p["Dskip"][c0:c1].copy()
    oracle.load()
    conn.send("ready")
    while conn.recv() == "run":
        oracle.train_blocks(s["x"], s["dt"], A, s["B"], s["C"], Dk, w.K)
        conn.send("done")


def cpu_model() -> str:
    """The host CPU's model name (first processor in /proc/cpuinfo), or ''."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


class OraclePool:
    """The fp64 oracle, unchanged, on every host core: `workers` spawned
    processes each own a contiguous slice of the channels (channels are
    independent in the scan) of the first n_seq sequences; a step runs all
    slices at once and its time is the wall-clock time until the last is done."""

    def __init__(self, w, seed, n_seq, workers=None):
        import multiprocessing as mp
        self.w, self.n_seq = w, n_seq
        self.workers = max(1, min(workers or os.cpu_count() or 1, w.D))
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for i in range(self.workers):
            c0, c1 = i * w.D // self.workers, (i + 1) * w.D // self.workers
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_oracle_worker, args=(b, w.name, seed, n_seq, c0, c1), daemon=True)
            pr.start()
            self.conns.append(a)
            self.procs.append(pr)
        for c in self.conns:
            assert c.recv() == "ready"

    def step(self) -> float:
        t0 = time.perf_counter()
        for c in self.conns:
            c.send("run")
        for c in self.conns:
            c.recv()
        return time.perf_counter() - t0

    def tokens_per_step(self) -> int:
        return self.n_seq * self.w.L

    def close(self):
        for c in self.conns:
            c.send("stop")
        for pr in self.procs:
            pr.join(timeout=30)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = I.WORKLOADS[WORKLOAD]
    pool = OraclePool(w, w.seed, w.batch)
    try:
        for _ in range(args.warmup):
            pool.step()
        times = [pool.step() for _ in range(args.steps)]
    finally:
        pool.close()
    per_step = statistics.mean(times)
    value = pool.tokens_per_step() / per_step
    sample = (f"all {w.batch} sequences x {w.L} tokens x {w.D} channels per step, channels split over "
              f"{pool.workers} processes")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": WORKLOAD, "batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N,
                   "block": w.K, "io_dtype": w.io, "parallelism": f"dp{args.gpus}", "sample": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
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

    # end to end through the public call with host buffers: every step copies its
    # inputs from pinned host memory, runs the pass and reads all its outputs
    # (y, boundary states, final state) back into pinned host memory. Steps are
    # pipelined on three streams with two device buffer sets: step k's upload
    # overlaps step k-1's pass and step k-2's download (PCIe is full duplex).
    hx = {k: up(v, pin=True) for k, v in s.items()}
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    hb = torch.empty(bnd.shape, dtype=bnd.dtype).pin_memory()
    hh = torch.empty(hout.shape, dtype=hout.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = hy.numel() * hy.element_size() + hb.numel() * hb.element_size() + hh.numel() * hh.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_c = stream
    bufs = []
    for i in range(2):
        bufs.append({"in": {k: torch.empty_like(v, device=dev) for k, v in hx.items()},
                     "y": y if i == 0 else torch.empty_like(y), "bnd": bnd if i == 0 else torch.empty_like(bnd),
                     "hout": hout if i == 0 else torch.empty_like(hout),
                     "ev_in": torch.cuda.Event(), "ev_c": torch.cuda.Event(), "ev_out": torch.cuda.Event()})

    def e2e_steps_run(n):
        for k in range(n):
            bf = bufs[k % 2]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(bf["ev_c"])        # the pass two steps back has read these inputs
                for name in hx:
                    bf["in"][name].copy_(hx[name], non_blocking=True)
                bf["ev_in"].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(bf["ev_in"])
                if k >= 2:
                    s_c.wait_event(bf["ev_out"])       # the download two steps back has read these outputs
                d = bf["in"]
                bdscan.train_blocks(d["x"], d["dt"], A, d["B"], d["C"], Dk, w.K, y=bf["y"], boundary=bf["bnd"],
                                    h_out=bf["hout"])
                bf["ev_c"].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(bf["ev_c"])
                hy.copy_(bf["y"], non_blocking=True)
                hb.copy_(bf["bnd"], non_blocking=True)
                hh.copy_(bf["hout"], non_blocking=True)
                bf["ev_out"].record(s_out)

    e2e_value = None
    if not args.no_e2e:
        e2e_steps = max(2, min(args.steps, 8))
        e2e_steps_run(2)
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_steps_run(e2e_steps)
        e1.record(s_out)
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
        pool = OraclePool(w, w.seed, w.batch)
        try:
            secs = pool.step()
        finally:
            pool.close()
        cpu = {"value": pool.tokens_per_step() / secs, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
               "sample": f"all {w.batch} sequences x {w.L} tokens x {w.D} channels once, channels split over "
                         f"{pool.workers} processes, {secs:.1f} s", "cpu": cpu_model()}

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
                             "frac_of_nominal_8000": hbm_gbs / 8000.0,
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


# ------------------------------------------------------- inference workloads
def step_bytes(w) -> int:
    """Algorithmic bytes of one block step: x, dt in, y out, B, C, A, Dskip, cache read."""
    s = 2 if w.io == "bf16" else 4
    return (w.batch * w.K * w.D * 3 * s + w.batch * w.K * w.N * 2 * s + 4 * w.D * w.N + 4 * w.D
            + 4 * w.batch * w.D * w.N)


def commit_bytes(w) -> int:
    s = 2 if w.io == "bf16" else 4
    return w.batch * w.K * w.D * 2 * s + w.batch * w.K * w.N * 2 * s + 4 * w.D * w.N + 8 * w.batch * w.D * w.N


def prefill_bytes(w, L) -> int:
    s = 2 if w.io == "bf16" else 4
    return w.batch * L * w.D * 3 * s + w.batch * L * w.N * 2 * s + 4 * w.D * w.N + 4 * w.D + 4 * w.batch * w.D * w.N


def run_inference(args, name):
    """Block-diffusion inference at a long context: prefill (forward-only scan of
    the context), then per block `steps` denoising steps (forward from the cache
    plus in-block reverse) and one commit. Reports the prefill, the single step
    (inputs from a rotating pool larger than twice L2, so they come from HBM) and
    the whole denoise loop replayed as a CUDA graph."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS[name]
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    L, K = w.L, w.K

    def up(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    p = I.make_params(w.seed, w.D, w.N)
    A, Dk = up(p["A"]), up(p["Dskip"])
    ctx = {k: torch.empty((w.batch, L, w.D if k in ("x", "dt") else w.N), dtype=torch.bfloat16, device=dev)
           for k in ("x", "dt", "B", "C")}
    span = 8 * I.CHUNK
    for t0 in range(0, L, span):
        n = min(span, L - t0)
        sq = I.make_sequence(w.seed, w.batch, n, w.D, w.N, w.io, stream=("context",), t0=t0)
        for k in ctx:
            ctx[k][:, t0:t0 + n] = up(sq[k])
    y_ctx = torch.empty((w.batch, L, w.D), dtype=torch.bfloat16, device=dev)
    cache = torch.empty((w.batch, w.D, w.N), dtype=torch.float32, device=dev)

    def prefill():
        bdscan.prefill(ctx["x"], ctx["dt"], A, ctx["B"], ctx["C"], Dk, K, y=y_ctx, h_out=cache)

    ws = torch.empty(max(16, bdscan.prefill_chunked_workspace_bytes(ctx["x"], ctx["B"], K)), dtype=torch.uint8,
                     device=dev)

    def prefill_chunked():
        bdscan.prefill_chunked(ctx["x"], ctx["dt"], A, ctx["B"], ctx["C"], Dk, K, y=y_ctx, h_out=cache, ws=ws)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    prefill_seq_ms = timed(prefill)
    prefill_ms = timed(prefill_chunked)

    # rotating pool of noisy block inputs, > 2x L2
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per = step_bytes(w)
    pool_n = max(64, int(2.2 * l2 / per) + 1)
    total_steps = w.blocks * w.steps
    nz = I.make_sequence(w.seed, w.batch, K * pool_n, w.D, w.N, w.io, stream=("noisy", 0, 0))
    pool = {k: up(v).view(w.batch, pool_n, K, -1).transpose(0, 1).contiguous() for k, v in nz.items()}
    cl = I.make_sequence(w.seed, w.batch, K * w.blocks, w.D, w.N, w.io, stream=("context",), t0=L)
    clean = {k: up(v).view(w.batch, w.blocks, K, -1).transpose(0, 1).contiguous() for k, v in cl.items()}
    y_step = torch.empty((w.batch, K, w.D), dtype=torch.bfloat16, device=dev)

    def step(i):
        q = {k: v[i % pool_n] for k, v in pool.items()}
        bdscan.block_step(q["x"], q["dt"], A, q["B"], q["C"], Dk, cache, y=y_step)

    for i in range(10):
        step(i)
    torch.cuda.synchronize(dev)
    n_meas = min(pool_n, 200)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_meas)]
    for i in range(n_meas):
        evs[i][0].record()
        step(i)
        evs[i][1].record()
    torch.cuda.synchronize(dev)
    step_us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3

    # the whole denoise loop (all blocks: steps + commit) as one CUDA graph
    cache0 = cache.clone()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        for i in range(2):   # warm up on the capture stream
            step(i)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for j in range(w.blocks):
                for st in range(w.steps):
                    step(j * w.steps + st)
                c = {k: v[j] for k, v in clean.items()}
                bdscan.commit_block(c["x"], c["dt"], A, c["B"], c["C"], Dk, cache)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    loop_ms = []
    for _ in range(3):
        cache.copy_(cache0)
        torch.cuda.synchronize(dev)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        loop_ms.append(e0.elapsed_time(e1))
    loop_ms = statistics.median(loop_ms)
    del g
    launches = total_steps + w.blocks

    # the full-sequence bidirectional comparator: one denoising step re-runs
    # the reverse scan over the whole context + block (DiffuMamba-style mixing)
    full_ms = None
    if w.batch * (L + K) * w.D * 2 * 3 < 40e9:
        fx = {k: torch.cat([ctx[k], pool[k][0]], dim=1).contiguous() for k in ctx}
        fy = torch.empty((w.batch, L + K, w.D), dtype=torch.bfloat16, device=dev)

        def full_step():
            bdscan.full_bidirectional(fx["x"], fx["dt"], A, fx["B"], fx["C"], Dk, y=fy)

        full_step()
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(3):
            full_step()
        e1.record()
        torch.cuda.synchronize(dev)
        full_ms = e0.elapsed_time(e1) / 3
        del fx, fy
    line = {
        "metric": METRIC, "workload": name, "n_gpus": 1, "dtype": "f32", "data": "synthetic",
        "config": {"workload": name, "batch": w.batch, "context": L, "d_inner": w.D, "d_state": w.N, "block": K,
                   "steps_per_block": w.steps, "blocks": w.blocks, "io_dtype": w.io},
        "prefill": {"ms": prefill_ms, "kind": "time-chunked (bdscan_prefill_chunked)",
                    "sequential_ms": prefill_seq_ms, "workspace_bytes": int(ws.numel()),
                    "tokens_per_s": w.batch * L / (prefill_ms * 1e-3),
                    "hbm_gbs": prefill_bytes(w, L) / (prefill_ms * 1e-3) / 1e9,
                    "hbm_frac": prefill_bytes(w, L) / (prefill_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "ex2_frac": w.batch * L * w.D * w.N / (prefill_ms * 1e-3) / 1e9 /
                                (EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e-3)},
        "step": {"us": step_us, "scanned_tokens_per_s": w.batch * K / (step_us * 1e-6),
                 "algorithmic_bytes": per, "hbm_gbs": per / (step_us * 1e-6) / 1e9,
                 "hbm_frac": per / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                 "inputs": f"rotating pool of {pool_n} step inputs ({pool_n * per / 1e6:.0f} MB > 2x L2)"},
        "loop": {"ms": loop_ms, "graph_launches": launches, "us_per_launch": loop_ms * 1e3 / launches,
                 "committed_tokens_per_s": w.batch * K * w.blocks / (loop_ms * 1e-3),
                 "scanned_tokens_per_s": w.batch * K * launches / (loop_ms * 1e-3),
                 "hbm_gbs": (total_steps * per + w.blocks * commit_bytes(w)) / (loop_ms * 1e-3) / 1e9},
        "full_sequence_step": None if full_ms is None else {
            "ms": full_ms, "tokens": L + K,
            "vs_block_step": full_ms * 1e3 / step_us,
            "note": "forward + reverse scan over context + active block per denoising step"},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_stack(args):
    """24-layer N = 64 stack: one full-block pass per layer (per-layer A, Dskip),
    for each block size; tokens/s = batch * L * layers / time."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS["stack350m"]
    dev = torch.device("cuda", 0)
    peaks = load_peaks()

    def up(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    g = {k: up(v) for k, v in s.items()}
    params = [I.make_params(w.seed, w.D, w.N, layer=l) for l in range(w.layers)]
    As = [up(q["A"]) for q in params]
    Ds = [up(q["Dskip"]) for q in params]
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device=dev)
    res = {}
    for K in I.STACK_BLOCK_SIZES:
        def layers():
            for l in range(w.layers):
                bdscan.train_blocks(g["x"], g["dt"], As[l], g["B"], g["C"], Ds[l], K, y=y)
        layers()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        layers()
        e1.record()
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        per_layer = ms / w.layers
        res[str(K)] = {"ms_24_layers": ms, "tokens_per_s": w.batch * w.L * w.layers / (ms * 1e-3),
                       "ex2_frac": w.batch * w.L * w.D * w.N / (per_layer * 1e-3) / 1e9 /
                                   (EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e-3),
                       "hbm_frac": algorithmic_bytes(w, boundary=False, h_out=False) / (per_layer * 1e-3) / 1e9
                                   / peaks["hbm_gbs"]}
    print(json.dumps({"metric": METRIC, "workload": "stack350m", "config": {"batch": w.batch, "seq_len": w.L,
                      "d_inner": w.D, "d_state": w.N, "layers": w.layers, "io_dtype": w.io},
                      "by_block": res}), flush=True)
    return 0


def backward_bytes(w) -> int:
    """Algorithmic bytes of one backward call: x, dt, dy in; dx, d(dt) out;
    B, C in and dB, dC out; the block-boundary states in; A, Dskip in and
    dA, dDskip out (workspace partials are not counted)."""
    s = 2 if w.io == "bf16" else 4
    n = w.batch * w.L * w.D * s * 5
    n += w.batch * w.L * w.N * s * 4
    n += w.batch * (w.L // w.K) * w.D * w.N * 4
    n += 2 * (w.D * w.N * 4 + w.D * 4)
    return n


def run_train_step(args):
    """Training step of the headline workload: the all-block forward pass
    (y + block-boundary states) and its backward pass given dy."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS["train"]
    dev = torch.device("cuda", 0)
    peaks = load_peaks()

    def up(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    p = I.make_params(w.seed, w.D, w.N)
    g = {k: up(v) for k, v in s.items()}
    A, Dk = up(p["A"]), up(p["Dskip"])
    dy = up(I.f32_to_bf16_bits(I.make_state(w.seed + 9, w.batch, w.L, w.D)))
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device=dev)
    bnd = torch.empty((w.batch, w.L // w.K, w.D, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(bdscan.train_blocks_backward_workspace_bytes(g["x"], g["B"], w.K), dtype=torch.uint8,
                     device=dev)
    grads = {"dx": torch.empty_like(g["x"]), "ddt": torch.empty_like(g["x"]), "dB": torch.empty_like(g["B"]),
             "dC": torch.empty_like(g["C"]), "dA": torch.empty_like(A), "dDskip": torch.empty_like(Dk),
             "dh0": torch.empty((w.batch, w.D, w.N), dtype=torch.float32, device=dev)}

    def fwd():
        bdscan.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, w.K, y=y, boundary=bnd)

    def bwd():
        bdscan.train_blocks_backward(g["x"], g["dt"], A, g["B"], g["C"], Dk, w.K, dy, bnd, grads=grads, ws=ws)

    for _ in range(max(args.warmup, 3)):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    n = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    with ClockSampler(0) as clk:
        for i in range(n):
            evs[i][0].record()
            fwd()
            evs[i][1].record()
            bwd()
            evs[i][2].record()
        torch.cuda.synchronize(dev)
    f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    b_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    tok = w.batch * w.L
    ex2_peak = EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e-3
    elem = w.batch * w.L * w.D * w.N
    line = {"metric": METRIC, "workload": "train_fwd_bwd", "n_gpus": 1, "steps": n, "dtype": "f32",
            "data": "synthetic",
            "config": {"batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N, "block": w.K,
                       "io_dtype": w.io, "gated": False},
            "forward_ms": f_ms, "backward_ms": b_ms, "step_ms": f_ms + b_ms,
            "tokens_per_s": tok / ((f_ms + b_ms) * 1e-3),
            "backward": {"kernels": 2, "ex2_frac": elem / (b_ms * 1e-3) / 1e9 / ex2_peak,
                         "hbm_gbs": backward_bytes(w) / (b_ms * 1e-3) / 1e9,
                         "hbm_frac": backward_bytes(w) / (b_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": backward_bytes(w),
                         "workspace_bytes": ws.numel()},
            "gpu_launches": 3 * n, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_context_parallel(args):
    """Prefill of the 262,144-token context (batch 4, 2048 channels) split over
    the ranks (torchrun, one rank per GPU): each rank generates and holds its
    consecutive chunk, computes its summary, joins one all-gather, folds its
    start state and prefills its chunk. Time: max over ranks."""
    import datetime
    import statistics as st_
    import torch
    import torch.distributed as dist
    from selective_ssm_scan_mamba_b200 import bdscan, context_parallel as cp
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29511")
        dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w = I.WORKLOADS["step262k"]
    K = w.K
    nblk = w.L // K
    b0, b1 = rank * nblk // world, (rank + 1) * nblk // world
    t0, n = b0 * K, (b1 - b0) * K

    def up(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    p = I.make_params(w.seed, w.D, w.N)
    A, Dk = up(p["A"]), up(p["Dskip"])
    ctx = {k: torch.empty((w.batch, n, w.D if k in ("x", "dt") else w.N), dtype=torch.bfloat16, device=dev)
           for k in ("x", "dt", "B", "C")}
    for c0 in range(0, n, 8 * I.CHUNK):
        m = min(8 * I.CHUNK, n - c0)
        sq = I.make_sequence(w.seed, w.batch, m, w.D, w.N, w.io, stream=("context",), t0=t0 + c0)
        for k in ctx:
            ctx[k][:, c0:c0 + m] = up(sq[k])

    def step():
        return cp.prefill_context_parallel(ctx["x"], ctx["dt"], A, ctx["B"], ctx["C"], Dk, K, want_y=True,
                                           want_boundary=True)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(max(args.steps, 1)):
        dist.barrier(device_ids=[local])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1))
    ms = st_.median(ts)
    (mx,) = max_over_ranks([ms], device=dev)
    if rank == 0:
        print(json.dumps({"metric": METRIC, "workload": "cp_prefill", "n_gpus": world, "steps": len(ts),
                          "config": {"batch": w.batch, "context": w.L, "d_inner": w.D, "d_state": w.N, "block": K,
                                     "io_dtype": w.io, "chunks": world},
                          "ms": mx, "tokens_per_s": w.batch * w.L / (mx * 1e-3),
                          "note": "chunk summary + one all-gather + carry fold + chunk prefill per rank"}),
              flush=True)
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
    ap.add_argument("--workload", default="train",
                    choices=["train", "train_fwd_bwd", "step65k", "step262k", "stack350m", "cp_prefill"],
                    help="train: the headline line; the others print their own measurement lines")
    args = ap.parse_args()
    if args.workload in ("step65k", "step262k"):
        return run_inference(args, args.workload)
    if args.workload == "stack350m":
        return run_stack(args)
    if args.workload == "train_fwd_bwd":
        return run_train_step(args)
    if args.workload == "cp_prefill":
        return run_context_parallel(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python
"""Benchmark of the block-confined bidirectional selective scan on B200.

One step = one pass of the mixer's hot path through every layer of the
350M-scale stack: 24 layers, each a full-block (all-block) pass over batch 16 x
8192 tokens x 2048 channels with N = 64 and blocks of 16 tokens (the forward
scan over every token, the reverse scan inside every block, the fused softplus
/ exp / skip / combine), bf16 I/O, fp32 state. This is the largest workload that
fits one GPU; per-layer A and Dskip, x/dt/B/C shared by the layers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun every rank runs its own batch
(independent sequences, no data-path collective: weak scaling); the timing is
the max over ranks. Besides the headline, the line carries (one GPU only) the
other block sizes of the stack and `secondary` records: the training workload
(batch 8 x 4096 x 1536, N = 16) forward and backward, and the 65,536- and
262,144-token inference workloads (prefill, block step, graph-replayed block
loop, full-sequence comparator). `--impl reference` times the fp64 CPU oracle
instead, on a bounded sample of the same workload.
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

WORKLOAD = "stack350m"
STACK_K = 16                 # headline block size of the stack (the others are sub-results)
ORACLE_SAMPLE_CHANNELS = 128  # oracle sample of the stack: one layer, all sequences, these channels
METRIC = "bidirectional block-scan tokens/s and achieved HBM GB/s vs B200 peak"
SM_COUNT = 148
EX2_PER_CLK_SM = 16          # MUFU.EX2 results per clock per SM: the nominal rate of the special-function
                             # unit (a throughput probe on this machine measured 15.9; not in the driver's peaks)
PROFILE_TRAFFIC = {"stack350m": os.path.join(ROOT, "profiles", "stack350m_traffic.json"),
                   "train": os.path.join(ROOT, "profiles", "train_traffic.json")}


def kernel_source_hash() -> str:
    """Hash of the code the forward scan kernels are compiled from (their
    device sources, with comments and whitespace removed: host-side launch
    code, the backward kernel and comment edits do not change it)."""
    import re
    h = hashlib.sha256()
    for name in ("bdscan_device.cuh", "bdscan_kernels.cuh", "bdscan_lag.cuh"):
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


def stack_tokens_per_step(w, world: int) -> int:
    """Token-layers per step of the stack: every layer scans every token of every sequence."""
    return w.batch * w.L * w.layers * world


def config_dict(w, world: int, K: int) -> dict:
    """The workload named in both arms' JSON lines (identical keys and values)."""
    return {"workload": w.name, "batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N,
            "layers": w.layers, "block": K, "io_dtype": w.io, "state_dtype": "f32",
            "outputs": "y of every layer", "count": "tokens x layers (each layer scans every token)",
            "parallelism": f"dp{world}",
            "l2": "working set 1.64 GB per layer launch > 126 MB L2 (no flush)"}


def _up(a, dev=None, pin=False):
    """numpy array (bf16 as uint16 bits) -> torch tensor on dev, or pinned host memory."""
    import torch
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    return t.pin_memory() if pin else t.to(dev)


# ------------------------------------------------------------------ CPU oracle
def _oracle_worker(conn):
    """One process of OraclePool: receives its channel slice once, then runs
    the oracle's full-block pass on it whenever asked."""
    import oracle
    oracle.load()
    job = conn.recv()
    fn = oracle.prefill if job.get("op") == "prefill" else oracle.train_blocks
    conn.send("ready")
    while conn.recv() == "run":
        fn(job["x"], job["dt"], job["A"], job["B"], job["C"], job["Dskip"], job["K"])
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
    processes each own a contiguous slice of the given channels (channels are
    independent in the scan); a step runs all slices at once and its time is
    the wall-clock time until the last is done. s: x, dt [n_seq, L, channels],
    B, C [n_seq, L, N]; A [channels, N], Dskip [channels]."""

    def __init__(self, s, A, Dskip, K, workers=None, op="train"):
        import multiprocessing as mp
        nch = s["x"].shape[2]
        self.workers = max(1, min(workers or os.cpu_count() or 1, nch))
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for i in range(self.workers):
            c0, c1 = i * nch // self.workers, (i + 1) * nch // self.workers
            a, b = ctx.Pipe()
            pr = ctx.Process(target=_oracle_worker, args=(b,), daemon=True)
            pr.start()
            a.send({"x": np.ascontiguousarray(s["x"][:, :, c0:c1]), "dt": np.ascontiguousarray(s["dt"][:, :, c0:c1]),
                    "B": s["B"], "C": s["C"], "A": np.ascontiguousarray(A[c0:c1]),
                    "Dskip": np.ascontiguousarray(Dskip[c0:c1]), "K": K, "op": op})
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

    def close(self):
        for c in self.conns:
            c.send("stop")
        for pr in self.procs:
            pr.join(timeout=30)


def stack_oracle_pool(w, seed, K):
    """The oracle on the bounded sample of the stack: layer 0, all sequences,
    all tokens, channels [0, ORACLE_SAMPLE_CHANNELS). The scan's cost is exactly
    linear in channels and layers, so a sample time t stands for
    t * (D / channels) * layers of the whole step."""
    chans = list(range(ORACLE_SAMPLE_CHANNELS))
    s = I.make_sequence(seed, w.batch, w.L, w.D, w.N, w.io, channels=chans)
    p = I.make_params(w.seed, w.D, w.N, layer=0)
    pool = OraclePool(s, p["A"][:len(chans)], p["Dskip"][:len(chans)], K)
    sample = (f"one layer, all {w.batch} sequences x {w.L} tokens, channels 0-{len(chans) - 1} of {w.D}, "
              f"block {K}, split over {pool.workers} processes; extrapolated linearly to {w.D} channels "
              f"and {w.layers} layers")
    return pool, sample


def oracle_value(w, secs: float) -> float:
    """Stack tokens x layers per second implied by one sample time."""
    full_step = secs * (w.D / ORACLE_SAMPLE_CHANNELS) * w.layers
    return w.batch * w.L * w.layers / full_step


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = I.WORKLOADS[WORKLOAD]
    pool, sample = stack_oracle_pool(w, w.seed, STACK_K)
    try:
        for _ in range(args.warmup):
            pool.step()
        times = [pool.step() for _ in range(args.steps)]
    finally:
        pool.close()
    per_sample = statistics.mean(times)
    value = oracle_value(w, per_sample)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": w.batch * w.L * w.layers / value * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": config_dict(w, args.gpus, STACK_K),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
                         "sample": sample, "sample_s": per_sample, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def traffic_for(workload: str):
    """ncu DRAM bytes per launch recorded for the kernel, if the kernel's code is
    unchanged since the capture (else None)."""
    path = PROFILE_TRAFFIC.get(workload)
    if path and os.path.exists(path):
        pt = json.load(open(path))
        if pt.get("kernel_source_hash") == kernel_source_hash():
            return pt.get("traffic_bytes_per_launch")
    return None


def ex2_peak_g(peaks) -> float:
    return EX2_PER_CLK_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e-3


def roofline(elem_steps: int, nbytes: int, launch_ms: float, peaks, traffic=None, kernel="") -> dict:
    """SFU roofline of one launch (one MUFU.EX2 per element-step) with the HBM
    fraction of its algorithmic bytes beside it."""
    rate = elem_steps / (launch_ms * 1e-3) / 1e9
    gbs = nbytes / (launch_ms * 1e-3) / 1e9
    return {"bound": "alu", "achieved": rate, "peak": ex2_peak_g(peaks), "unit": "Gex2/s",
            "frac": rate / ex2_peak_g(peaks), "traffic": traffic,
            "peak_source": f"nominal {EX2_PER_CLK_SM} MUFU.EX2/clk/SM x {SM_COUNT} SMs x "
                           f"{peaks['sm_max_mhz']:.0f} MHz (probe on this pool: 15.9/clk/SM)",
            "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                    "peak_source": peaks["source"], "frac_of_nominal_8000": gbs / 8000.0,
                    "algorithmic_bytes_per_launch": nbytes},
            "ex2_per_launch": elem_steps, "kernel": kernel, "kernel_ms": launch_ms}


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
    K = STACK_K
    seed = rank_seed(w.seed, rank)
    s = I.make_sequence(seed, w.batch, w.L, w.D, w.N, w.io)
    params = [I.make_params(w.seed, w.D, w.N, layer=l) for l in range(w.layers)]
    g = {k: _up(v, dev) for k, v in s.items()}
    As = [_up(q["A"], dev) for q in params]
    Ds = [_up(q["Dskip"], dev) for q in params]
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def layers(inp, yout, Kb, evs=None):
        for l in range(w.layers):
            if evs is not None:
                evs[l][0].record(stream)
            bdscan.train_blocks(inp["x"], inp["dt"], As[l], inp["B"], inp["C"], Ds[l], Kb, y=yout)
            if evs is not None:
                evs[l][1].record(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    warm = max(args.warmup, 3)
    for _ in range(warm):
        layers(g, y, K)
    torch.cuda.synchronize(dev)

    # timed region: device time with CUDA events on the launching stream; one
    # event pair per layer launch gives the per-launch duration for the roofline
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(w.layers)]
          for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(args.steps):
            layers(g, y, K, ev[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    elapsed_ms, launch_ms = max_over_ranks(
        [start.elapsed_time(stop), statistics.mean(a.elapsed_time(b) for st in ev for a, b in st)], device=dev)
    ms_per_step = elapsed_ms / args.steps
    tokens_per_step = stack_tokens_per_step(w, world)
    value = tokens_per_step / (ms_per_step * 1e-3)
    peaks = load_peaks()
    elem = w.batch * w.L * w.D * w.N
    nbytes = algorithmic_bytes(w, boundary=False, h_out=False)
    roof = roofline(elem, nbytes, launch_ms, peaks, traffic_for("stack350m"),
                    kernel=f"bdscan_lag_kernel<bf16, N=64, K={K}, 8 states per lane>")

    # the other block sizes of the stack (same inputs, 24 layers each)
    by_block = {str(K): {"ms_24_layers": ms_per_step, "tokens_per_s": value / world, "sfu_frac": roof["frac"],
                         "hbm_frac": roof["hbm"]["frac"]}}
    for Kb in (k for k in I.STACK_BLOCK_SIZES if k != K):
        layers(g, y, Kb)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 2
        e0.record(stream)
        for _ in range(reps):
            layers(g, y, Kb)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / reps
        per_layer = ms / w.layers
        by_block[str(Kb)] = {"ms_24_layers": ms, "tokens_per_s": w.batch * w.L * w.layers / (ms * 1e-3),
                             "sfu_frac": elem / (per_layer * 1e-3) / 1e9 / ex2_peak_g(peaks),
                             "hbm_frac": nbytes / (per_layer * 1e-3) / 1e9 / peaks["hbm_gbs"]}

    # end to end through the public call with host buffers: every step copies
    # x, dt, B, C from pinned host memory, runs the 24 layers and reads the last
    # layer's y back into pinned host memory. Steps are pipelined on three
    # streams with two device buffer sets: step k's upload overlaps step k-1's
    # layers and step k-2's download (PCIe is full duplex).
    e2e_value, h2d, d2h = None, 0, 0
    if not args.no_e2e:
        hx = {k: _up(v, pin=True) for k, v in s.items()}
        hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in hx.values())
        d2h = hy.numel() * hy.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        bufs = []
        for i in range(2):
            bufs.append({"in": {k: torch.empty_like(v, device=dev) for k, v in hx.items()},
                         "y": y if i == 0 else torch.empty_like(y),
                         "ev_in": torch.cuda.Event(), "ev_c": torch.cuda.Event(), "ev_out": torch.cuda.Event()})

        def e2e_steps_run(n):
            for k in range(n):
                bf = bufs[k % 2]
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(bf["ev_c"])        # the layers two steps back have read these inputs
                    for name in hx:
                        bf["in"][name].copy_(hx[name], non_blocking=True)
                    bf["ev_in"].record(s_in)
                stream.wait_event(bf["ev_in"])
                if k >= 2:
                    stream.wait_event(bf["ev_out"])        # the download two steps back has read this y
                layers(bf["in"], bf["y"], K)
                bf["ev_c"].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(bf["ev_c"])
                    hy.copy_(bf["y"], non_blocking=True)
                    bf["ev_out"].record(s_out)

        e2e_steps = max(2, min(args.steps, 6))
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
        del bufs, hx, hy
    clocks = clk.summary()
    del g
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pool, sample = stack_oracle_pool(w, w.seed, K)
        try:
            secs = pool.step()
        finally:
            pool.close()
        cpu = {"value": oracle_value(w, secs), "unit": "tokens/s", "cores": pool.workers, "kind": "oracle",
               "sample": f"{sample}; {secs:.1f} s", "cpu": cpu_model()}

    secondary = None
    if world == 1 and not args.no_secondary:
        secondary = {}
        for name, fn in (("train", lambda: measure_train(dev, peaks, 20, 5)),
                         ("train_fwd_bwd", lambda: measure_train_step(dev, peaks, 5, 3)),
                         ("step65k", lambda: measure_inference("step65k", dev, peaks)),
                         ("step262k", lambda: measure_inference("step262k", dev, peaks))):
            try:
                secondary[name] = fn()
            except Exception as e:   # reported in the line, the headline stands
                secondary[name] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_dict(w, world, K),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * w.layers,
        "clocks": clocks,
        "by_block": by_block,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if secondary is not None:
        line["secondary"] = secondary
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_train(dev, peaks, steps=20, warmup=5) -> dict:
    """The training workload (batch 8 x 4096 x 1536, N = 16, K = 16): one
    full-block pass writing y, every block-boundary state and the final state."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS["train"]
    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    p = I.make_params(w.seed, w.D, w.N)
    g = {k: _up(v, dev) for k, v in s.items()}
    A, Dk = _up(p["A"], dev), _up(p["Dskip"], dev)
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device=dev)
    bnd = torch.empty((w.batch, w.L // w.K, w.D, w.N), dtype=torch.float32, device=dev)
    hout = torch.empty((w.batch, w.D, w.N), dtype=torch.float32, device=dev)

    def step():
        bdscan.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, w.K, y=y, boundary=bnd, h_out=hout)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        a.record()
        step()
        b.record()
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    return {"config": {"batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N, "block": w.K,
                       "io_dtype": w.io, "outputs": "y + all block-boundary states + final state"},
            "ms": ms, "tokens_per_s": w.batch * w.L / (ms * 1e-3),
            "roofline": roofline(w.batch * w.L * w.D * w.N, algorithmic_bytes(w), ms, peaks, traffic_for("train"),
                                 kernel="bdscan_lag_kernel<bf16, N=16, K=16, 4 states per lane>")}


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


def measure_inference(name, dev, peaks) -> dict:
    """Block-diffusion inference at a long context: prefill (forward-only scan of
    the context), then per block `steps` denoising steps (forward from the cache
    plus in-block reverse) and one commit. Reports the prefill, the single step
    (inputs from a rotating pool larger than twice L2, so they come from HBM;
    device time and the host time of an eager call through the binding) and the
    whole denoise loop replayed as a CUDA graph."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS[name]
    L, K = w.L, w.K
    sfu = ex2_peak_g(peaks)
    p = I.make_params(w.seed, w.D, w.N)
    A, Dk = _up(p["A"], dev), _up(p["Dskip"], dev)
    ctx = {k: torch.empty((w.batch, L, w.D if k in ("x", "dt") else w.N), dtype=torch.bfloat16, device=dev)
           for k in ("x", "dt", "B", "C")}
    span = 8 * I.CHUNK
    for t0 in range(0, L, span):
        n = min(span, L - t0)
        sq = I.make_sequence(w.seed, w.batch, n, w.D, w.N, w.io, stream=("context",), t0=t0)
        for k in ctx:
            ctx[k][:, t0:t0 + n] = _up(sq[k], dev)
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
    chunked = int(ws.numel()) > 16

    # rotating pool of noisy block inputs, > 2x L2
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per = step_bytes(w)
    pool_n = max(64, int(2.2 * l2 / per) + 1)
    total_steps = w.blocks * w.steps
    nz = I.make_sequence(w.seed, w.batch, K * pool_n, w.D, w.N, w.io, stream=("noisy", 0, 0))
    pool = {k: _up(v, dev).view(w.batch, pool_n, K, -1).transpose(0, 1).contiguous() for k, v in nz.items()}
    cl = I.make_sequence(w.seed, w.batch, K * w.blocks, w.D, w.N, w.io, stream=("context",), t0=L)
    clean = {k: _up(v, dev).view(w.batch, w.blocks, K, -1).transpose(0, 1).contiguous() for k, v in cl.items()}
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
    # host cost of an eager call through the Python binding (argument checks,
    # marshalling, launch), the step's inputs prepared beforehand
    qs = [{k: v[i % pool_n] for k, v in pool.items()} for i in range(200)]
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for q in qs:
        bdscan.block_step(q["x"], q["dt"], A, q["B"], q["C"], Dk, cache, y=y_step)
    host_us = (time.perf_counter() - t0) / len(qs) * 1e6
    torch.cuda.synchronize(dev)
    eager_us = (time.perf_counter() - t0) / len(qs) * 1e6
    # the same through a prepared bdscan.BlockStep (A, Dskip, cache checked once)
    prep = bdscan.BlockStep(A, Dk, cache, K)
    for q in qs[:10]:
        prep(q["x"], q["dt"], q["B"], q["C"], y=y_step)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    for q in qs:
        prep(q["x"], q["dt"], q["B"], q["C"], y=y_step)
    prep_host_us = (time.perf_counter() - t0) / len(qs) * 1e6
    torch.cuda.synchronize(dev)
    prep_us = (time.perf_counter() - t0) / len(qs) * 1e6
    del qs, prep

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
    loop_bytes = total_steps * per + w.blocks * commit_bytes(w)
    loop_elem = (total_steps + w.blocks) * w.batch * K * w.D * w.N

    # the full-sequence bidirectional comparator: one denoising step re-runs
    # the reverse scan over the whole context + block (DiffuMamba-style mixing)
    full_ms = None
    if w.batch * (L + K) * w.D * 2 * 3 < 40e9:
        del pool
        fx = {k: torch.cat([ctx[k], clean[k][0]], dim=1).contiguous() for k in ctx}
        del ctx, y_ctx
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
    pf_elem = w.batch * L * w.D * w.N
    pf_bytes = prefill_bytes(w, L)
    return {
        "config": {"batch": w.batch, "context": L, "d_inner": w.D, "d_state": w.N, "block": K,
                   "steps_per_block": w.steps, "blocks": w.blocks, "io_dtype": w.io},
        "prefill": {"ms": prefill_ms,
                    "kind": "time-chunked (bdscan_prefill_chunked)" if chunked else
                            "sequential (bdscan_prefill_chunked runs the sequential scan: enough rows)",
                    "sequential_ms": prefill_seq_ms, "workspace_bytes": int(ws.numel()) if chunked else 0,
                    "tokens_per_s": w.batch * L / (prefill_ms * 1e-3),
                    "algorithmic_bytes": pf_bytes,
                    "hbm_gbs": pf_bytes / (prefill_ms * 1e-3) / 1e9,
                    "hbm_frac": pf_bytes / (prefill_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "sfu_frac": pf_elem / (prefill_ms * 1e-3) / 1e9 / sfu},
        "step": {"us": step_us, "scanned_tokens_per_s": w.batch * K / (step_us * 1e-6),
                 "algorithmic_bytes": per, "hbm_gbs": per / (step_us * 1e-6) / 1e9,
                 "hbm_frac": per / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                 "sfu_frac": w.batch * K * w.D * w.N / (step_us * 1e-6) / 1e9 / sfu,
                 "eager_call_us": eager_us, "eager_host_us": host_us,
                 "prepared_call_us": prep_us, "prepared_host_us": prep_host_us,
                 "inputs": f"rotating pool of {pool_n} step inputs ({pool_n * per / 1e6:.0f} MB > 2x L2)"},
        "loop": {"ms": loop_ms, "graph_launches": launches, "us_per_launch": loop_ms * 1e3 / launches,
                 "committed_tokens_per_s": w.batch * K * w.blocks / (loop_ms * 1e-3),
                 "scanned_tokens_per_s": w.batch * K * launches / (loop_ms * 1e-3),
                 "hbm_gbs": loop_bytes / (loop_ms * 1e-3) / 1e9,
                 "hbm_frac": loop_bytes / (loop_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                 "sfu_frac": loop_elem / (loop_ms * 1e-3) / 1e9 / sfu},
        "full_sequence_step": None if full_ms is None else {
            "ms": full_ms, "tokens": L + K,
            "vs_block_step": full_ms * 1e3 / step_us,
            "note": "forward + reverse scan over context + active block per denoising step"},
    }


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


def measure_train_step(dev, peaks, steps=5, warmup=3) -> dict:
    """Training step of the training workload: the all-block forward pass
    (y + block-boundary states) and its backward pass given dy."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    w = I.WORKLOADS["train"]
    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    p = I.make_params(w.seed, w.D, w.N)
    g = {k: _up(v, dev) for k, v in s.items()}
    A, Dk = _up(p["A"], dev), _up(p["Dskip"], dev)
    dy = _up(I.f32_to_bf16_bits(I.make_state(w.seed + 9, w.batch, w.L, w.D)), dev)
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

    for _ in range(warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record()
        fwd()
        evs[i][1].record()
        bwd()
        evs[i][2].record()
    torch.cuda.synchronize(dev)
    f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    b_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    elem = w.batch * w.L * w.D * w.N
    return {"config": {"batch": w.batch, "seq_len": w.L, "d_inner": w.D, "d_state": w.N, "block": w.K,
                       "io_dtype": w.io, "gated": False},
            "forward_ms": f_ms, "backward_ms": b_ms, "step_ms": f_ms + b_ms,
            "tokens_per_s": w.batch * w.L / ((f_ms + b_ms) * 1e-3),
            "backward": {"kernels": 2, "sfu_frac": elem / (b_ms * 1e-3) / 1e9 / ex2_peak_g(peaks),
                         "hbm_gbs": backward_bytes(w) / (b_ms * 1e-3) / 1e9,
                         "hbm_frac": backward_bytes(w) / (b_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": backward_bytes(w), "workspace_bytes": ws.numel()}}


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


def _oracle_sample(name, scale=1):
    """Bounded oracle sample of a workload's timed unit: (inputs, params, what the
    unit is, element-steps of the full unit / of the sample, call). Channels are
    independent, so the cost of the unit is exactly linear in the channels and
    sequences sampled; config 5 also multiplies by its 24 layers."""
    import oracle
    w = I.WORKLOADS[name]
    if name == "pr1":
        nch, n_seq, L, op, unit = w.D, w.batch, w.L, "train", "train_blocks, 256 tokens"
    elif name == "train":
        nch, n_seq, L, op, unit = 192, w.batch, w.L, "train", "train_blocks, 8 x 4096 tokens"
    elif name == "stack350m":
        nch, n_seq, L, op, unit = 32, w.batch, w.L, "train", "24 layers, 16 x 8192 tokens, K = 16"
    else:   # inference: the context prefill (forward-only scan) of all sequences
        nch, n_seq, L, op, unit = 64, w.batch, 8192, "prefill", f"prefill of {w.batch} x {w.L} context tokens"
    chans = list(range(min(w.D, nch * scale)))   # (scale: one sample's worth per worker)
    s = I.make_sequence(w.seed, n_seq, L, w.D, w.N, w.io, stream="seq" if op == "train" else ("context",),
                        channels=chans)
    p = I.make_params(w.seed, w.D, w.N)
    A, Dk = p["A"][chans], p["Dskip"][chans]
    full = w.batch * w.L * w.D * w.N * w.layers
    part = n_seq * L * len(chans) * w.N
    if op == "train":
        fn = lambda: oracle.train_blocks(s["x"], s["dt"], A, s["B"], s["C"], Dk, w.K)  # noqa: E731
    else:
        fn = lambda: oracle.prefill(s["x"], s["dt"], A, s["B"], s["C"], Dk, w.K)  # noqa: E731
    return s, A, Dk, unit, full, part, fn, op


def baseline_table(bench_path=None) -> str:
    """Markdown rows of the oracle (single thread and all host cores) and of the
    GPU (from a bench.py JSON line) per workload."""
    import oracle
    oracle.load()
    gpu = json.load(open(bench_path)) if bench_path else {}
    sec = gpu.get("secondary", {})
    rows = ["| config | timed unit | oracle 1 thread | oracle all cores | GPU (this build) | GPU tokens/s | "
            "HBM GB/s (% of measured / of 8000) | SFU % |", "|---|---|---|---|---|---|---|---|"]
    for cfg, name in enumerate(["pr1", "train", "step65k", "step262k", "stack350m"], start=1):
        w = I.WORKLOADS[name]
        s, A, Dk, unit, full, part, fn, op = _oracle_sample(name)
        t0 = time.perf_counter()
        fn()
        t1 = (time.perf_counter() - t0) * full / part
        # all cores: one single-thread sample's worth of channels per worker
        s, A, Dk, unit, full, part, fn, op = _oracle_sample(name, scale=os.cpu_count() or 1)
        pool = OraclePool(s, A, Dk, w.K, op=op)
        try:
            ta = pool.step() * full / part
        finally:
            pool.close()
        gcol = tcol = hcol = scol = "-"
        if name == "stack350m" and gpu.get("value"):
            gcol = f"{gpu['ms_per_step']:.1f} ms per step"
            tcol = f"{gpu['value'] / 1e6:.1f} M"
            hb = gpu["roofline"]["hbm"]
            hcol = f"{hb['achieved']:.0f} ({100 * hb['frac']:.1f} % / {100 * hb['frac_of_nominal_8000']:.1f} %)"
            scol = f"{100 * gpu['roofline']['frac']:.1f}"
        elif name == "train" and "train" in sec and "ms" in sec["train"]:
            r = sec["train"]
            gcol, tcol = f"{r['ms']:.3f} ms", f"{r['tokens_per_s'] / 1e6:.1f} M"
            hb = r["roofline"]["hbm"]
            hcol = f"{hb['achieved']:.0f} ({100 * hb['frac']:.1f} % / {100 * hb['frac_of_nominal_8000']:.1f} %)"
            scol = f"{100 * r['roofline']['frac']:.1f}"
        elif name in sec and "prefill" in sec[name]:
            r = sec[name]["prefill"]
            gcol, tcol = f"{r['ms']:.2f} ms", f"{r['tokens_per_s'] / 1e6:.1f} M"
            hcol = f"{r['hbm_gbs']:.0f} ({100 * r['hbm_frac']:.1f} % / {100 * r['hbm_gbs'] / 8000:.1f} %)"
            scol = f"{100 * r['sfu_frac']:.1f}"
        tokens = w.batch * w.L * w.layers

        def sec_(v):
            return f"{v * 1e3:.1f} ms" if v < 1 else f"{v:.1f} s"
        label = f"{cfg} {name}"
        rows.append(f"| {label} | {unit} | {sec_(t1)} ({tokens / t1 / 1e3:.1f} K tok/s) | {sec_(ta)} "
                    f"({tokens / ta / 1e3:.1f} K tok/s, {pool.workers} cores) | {gcol} | {tcol} | {hcol} | {scol} |")
    rows.append("")
    rows.append(f"Oracle: `oracle/bdscan_oracle.c` (fp64, single-threaded C) on {cpu_model() or 'the host'}; "
                "all-cores = one spawned process per core over channel slices. Timed on bounded channel samples "
                "and extrapolated linearly (the cost is exactly linear in channels, sequences and layers); the "
                "inference rows time the forward-only prefill of the context.")
    return "\n".join(rows)


PROFILE_CASES = {
    # name: (workload the case reduces, batch, L, D, N, K, op)
    "stack_k4": ("stack350m", 4, 8192, 2048, 64, 4, "train"),
    "stack_k16": ("stack350m", 4, 8192, 2048, 64, 16, "train"),
    "stack_k64": ("stack350m", 4, 8192, 2048, 64, 64, "train"),
    "train_k16": ("train", 8, 4096, 1536, 16, 16, "train_states"),
    "backward_k16": ("train", 8, 4096, 1536, 16, 16, "backward"),
    "prefill262k_rows": ("step262k", 4, 32768, 2048, 16, 32, "prefill"),
    "prefill65k_chunked": ("step65k", 1, 65536, 1536, 16, 32, "prefill_chunked"),
    "step65k": ("step65k", 1, 32, 1536, 16, 32, "step"),
    "step262k": ("step262k", 4, 32, 2048, 16, 32, "step"),
}


def run_profile_case(name, warm=3, reps=5):
    """One kernel case, reduced from a workload to a size an ncu capture
    finishes quickly (inputs still larger than L2 where the workload's are):
    `warm` untimed calls, then `reps` timed ones. The stack cases keep the
    stack's grid shape per wave at a quarter of its batch, the 262K prefill
    case keeps its 256 CTAs at an eighth of the context."""
    import torch
    from selective_ssm_scan_mamba_b200 import bdscan
    wname, Bt, L, D, N, K, op = PROFILE_CASES[name]
    w = I.WORKLOADS[wname]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = I.make_sequence(w.seed, Bt, L, D, N, w.io)
    p = I.make_params(w.seed, D, N)
    g = {k: _up(v, dev) for k, v in s.items()}
    A, Dk = _up(p["A"], dev), _up(p["Dskip"], dev)
    y = torch.empty((Bt, L, D), dtype=torch.bfloat16, device=dev)
    if op == "train":
        fn = lambda: bdscan.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, y=y)  # noqa: E731
    elif op in ("train_states", "backward"):
        bnd = torch.empty((Bt, L // K, D, N), dtype=torch.float32, device=dev)
        ho = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
        fn = lambda: bdscan.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, y=y, boundary=bnd,  # noqa: E731
                                         h_out=ho)
        if op == "backward":
            fn()
            dy = _up(I.f32_to_bf16_bits(I.make_state(w.seed + 9, Bt, L, D)), dev)
            ws = torch.empty(bdscan.train_blocks_backward_workspace_bytes(g["x"], g["B"], K), dtype=torch.uint8,
                             device=dev)
            gr = {}
            fn = lambda: bdscan.train_blocks_backward(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, dy, bnd,  # noqa
                                                      ws=ws, grads=gr)
    elif op == "prefill":
        ho = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
        fn = lambda: bdscan.prefill(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, y=y, h_out=ho)  # noqa: E731
    elif op == "prefill_chunked":
        ho = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
        ws = torch.empty(max(16, bdscan.prefill_chunked_workspace_bytes(g["x"], g["B"], K)), dtype=torch.uint8,
                         device=dev)
        fn = lambda: bdscan.prefill_chunked(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, y=y, h_out=ho,  # noqa
                                            ws=ws)
    else:   # one block step from a random cache
        hc = _up(I.make_state(w.seed + 5, Bt, D, N, scale=0.5), dev)
        fn = lambda: bdscan.block_step(g["x"], g["dt"], A, g["B"], g["C"], Dk, hc, y=y)  # noqa: E731
    for _ in range(warm):
        fn()
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1))
    ms = statistics.median(ts)
    elem = Bt * L * D * N
    print(json.dumps({"profile_case": name, "batch": Bt, "L": L, "D": D, "N": N, "K": K, "op": op, "ms": ms,
                      "sfu_frac": elem / (ms * 1e-3) / 1e9 / ex2_peak_g(load_peaks())}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--no-secondary", action="store_true", help="headline only (profiling runs)")
    ap.add_argument("--baseline-table", nargs="?", const="", metavar="BENCH_JSON",
                    help="print the oracle / GPU table of every workload (GPU columns from a bench.py JSON line)")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run one reduced kernel case (for ncu captures) and exit")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "train", "train_fwd_bwd", "step65k", "step262k", "cp_prefill"],
                    help=f"{WORKLOAD}: the headline line; the others print one measurement line each")
    args = ap.parse_args()
    if args.baseline_table is not None:
        print(baseline_table(args.baseline_table or None))
        return 0
    if args.profile_case:
        return run_profile_case(args.profile_case, max(args.warmup, 1), max(args.steps, 1))
    if args.workload == "cp_prefill":
        return run_context_parallel(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == WORKLOAD:
        return run_ours(args)
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    if args.workload == "train":
        rec = measure_train(dev, peaks, args.steps, max(args.warmup, 3))
    elif args.workload == "train_fwd_bwd":
        rec = measure_train_step(dev, peaks, args.steps, max(args.warmup, 3))
    else:
        rec = measure_inference(args.workload, dev, peaks)
    print(json.dumps({"metric": METRIC, "workload": args.workload, "n_gpus": 1, **rec}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

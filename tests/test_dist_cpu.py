"""Data-parallel plumbing of bench.py on CPU: two gloo ranks, each scanning its
own independent sequences, with the job time taken as the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from selective_ssm_scan_mamba_b200 import inputs as I
        w = I.WORKLOADS[bench.WORKLOAD]
        seed = bench.rank_seed(w.seed, rank)
        x = I.make_sequence(seed, 1, 64, 16, 16, "bf16")["x"]
        # the slowest rank sets the job time
        mx = bench.max_over_ranks([10.0 + rank, 5.0 * (world - rank)])
        q.put((rank, seed, x.tobytes(), mx, bench.stack_tokens_per_step(w, world)))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, s0, x0, m0, t0), (r1, s1, x1, m1, t1) = res
    assert s0 != s1 and x0 != x1, "ranks must scan different sequences"
    assert m0 == m1 == [11.0, 10.0]
    assert t0 == t1 == 16 * 8192 * 24 * 2   # token-layers of both ranks' stacks


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_matches_our_config(monkeypatch, capsys):
    """Rank 0 of the reference arm prints one line on the headline's config,
    with the oracle's sample and core count (a reduced channel sample keeps
    this CPU check short)."""
    import json

    import bench
    from selective_ssm_scan_mamba_b200 import inputs as I
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(bench, "ORACLE_SAMPLE_CHANNELS", 4)

    class A:
        steps, warmup, gpus = 1, 0, 1
    assert bench.run_reference(A()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    w = I.WORKLOADS[bench.WORKLOAD]
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["config"] == bench.config_dict(w, 1, bench.STACK_K)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"] > 0

"""Context-parallel prefill plumbing on CPU: two gloo ranks each hold one chunk
of a context; the library's three steps (chunk summary, carry fold, local
prefill) are replaced by float64 stand-ins built on the oracle, so the test
checks the exchange, its rank order and the composition, not the kernels."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import oracle
from selective_ssm_scan_mamba_b200 import inputs as I
from tests.oracle_pins import _close

Bt, L, D, N, K = 2, 48, 3, 4, 8
CUT = 24   # rank 0 holds tokens [0, 24), rank 1 [24, 48)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case():
    s = I.make_sequence(41, Bt, L, D, N, "f32")
    s.update(I.make_params(41, D, N))
    s["h0"] = I.make_state(42, Bt, D, N, scale=0.5)
    return s


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from selective_ssm_scan_mamba_b200 import bdscan, context_parallel as cp

        def summary(x, dt, A, B, C, Dskip, block, dt_softplus=True):
            f = oracle.forward(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(), Dskip.numpy(), block)
            ones = np.ones((x.shape[0], x.shape[2], B.shape[2]))
            p = oracle.forward(np.zeros_like(x.numpy()), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                               Dskip.numpy(), block, h0=ones)
            return torch.from_numpy(f["h_out"]), torch.from_numpy(p["h_out"])

        def fold(H_all, P_all, index, h0=None, out=None):
            h = torch.zeros_like(H_all[0]) if h0 is None else h0.clone()
            for qq in range(index):
                h = P_all[qq] * h + H_all[qq]
            return h

        def prefill(x, dt, A, B, C, Dskip, block, z=None, h0=None, **kw):
            r = oracle.prefill(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(), Dskip.numpy(), block,
                               h0=h0.numpy())
            return torch.from_numpy(r["y"]), torch.from_numpy(r["h_out"]), torch.from_numpy(r["boundary"])

        bdscan.chunk_summary, bdscan.carry_fold, bdscan.prefill = summary, fold, prefill
        s = _case()
        sl = slice(0, CUT) if rank == 0 else slice(CUT, L)
        t = {k: torch.from_numpy(np.ascontiguousarray(oracle.decode(s[k])[:, sl])) for k in ("x", "dt", "B", "C")}
        y, h, bnd = cp.prefill_context_parallel(t["x"], t["dt"], torch.from_numpy(oracle.decode(s["A"])), t["B"],
                                                t["C"], torch.from_numpy(oracle.decode(s["Dskip"])), K,
                                                h0=torch.from_numpy(oracle.decode(s["h0"])))
        q.put((rank, y.numpy(), h.numpy(), bnd.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_prefill_equals_one_prefill():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in procs], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s = _case()
    full = oracle.prefill(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, h0=s["h0"])
    y = np.concatenate([res[0][1], res[1][1]], axis=1)
    bnd = np.concatenate([res[0][3], res[1][3]], axis=1)
    assert _close(y, full["y"], rtol=1e-12, atol=1e-13)
    assert _close(bnd, full["boundary"], rtol=1e-12, atol=1e-13)
    assert _close(res[1][2], full["h_out"], rtol=1e-12, atol=1e-13)
    assert _close(res[0][2], full["boundary"][:, CUT // K - 1], rtol=1e-12, atol=1e-13)

"""The five mixer workloads at full size on the GPU, checked against the fp64
oracle on sampled channels (every (batch, channel) recurrence is independent,
so the oracle run on a channel subset is exact for those channels), plus the
cache-exactness invariant GPU-vs-GPU on the whole tensors."""
import numpy as np
import pytest

import oracle
from selective_ssm_scan_mamba_b200 import inputs as I
from tests.gpu_util import RTOL_Y, assert_c12, assert_state, to_dev, to_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def bd():
    from selective_ssm_scan_mamba_b200 import bdscan
    return bdscan


def sample_channels(D, k, seed):
    return np.sort(np.random.default_rng(seed).choice(D, size=k, replace=False))


def sub(s, ch):
    """Restrict per-channel inputs to channel subset ch (B and C are shared)."""
    return {"x": np.ascontiguousarray(s["x"][:, :, ch]), "dt": np.ascontiguousarray(s["dt"][:, :, ch]),
            "B": s["B"], "C": s["C"], "A": np.ascontiguousarray(s["A"][ch]),
            "Dskip": np.ascontiguousarray(s["Dskip"][ch])}


def otrain(d, K):
    return oracle.train_blocks(d["x"], d["dt"], d["A"], d["B"], d["C"], d["Dskip"], K)


def test_pr1_full(bd):
    w = I.WORKLOADS["pr1"]
    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    s.update(I.make_params(w.seed, w.D, w.N))
    g = {k: to_dev(v) for k, v in s.items()}
    y, bnd, hout = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], w.K,
                                   want_boundary=True, want_h_out=True)
    torch.cuda.synchronize()
    o = oracle.train_blocks(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], w.K)
    assert bnd.shape == (1, 16, 64, 16)
    assert_c12(to_f64(y), o["y"], RTOL_Y["f32"], "y")
    assert_state(to_f64(bnd), o["boundary"], "16 block-boundary states")
    assert_state(to_f64(hout), o["h_out"], "final state")


def test_train_full_block_objective(bd):
    w = I.WORKLOADS["train"]
    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    s.update(I.make_params(w.seed, w.D, w.N))
    g = {k: to_dev(v) for k, v in s.items()}
    y, bnd, hout = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], w.K,
                                   want_boundary=True, want_h_out=True)
    _, ph, pb = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], w.K, want_y=False,
                           want_boundary=True)
    torch.cuda.synchronize()
    assert torch.equal(bnd, pb) and torch.equal(hout, ph), "training states must equal the prefill caches"
    ch = sample_channels(w.D, 16, 11)
    cht = ch.tolist()
    o = otrain(sub(s, ch), w.K)
    assert_c12(to_f64(y[:, :, cht]), o["y"], RTOL_Y[w.io], "y (sampled channels)")
    assert_state(to_f64(bnd[:, :, cht]), o["boundary"], "256 boundary states per sequence")


def _context_on_device(w, L_total, ch):
    """Generate the clean context stream chunk by chunk straight into device
    tensors; keep the sampled channels on the host for the oracle."""
    dev = {"x": torch.empty((w.batch, L_total, w.D), dtype=torch.bfloat16, device="cuda"),
           "dt": torch.empty((w.batch, L_total, w.D), dtype=torch.bfloat16, device="cuda"),
           "B": torch.empty((w.batch, L_total, w.N), dtype=torch.bfloat16, device="cuda"),
           "C": torch.empty((w.batch, L_total, w.N), dtype=torch.bfloat16, device="cuda")}
    host = {"x": np.empty((w.batch, L_total, len(ch)), np.uint16), "dt": np.empty((w.batch, L_total, len(ch)), np.uint16),
            "B": np.empty((w.batch, L_total, w.N), np.uint16), "C": np.empty((w.batch, L_total, w.N), np.uint16)}
    span = 8 * I.CHUNK
    for t0 in range(0, L_total, span):
        n = min(span, L_total - t0)
        s = I.make_sequence(w.seed, w.batch, n, w.D, w.N, w.io, stream=("context",), t0=t0)
        for k in dev:
            dev[k][:, t0:t0 + n] = to_dev(s[k])
        host["x"][:, t0:t0 + n] = s["x"][:, :, ch]
        host["dt"][:, t0:t0 + n] = s["dt"][:, :, ch]
        host["B"][:, t0:t0 + n] = s["B"]
        host["C"][:, t0:t0 + n] = s["C"]
    return dev, host


@pytest.mark.parametrize("name", ["step65k", "step262k"])
def test_inference_block_steps(bd, name):
    """Prefill the long context, then per block: `steps` denoising steps with
    fresh noisy inputs (forward from the cache + in-block reverse) and one
    commit of the clean block. The committed caches must equal a one-shot
    prefill over context + committed blocks (GPU, bit for bit) and the oracle."""
    w = I.WORKLOADS[name]
    K, L = w.K, w.L
    L_total = L + w.blocks * K
    ch = sample_channels(w.D, 8 if w.batch > 1 else 16, 13)
    p = I.make_params(w.seed, w.D, w.N)
    A, Dk = to_dev(p["A"]), to_dev(p["Dskip"])
    g, host = _context_on_device(w, L_total, ch)
    # one-shot prefill over everything (reference for cache exactness)
    _, h_all, bnd_all = bd.prefill(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, want_y=False, want_boundary=True)
    # the inference flow
    ctx = {k: v[:, :L] for k, v in g.items()}
    y_ctx, cache, _ = bd.prefill(ctx["x"].contiguous(), ctx["dt"].contiguous(), A, ctx["B"].contiguous(),
                                 ctx["C"].contiguous(), Dk, K)
    checked_steps = []
    for j in range(w.blocks):
        for st in range(w.steps):
            nz = I.make_sequence(w.seed, w.batch, K, w.D, w.N, w.io, stream=("noisy", j, st))
            gn = {k: to_dev(v) for k, v in nz.items()}
            y = bd.block_step(gn["x"], gn["dt"], A, gn["B"], gn["C"], Dk, cache)
            if st in (0, w.steps - 1):
                checked_steps.append((j, st, to_f64(y[:, :, ch.tolist()]), to_f64(cache[:, ch.tolist()]),
                                      {k: np.ascontiguousarray(nz[k][:, :, ch]) if k in ("x", "dt") else nz[k]
                                       for k in nz}))
        sl = slice(L + j * K, L + (j + 1) * K)
        bd.commit_block(g["x"][:, sl].contiguous(), g["dt"][:, sl].contiguous(), A, g["B"][:, sl].contiguous(),
                        g["C"][:, sl].contiguous(), Dk, cache)
        torch.cuda.synchronize()
        assert torch.equal(cache, bnd_all[:, L // K + j]), f"commit {j}: cache differs from one-shot prefill"
    assert torch.equal(cache, h_all)

    # oracle on sampled channels: context prefill, then the commits; the step outputs
    sp = {"A": np.ascontiguousarray(p["A"][ch]), "Dskip": np.ascontiguousarray(p["Dskip"][ch])}
    o = oracle.prefill(host["x"], host["dt"], sp["A"], host["B"], host["C"], sp["Dskip"], K)
    bnd_dev = to_f64(bnd_all[:, :, ch.tolist()])
    assert_state(bnd_dev[:, L // K + w.blocks - 1], o["boundary"][:, -1], "final cache vs oracle")
    assert_state(bnd_dev[:, L // K - 1], o["boundary"][:, L // K - 1], "context cache vs oracle")
    assert_c12(to_f64(y_ctx[:, :, ch.tolist()]), o["y"][:, :L], RTOL_Y[w.io], "context y vs oracle")
    for j, st, y_dev, cache_dev, nz in checked_steps:
        assert_state(cache_dev, o["boundary"][:, L // K - 1 + j], f"cache before block {j}")
        o_y = oracle.block_step(nz["x"], nz["dt"], sp["A"], nz["B"], nz["C"], sp["Dskip"],
                                np.ascontiguousarray(o["boundary"][:, L // K - 1 + j]))
        assert_c12(y_dev, o_y, RTOL_Y[w.io], f"step y block {j} step {st}")


def test_stack350m_block_sweep(bd):
    w = I.WORKLOADS["stack350m"]
    s = I.make_sequence(w.seed, w.batch, w.L, w.D, w.N, w.io)
    g = {k: to_dev(v) for k, v in s.items()}
    rng = np.random.default_rng(17)
    y = torch.empty((w.batch, w.L, w.D), dtype=torch.bfloat16, device="cuda")
    for K in I.STACK_BLOCK_SIZES:
        check_layers = {int(rng.integers(0, w.layers)), w.layers - 1}
        for layer in range(w.layers):
            p = I.make_params(w.seed, w.D, w.N, layer=layer)
            bd.train_blocks(g["x"], g["dt"], to_dev(p["A"]), g["B"], g["C"], to_dev(p["Dskip"]), K, y=y)
            if layer in check_layers:
                ch = sample_channels(w.D, 4, layer * 100 + K)
                rows = np.sort(rng.choice(w.batch, size=4, replace=False))
                torch.cuda.synchronize()
                got = to_f64(y[rows.tolist()][:, :, ch.tolist()])
                ss = {k: np.ascontiguousarray(v[rows]) for k, v in s.items()}
                ss.update(p)
                o = otrain(sub(ss, ch), K)
                assert_c12(got, o["y"], RTOL_Y[w.io], f"layer {layer} block {K}")
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all()

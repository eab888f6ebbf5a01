"""Two-stream all-block training pass (clean prefix stream + noisy active
blocks) on the GPU against the fp64 oracle."""
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


def streams(seed, Bt, L, D, N, io, gated):
    clean = I.make_sequence(seed, Bt, L, D, N, io, stream=("clean", 0), gated=gated)
    noisy = I.make_sequence(seed, Bt, L, D, N, io, stream=("noisy", 0, 0), gated=gated)
    return clean, noisy


CASES = [   # (Bt, L, D, N, K, io, gated, h0)
    (2, 96, 72, 16, 16, "bf16", True, True),
    (1, 64, 64, 16, 32, "f32", False, True),
    (2, 80, 40, 16, 4, "f32", False, False),
    (1, 90, 64, 16, 3, "bf16", False, True),
    (1, 96, 32, 16, 48, "f32", True, True),
    (2, 64, 24, 64, 16, "bf16", False, True),
    (1, 64, 16, 64, 4, "f32", True, False),
    (1, 128, 32, 64, 64, "bf16", True, True),
    (1, 512, 16, 64, 512, "bf16", False, True),
]


@pytest.mark.parametrize("Bt,L,D,N,K,io,gated,with_h0", CASES)
def test_two_stream_vs_oracle(bd, Bt, L, D, N, K, io, gated, with_h0):
    clean, noisy = streams(L + K + D + N, Bt, L, D, N, io, gated)
    p = I.make_params(L * 3 + K, D, N)
    h0 = I.make_state(K + N, Bt, D, N, scale=0.5) if with_h0 else None
    gc = {k: to_dev(v) for k, v in clean.items()}
    gn = {k: to_dev(v) for k, v in noisy.items()}
    yc, yn, bnd, hout = bd.train_two_stream(gc, gn, to_dev(p["A"]), to_dev(p["Dskip"]), K,
                                            h0=None if h0 is None else to_dev(h0), want_h_out=True)
    torch.cuda.synchronize()
    o = oracle.two_stream(clean, noisy, p["A"], p["Dskip"], K, h0=h0, z_noisy=noisy.get("z"))
    oc = oracle.prefill(clean["x"], clean["dt"], p["A"], clean["B"], clean["C"], p["Dskip"], K, z=clean.get("z"), h0=h0)
    assert_c12(to_f64(yn), o["y_noisy"], RTOL_Y[io], "y_noisy")
    assert_c12(to_f64(yc), oc["y"], RTOL_Y[io], "y_clean")
    assert_state(to_f64(bnd), o["boundary"], "clean caches")
    assert_state(to_f64(hout), o["h_out"], "final state")


@pytest.mark.parametrize("K", [16, 4, 48])
def test_noisy_equal_clean_is_the_single_stream_pass(bd, K):
    """Bit for bit: restarting each block from the clean cache is the carried state."""
    Bt, L, D, N = 2, 192, 64, 16
    clean, _ = streams(7 + K, Bt, L, D, N, "bf16", gated=True)
    p = I.make_params(8, D, N)
    g = {k: to_dev(v) for k, v in clean.items()}
    A, Dk = to_dev(p["A"]), to_dev(p["Dskip"])
    _, yn, bnd, _ = bd.train_two_stream(g, g, A, Dk, K)
    y1, b1, _ = bd.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, K, z=g["z"], want_boundary=True)
    torch.cuda.synchronize()
    assert torch.equal(yn, y1)
    assert torch.equal(bnd, b1)


def test_two_stream_training_size(bd):
    """The training workload's sizes, both streams; sampled channels vs the oracle."""
    w = I.WORKLOADS["train"]
    clean, noisy = streams(w.seed, w.batch, w.L, w.D, w.N, w.io, gated=False)
    p = I.make_params(w.seed, w.D, w.N)
    gc = {k: to_dev(v) for k, v in clean.items()}
    gn = {k: to_dev(v) for k, v in noisy.items()}
    yc, yn, bnd, _ = bd.train_two_stream(gc, gn, to_dev(p["A"]), to_dev(p["Dskip"]), w.K)
    torch.cuda.synchronize()
    ch = np.sort(np.random.default_rng(5).choice(w.D, size=8, replace=False))
    sub = lambda s: {k: (np.ascontiguousarray(v[:, :, ch]) if k in ("x", "dt") else v) for k, v in s.items()}  # noqa: E731
    o = oracle.two_stream(sub(clean), sub(noisy), np.ascontiguousarray(p["A"][ch]),
                          np.ascontiguousarray(p["Dskip"][ch]), w.K)
    cl = ch.tolist()
    assert_c12(to_f64(yn[:, :, cl]), o["y_noisy"], RTOL_Y[w.io], "y_noisy")
    assert_c12(to_f64(yc[:, :, cl]), o["y_clean"], RTOL_Y[w.io], "y_clean")
    assert_state(to_f64(bnd[:, :, cl]), o["boundary"], "clean caches")

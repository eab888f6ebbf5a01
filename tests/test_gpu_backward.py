"""GPU backward pass of the all-block training scan vs the fp64 CPU oracle's
adjoint, on shapes that span several 8-token tiles, ragged tails, short
blocks grouped into tiles, long blocks with checkpoints, both state sizes,
both I/O types, gated and ungated; plus determinism and the error paths."""
import numpy as np
import pytest

import oracle
from selective_ssm_scan_mamba_b200 import inputs as I
from tests.gpu_util import RTOL_GRAD, assert_c12, assert_state, to_dev, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def bd():
    from selective_ssm_scan_mamba_b200 import bdscan
    return bdscan


def make_case(seed, Bt, L, D, N, io, gated, with_h0, sp=True):
    s = I.make_sequence(seed, Bt, L, D, N, io, gated=gated)
    s.update(I.make_params(seed, D, N))
    if not sp:
        s["dt"] = I.f32_to_bf16_bits(np.abs(oracle.decode(s["dt"])).astype(np.float32) * 0.1) \
            if io == "bf16" else (np.abs(s["dt"]) * np.float32(0.1)).astype(np.float32)
    s["h0"] = I.make_state(seed + 1, Bt, D, N, scale=0.5) if with_h0 else None
    dy = I.make_state(seed + 2, Bt, L, D)
    s["dy"] = I.f32_to_bf16_bits(dy) if io == "bf16" else dy
    return s


def run_gpu(bd, s, K, sp=True):
    g = {k: (None if v is None else to_dev(v)) for k, v in s.items()}
    _, bnd, _ = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, z=g.get("z"), h0=g["h0"],
                                dt_softplus=sp, want_boundary=True)
    out = bd.train_blocks_backward(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, g["dy"], bnd,
                                   z=g.get("z"), h0=g["h0"], dt_softplus=sp)
    torch.cuda.synchronize()
    return out


def check(out, want, io):
    rt = RTOL_GRAD[io]
    for k in ("dx", "ddt", "dz", "dB", "dC"):
        if want[k] is None:
            assert out[k] is None
            continue
        assert_c12(to_f64(out[k]), want[k], rt, k)
    # parameter and state gradients are fp32 sums over many tokens: normwise
    assert_state(to_f64(out["dA"])[None], want["dA"][None], "dA", rtol=RTOL_GRAD["param"])
    assert_c12(to_f64(out["dDskip"]), want["dDskip"], RTOL_GRAD["param"], "dDskip")
    assert_state(to_f64(out["dh0"]), want["dh0"], "dh0", rtol=RTOL_GRAD["param"])


CASES = [
    # (Bt, L, D, N, K, io, gated, h0, softplus)
    (2, 96, 72, 16, 16, "f32", False, False, True),
    (2, 96, 72, 16, 16, "bf16", True, True, True),
    (1, 80, 64, 16, 4, "f32", True, True, True),
    (2, 90, 40, 16, 3, "f32", False, True, True),
    (1, 85, 24, 16, 17, "bf16", False, False, True),
    (1, 64, 16, 16, 1, "f32", True, True, True),
    (2, 144, 64, 16, 48, "f32", True, True, True),
    (1, 128, 32, 16, 64, "bf16", False, True, True),
    (1, 256, 32, 16, 256, "f32", True, False, True),
    (1, 96, 40, 16, 32, "f32", False, True, False),
    (2, 96, 24, 64, 16, "f32", False, True, True),
    (1, 96, 40, 64, 4, "bf16", True, False, True),
    (1, 128, 16, 64, 64, "f32", True, True, True),
    (1, 70, 24, 64, 7, "f32", False, True, True),
    (1, 40, 32, 16, 8, "f32", True, True, True),
    (1, 24, 32, 16, 24, "f32", True, True, True),
    # blocks of 16 at N = 16 (each block staged once): one block with a ragged
    # channel tile and no softplus, and ten gated blocks over three channel tiles
    (1, 16, 40, 16, 16, "bf16", False, True, False),
    (3, 160, 96, 16, 16, "f32", True, True, True),
]


@pytest.mark.parametrize("Bt,L,D,N,K,io,gated,with_h0,sp", CASES)
def test_backward_vs_oracle(bd, Bt, L, D, N, K, io, gated, with_h0, sp):
    s = make_case(L * 13 + K * 5 + D + N, Bt, L, D, N, io, gated, with_h0, sp)
    out = run_gpu(bd, s, K, sp)
    want = oracle.train_blocks_backward(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, s["dy"],
                                        z=s.get("z"), h0=s["h0"], dt_softplus=sp)
    check(out, want, io)


def test_backward_at_training_size_sampled(bd):
    """Batch 8 x 4096 tokens x 1536 channels, N = 16, blocks of 16, bf16.
    dx and d(dt) depend only on their own channel, dA and dDskip on their
    channel summed over the batch: the oracle recomputes a sample of channels
    in full for those. dB[b] and dC[b] sum over all channels of batch row b
    only (the GPU reduces 48 CTA partial rows per token): the oracle runs
    batch row 0 in full (4096 x 1536) and they are checked element by
    element there, together with that row's dx and d(dt)."""
    Bt, L, D, N, K = 8, 4096, 1536, 16, 16
    s = I.make_sequence(1, Bt, L, D, N, "bf16")
    s.update(I.make_params(1, D, N))
    rng = np.random.default_rng(77)
    dy = I.f32_to_bf16_bits(rng.standard_normal((Bt, L, D)).astype(np.float32))
    g = {k: to_dev(v) for k, v in s.items()}
    gdy = to_dev(dy)
    y, bnd, _ = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, want_boundary=True)
    out = bd.train_blocks_backward(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, gdy, bnd)
    torch.cuda.synchronize()
    ch = np.array([0, 1, 31, 32, 700, 1535])
    sub = {k: np.ascontiguousarray(s[k][:, :, ch]) for k in ("x", "dt")}
    want = oracle.train_blocks_backward(sub["x"], sub["dt"], s["A"][ch], s["B"], s["C"], s["Dskip"][ch], K,
                                        np.ascontiguousarray(dy[:, :, ch]))
    for k in ("dx", "ddt"):
        assert_c12(to_f64(out[k])[:, :, ch], want[k], RTOL_GRAD["bf16"], k)
    assert_state(to_f64(out["dA"])[ch][None], want["dA"][None], "dA", rtol=RTOL_GRAD["param"])
    assert_c12(to_f64(out["dDskip"])[ch], want["dDskip"], RTOL_GRAD["param"], "dDskip")
    # batch row 0 in full: dB and dC element by element
    row = {k: np.ascontiguousarray(s[k][:1]) for k in ("x", "dt", "B", "C")}
    want0 = oracle.train_blocks_backward(row["x"], row["dt"], s["A"], row["B"], row["C"], s["Dskip"], K,
                                         np.ascontiguousarray(dy[:1]))
    for k in ("dB", "dC", "dx", "ddt"):
        assert_c12(to_f64(out[k])[:1], want0[k], RTOL_GRAD["bf16"], f"{k} (batch row 0)")


def test_backward_is_deterministic(bd):
    s = make_case(5, 2, 256, 96, 16, "bf16", True, True)
    a = run_gpu(bd, s, 16)
    b = run_gpu(bd, s, 16)
    for k in a:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k


def test_backward_empty(bd):
    s = make_case(6, 1, 16, 32, 16, "f32", False, True)
    g = {k: (None if v is None else to_dev(v)) for k, v in s.items()}
    e = {k: v[:, :0].contiguous() for k, v in g.items() if k in ("x", "dt", "B", "C", "dy")}
    out = bd.train_blocks_backward(e["x"], e["dt"], g["A"], e["B"], e["C"], g["Dskip"], 16, e["dy"], None, h0=g["h0"])
    torch.cuda.synchronize()
    assert torch.count_nonzero(out["dA"]) == 0 and torch.count_nonzero(out["dDskip"]) == 0
    assert torch.count_nonzero(out["dh0"]) == 0


def test_backward_rejects_bad_arguments(bd):
    s = make_case(7, 1, 64, 32, 16, "f32", False, False)
    g = {k: (None if v is None else to_dev(v)) for k, v in s.items()}
    with pytest.raises(bd.BdscanError, match="INVALID_ARG"):   # boundary states required for L > K
        bd.train_blocks_backward(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, g["dy"], None)
    _, bnd, _ = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, want_boundary=True)
    need = bd.train_blocks_backward_workspace_bytes(g["x"], g["B"], 16)
    with pytest.raises(bd.BdscanError, match="WORKSPACE"):
        bd.train_blocks_backward(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, g["dy"], bnd,
                                 ws=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))

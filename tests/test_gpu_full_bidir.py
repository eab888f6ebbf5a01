"""Full-sequence bidirectional pass (the comparator the block-confined design
replaces) on the GPU: equals the all-block pass with one block of length L."""
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


@pytest.mark.parametrize("Bt,L,D,N,io,gated,with_h0", [
    (2, 100, 72, 16, "f32", True, True), (1, 1000, 64, 16, "bf16", False, False),
    (2, 64, 40, 64, "bf16", True, True), (1, 333, 16, 64, "f32", False, True), (1, 1, 8, 16, "bf16", True, False),
])
def test_full_bidirectional_vs_oracle(bd, Bt, L, D, N, io, gated, with_h0):
    s = I.make_sequence(L + D, Bt, L, D, N, io, gated=gated)
    p = I.make_params(L + N, D, N)
    h0 = I.make_state(L, Bt, D, N, scale=0.5) if with_h0 else None
    g = {k: to_dev(v) for k, v in s.items()}
    y, hout = bd.full_bidirectional(g["x"], g["dt"], to_dev(p["A"]), g["B"], g["C"], to_dev(p["Dskip"]),
                                    z=g.get("z"), h0=None if h0 is None else to_dev(h0), want_h_out=True)
    torch.cuda.synchronize()
    o = oracle.train_blocks(s["x"], s["dt"], p["A"], s["B"], s["C"], p["Dskip"], L, z=s.get("z"), h0=h0)
    # bf16 y is rounded twice (after the forward pass and at the end)
    assert_c12(to_f64(y), o["y"], RTOL_Y[io], "y")
    assert_state(to_f64(hout), o["h_out"], "final state")


def test_matches_long_block_pass(bd):
    Bt, L, D, N = 2, 512, 64, 16
    s = I.make_sequence(9, Bt, L, D, N, "f32")
    p = I.make_params(9, D, N)
    g = {k: to_dev(v) for k, v in s.items()}
    A, Dk = to_dev(p["A"]), to_dev(p["Dskip"])
    y1, _ = bd.full_bidirectional(g["x"], g["dt"], A, g["B"], g["C"], Dk)
    y2, _, _ = bd.train_blocks(g["x"], g["dt"], A, g["B"], g["C"], Dk, L)
    torch.cuda.synchronize()
    assert_c12(to_f64(y1), to_f64(y2), 1e-5, "full pass vs one-block pass")

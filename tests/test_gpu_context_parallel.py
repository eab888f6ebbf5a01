"""Context-parallel prefill kernels on one GPU: the ranks of a split context
are run one after another (the all-gather is a stack), and the chunks'
outputs must equal one prefill of the whole context and the oracle."""
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


@pytest.mark.parametrize("Bt,D,N,K,io,cuts", [
    (2, 64, 16, 16, "bf16", [0, 64, 160, 256]),        # three chunks of unequal length
    (1, 40, 16, 4, "f32", [0, 100, 200]),
    (1, 32, 64, 32, "bf16", [0, 96, 96, 192]),         # an empty chunk in the middle
    (2, 24, 16, 1, "f32", [0, 37, 80]),
])
def test_chunks_compose_to_one_prefill(bd, Bt, D, N, K, io, cuts):
    L = cuts[-1]
    s = I.make_sequence(L + D + K, Bt, L, D, N, io, gated=True)
    s.update(I.make_params(L + K, D, N))
    h0 = I.make_state(L + 1, Bt, D, N, scale=0.5)
    g = {k: to_dev(v) for k, v in s.items()}
    gh0 = to_dev(h0)
    pieces = [slice(a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    loc = [{k: g[k][:, sl].contiguous() for k in ("x", "dt", "B", "C", "z")} for sl in pieces]
    sums = [bd.chunk_summary(c["x"], c["dt"], g["A"], c["B"], c["C"], g["Dskip"], K) for c in loc]
    H_all = torch.stack([h for h, _ in sums])
    P_all = torch.stack([p for _, p in sums])
    ys, bnds, starts = [], [], []
    for r, c in enumerate(loc):
        h_in = bd.carry_fold(H_all, P_all, r, h0=gh0)
        starts.append(h_in)
        y, h, bnd = bd.prefill(c["x"], c["dt"], g["A"], c["B"], c["C"], g["Dskip"], K, z=c["z"], h0=h_in,
                               want_boundary=True)
        ys.append(y)
        bnds.append(bnd)
    torch.cuda.synchronize()
    o = oracle.prefill(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, z=s["z"], h0=h0)
    assert_c12(to_f64(torch.cat(ys, 1)), o["y"], RTOL_Y[io], "y")
    assert_state(to_f64(torch.cat(bnds, 1)), o["boundary"], "boundary states")
    assert_state(to_f64(h), o["h_out"], "final state")
    for r, sl in enumerate(pieces):   # each chunk's start state is the oracle's state there
        want = oracle.decode(h0) if sl.start == 0 else o["boundary"][:, sl.start // K - 1]
        assert_state(to_f64(starts[r]), want, f"start state of chunk {r}")


def test_summary_of_a_context(bd):
    """H is the state reached from zero; P is the product of the decays (the
    state reached from ones with x = 0); an empty context is the identity."""
    Bt, L, D, N, K = 2, 80, 32, 16, 16
    s = I.make_sequence(5, Bt, L, D, N, "f32")
    s.update(I.make_params(5, D, N))
    g = {k: to_dev(v) for k, v in s.items()}
    H, P = bd.chunk_summary(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K)
    He, Pe = bd.chunk_summary(g["x"][:, :0].contiguous(), g["dt"][:, :0].contiguous(), g["A"],
                              g["B"][:, :0].contiguous(), g["C"][:, :0].contiguous(), g["Dskip"], K)
    torch.cuda.synchronize()
    fH = oracle.forward(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K)["h_out"]
    fP = oracle.forward(np.zeros_like(s["x"]), s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K,
                        h0=np.ones((Bt, D, N)))["h_out"]
    assert_state(to_f64(H), fH, "H")
    # P multiplies L decays: each ex2 carries ~2^-22 relative error and its
    # argument delta*A*log2(e) the rounding of delta, which scales with |ln P|;
    # bound the relative error by 5e-7 * (L + |ln P|) where P is representable
    gP = to_f64(P)
    big = fP > 1e-30
    rel = np.abs(gP[big] - fP[big]) / fP[big]
    assert np.all(rel <= 5e-7 * (L + np.abs(np.log(fP[big])))), float(np.max(rel))
    assert np.all(np.abs(gP[~big]) <= 1e-29)
    assert torch.count_nonzero(He) == 0 and bool(torch.all(Pe == 1))


def test_carry_fold_rejects_bad_index(bd):
    H = torch.zeros(2, 1, 32, 16, device="cuda")
    with pytest.raises(bd.BdscanError, match="INVALID_ARG"):
        bd.carry_fold(H, H, 2)

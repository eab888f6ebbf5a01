"""The compiled per-step marshalling (block_step, commit_block, BlockStep) and
the ctypes marshalling reach the same C-ABI entry points: outputs bit for bit
equal, and the library's status passes through as the same exception."""
import pytest

from selective_ssm_scan_mamba_b200 import inputs as I
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture
def bd():
    from selective_ssm_scan_mamba_b200 import bdscan
    assert bdscan.FASTPATH_LOADED
    return bdscan


@pytest.mark.parametrize("Bt,K,D,N,io,gated", [(2, 32, 96, 16, "bf16", True), (1, 16, 64, 64, "f32", False)])
def test_compiled_and_ctypes_marshalling_agree(bd, monkeypatch, Bt, K, D, N, io, gated):
    s = I.make_sequence(K + D + N, Bt, K, D, N, io, gated=gated)
    s.update(I.make_params(K + D + N, D, N))
    g = {k: to_dev(v) for k, v in s.items()}
    h = to_dev(I.make_state(K + D + N + 1, Bt, D, N, scale=0.5))
    z = g.get("z")
    fast = bd._fast
    y_fast = bd.block_step(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], h, z=z)
    y_prep = bd.BlockStep(g["A"], g["Dskip"], h, K, dtype=g["x"].dtype, gated=gated)(g["x"], g["dt"], g["B"], g["C"],
                                                                                      z=z)
    h_fast = h.clone()
    yc_fast = bd.commit_block(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], h_fast, z=z, want_y=True)
    monkeypatch.setattr(bd, "_fast", None)   # the ctypes marshalling alone
    y_ct = bd.block_step(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], h, z=z)
    y_prep_ct = bd.BlockStep(g["A"], g["Dskip"], h, K, dtype=g["x"].dtype, gated=gated)(g["x"], g["dt"], g["B"],
                                                                                         g["C"], z=z)
    h_ct = h.clone()
    yc_ct = bd.commit_block(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], h_ct, z=z, want_y=True)
    torch.cuda.synchronize()
    assert torch.equal(y_fast, y_ct) and torch.equal(y_prep, y_ct) and torch.equal(y_prep_ct, y_ct)
    assert torch.equal(yc_fast, yc_ct) and torch.equal(h_fast, h_ct)
    monkeypatch.setattr(bd, "_fast", fast)
    # a caller's y is written in place
    y_out = torch.empty_like(y_ct)
    assert bd.block_step(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], h, z=z, y=y_out) is y_out
    torch.cuda.synchronize()
    assert torch.equal(y_out, y_ct)


def test_library_status_passes_through_the_compiled_path(bd):
    # N = 32 is outside the supported state sizes: the library refuses it
    # before any launch, and the compiled path raises what the ctypes path does
    Bt, K, D, N = 1, 16, 64, 32
    x = torch.zeros(Bt, K, D, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(Bt, K, N, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(D, N, device="cuda")
    Dk = torch.zeros(D, device="cuda")
    h = torch.zeros(Bt, D, N, device="cuda")
    with pytest.raises(bd.BdscanError) as e:
        bd.block_step(x, x, A, B, B, Dk, h)
    assert e.value.status == 2
    with pytest.raises(bd.BdscanError) as e:
        bd.commit_block(x, x, A, B, B, Dk, h)
    assert e.value.status == 2

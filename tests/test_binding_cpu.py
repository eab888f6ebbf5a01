"""The Python binding's marshalling, driven on CPU tensors against a fake
library that records each call (no GPU, no kernel launch)."""
import ctypes as ct

import pytest
import torch

from selective_ssm_scan_mamba_b200 import bdscan


class FakeLib:
    def __init__(self, rc=0):
        self.calls = []
        self.rc = rc

    def _rec(self, name):
        def f(*args):
            self.calls.append((name, args))
            return self.rc
        return f

    def __getattr__(self, name):
        if name.startswith("bdscan_"):
            return self._rec(name)
        raise AttributeError(name)


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(bdscan, "_lib", lib)
    monkeypatch.setattr(bdscan, "_check_device", lambda d: None)
    monkeypatch.setattr(bdscan, "_stream", lambda d: 1234)
    return lib


def tensors(Bt=2, L=32, D=64, N=16, io=torch.bfloat16):
    return dict(x=torch.zeros(Bt, L, D, dtype=io), dt=torch.zeros(Bt, L, D, dtype=io),
                A=torch.zeros(D, N), B=torch.zeros(Bt, L, N, dtype=io), C=torch.zeros(Bt, L, N, dtype=io),
                Dskip=torch.zeros(D))


def _dims(arg):
    return ct.cast(arg, ct.POINTER(bdscan.Dims)).contents if not isinstance(arg, bdscan.Dims) else arg


def test_train_blocks_marshalling(fake):
    t = tensors()
    y, bnd, h = bdscan.train_blocks(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16,
                                    want_boundary=True, want_h_out=True)
    name, args = fake.calls[-1]
    assert name == "bdscan_train_blocks"
    assert y.shape == (2, 32, 64) and y.dtype == torch.bfloat16
    assert bnd.shape == (2, 2, 64, 16) and h.shape == (2, 64, 16)
    assert args[2] is None and args[3] == y.data_ptr() and args[4] == bnd.data_ptr() and args[5] == h.data_ptr()
    assert args[6] == 1234


def test_each_entry_point_reaches_the_library(fake):
    t = tensors(L=16)
    cache = torch.zeros(2, 64, 16)
    bdscan.prefill(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16)
    bdscan.block_step(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], cache)
    bdscan.commit_block(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], cache, want_y=True)
    assert [c[0] for c in fake.calls] == ["bdscan_prefill", "bdscan_block_step", "bdscan_commit_block"]
    assert fake.calls[1][1][2] == cache.data_ptr() and fake.calls[2][1][2] == cache.data_ptr()


def test_status_becomes_exception(monkeypatch):
    lib = FakeLib(rc=2)
    lib.bdscan_status_string = lambda s: b"BDSCAN_ERR_UNSUPPORTED"
    monkeypatch.setattr(bdscan, "_lib", lib)
    monkeypatch.setattr(bdscan, "_check_device", lambda d: None)
    monkeypatch.setattr(bdscan, "_stream", lambda d: 0)
    t = tensors()
    with pytest.raises(bdscan.BdscanError, match="UNSUPPORTED"):
        bdscan.train_blocks(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16)


def test_shape_dtype_and_layout_checks(fake):
    t = tensors()
    with pytest.raises(TypeError):
        bdscan.train_blocks(t["x"].float(), t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16)
    with pytest.raises(ValueError):
        bdscan.train_blocks(t["x"], t["dt"], t["A"][:32], t["B"], t["C"], t["Dskip"], 16)
    with pytest.raises(ValueError):
        bdscan.train_blocks(t["x"].transpose(1, 2).contiguous().transpose(1, 2), t["dt"], t["A"], t["B"],
                            t["C"], t["Dskip"], 16)
    assert not fake.calls


def test_cpu_tensors_are_refused_without_fallback():
    t = tensors()
    with pytest.raises(ValueError, match="CUDA"):
        bdscan.train_blocks(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16)


def test_backward_marshalling(fake):
    t = tensors()
    z = torch.zeros(2, 32, 64, dtype=torch.bfloat16)
    dy = torch.zeros(2, 32, 64, dtype=torch.bfloat16)
    bnd = torch.zeros(2, 2, 64, 16)
    h0 = torch.zeros(2, 64, 16)
    g = bdscan.train_blocks_backward(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16, dy, bnd, z=z, h0=h0)
    name, args = fake.calls[-1]
    assert name == "bdscan_train_blocks_backward"
    assert args[2] == h0.data_ptr() and args[3] == bnd.data_ptr() and args[4] == dy.data_ptr()
    gr = ct.cast(args[5], ct.POINTER(bdscan.Grads)).contents
    for k in ("dx", "ddt", "dz", "dB", "dC", "dA", "dDskip", "dh0"):
        assert getattr(gr, k) == g[k].data_ptr(), k
    assert g["dx"].dtype == torch.bfloat16 and g["dA"].dtype == torch.float32 and g["dB"].shape == (2, 32, 16)
    assert args[8] == 1234
    # no gate: no dz output and a NULL pointer for it
    g2 = bdscan.train_blocks_backward(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16, dy, bnd,
                                      want_dh0=False)
    gr2 = ct.cast(fake.calls[-1][1][5], ct.POINTER(bdscan.Grads)).contents
    assert g2["dz"] is None and gr2.dz is None and g2["dh0"] is None and gr2.dh0 is None


def test_noalloc_prefill_needs_caller_outputs(fake):
    t = tensors()
    y = torch.zeros(2, 32, 64, dtype=torch.bfloat16)
    h = torch.zeros(2, 64, 16)
    bdscan.prefill_chunked_noalloc(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16, y, h)
    name, args = fake.calls[-1]
    assert name == "bdscan_prefill_chunked_noalloc"
    assert args[3] == y.data_ptr() and args[4] == h.data_ptr() and args[5] is None and args[6] == 1234
    with pytest.raises(ValueError):   # outputs are checked like inputs
        bdscan.prefill_chunked_noalloc(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], 16, y[:, :16], h)


def test_prepared_block_step_marshalling(fake):
    t = tensors(L=32)
    h = torch.zeros(2, 64, 16)
    step = bdscan.BlockStep(t["A"], t["Dskip"], h, 32)
    y = step(t["x"], t["dt"], t["B"], t["C"])
    name, args = fake.calls[-1]
    assert name == "bdscan_block_step"
    d = _dims(args[0]._obj)
    assert (d.batch, d.seqlen, d.d_inner, d.d_state, d.block, d.io_dtype, d.dt_softplus) == (2, 32, 64, 16, 32, 1, 1)
    ins = args[1]._obj
    assert (ins.x, ins.dt, ins.B, ins.C, ins.z) == (t["x"].data_ptr(), t["dt"].data_ptr(), t["B"].data_ptr(),
                                                    t["C"].data_ptr(), None)
    assert (ins.A, ins.Dskip) == (t["A"].data_ptr(), t["Dskip"].data_ptr())
    assert args[2] == h.data_ptr() and args[3] == y.data_ptr() and args[4] == 1234
    y2 = torch.empty_like(y)
    assert step(t["x"], t["dt"], t["B"], t["C"], y=y2) is y2
    with pytest.raises(ValueError, match="shape"):        # a block of another length
        step(t["x"][:, :16].contiguous(), t["dt"], t["B"], t["C"])
    with pytest.raises(TypeError, match="dtype"):
        step(t["x"].float(), t["dt"], t["B"], t["C"])
    with pytest.raises(ValueError, match="gate"):
        step(t["x"], t["dt"], t["B"], t["C"], z=t["x"])
    with pytest.raises(ValueError, match="shape"):        # A of another width than the cache
        bdscan.BlockStep(torch.zeros(32, 16), t["Dskip"], h, 32)
    gated = bdscan.BlockStep(t["A"], t["Dskip"], h, 32, gated=True)
    with pytest.raises(TypeError, match="Tensor"):
        gated(t["x"], t["dt"], t["B"], t["C"])
    gated(t["x"], t["dt"], t["B"], t["C"], z=t["x"])
    assert fake.calls[-1][1][1]._obj.z == t["x"].data_ptr()


def test_compiled_step_marshalling_declines_other_cases():
    """The compiled per-step module loads with the binding and links the same
    library. For anything outside the common case (here: CPU tensors, a
    non-tensor argument) it answers NOT_COMMON without a library call, and the
    checked path raises the specific error as before."""
    assert bdscan.FASTPATH_LOADED
    f = bdscan._fast
    t = tensors(L=32)
    h = torch.zeros(2, 64, 16)
    rc, y = f.block_step(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], h, None, True, None)
    assert rc == f.NOT_COMMON and y is None
    rc, y = f.commit_block(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], h, None, True, True, None)
    assert rc == f.NOT_COMMON and y is None
    rc, y = f.prepared_step(t["x"], t["dt"], t["B"], t["C"], None, None, 2, 32, 64, 16, True, True, 0, 0, 0)
    assert rc == f.NOT_COMMON and y is None
    with pytest.raises(ValueError, match="CUDA"):
        bdscan.block_step(t["x"], t["dt"], t["A"], t["B"], t["C"], t["Dskip"], h)


def test_non_tensor_argument_reaches_the_checked_path(fake):
    # the compiled module's argument conversion refuses a list; the checked
    # path then names the argument
    t = tensors(L=32)
    h = torch.zeros(2, 64, 16)
    with pytest.raises(TypeError, match="Dskip must be a torch.Tensor"):
        bdscan.block_step(t["x"], t["dt"], t["A"], t["B"], t["C"], [0.0], h)
    with pytest.raises(TypeError, match="Dskip must be a torch.Tensor"):
        bdscan.commit_block(t["x"], t["dt"], t["A"], t["B"], t["C"], [0.0], h)
    assert fake.calls == []

"""Python binding of ``libbdscan.so`` (C ABI in ``include/bdscan.h``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, output tensors are allocated with PyTorch when the caller does not
pass them, and the call is queued on PyTorch's current CUDA stream. Every step
of the scan runs in the library's CUDA kernels; there is no other code path.
If the library has not been built this module fails to import.
"""
from __future__ import annotations

import ctypes as ct
import importlib.util
import os
import sysconfig

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libbdscan.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m selective_ssm_scan_mamba_b200.build`")
_lib = ct.CDLL(_LIB_PATH)

F32, BF16 = 0, 1
_STATUS = {0: "BDSCAN_OK", 1: "BDSCAN_ERR_INVALID_ARG", 2: "BDSCAN_ERR_UNSUPPORTED",
           3: "BDSCAN_ERR_ALIGNMENT", 4: "BDSCAN_ERR_WORKSPACE", 5: "BDSCAN_ERR_CUDA"}


class Dims(ct.Structure):
    _fields_ = [("batch", ct.c_int64), ("seqlen", ct.c_int64), ("d_inner", ct.c_int64),
                ("d_state", ct.c_int64), ("block", ct.c_int64), ("io_dtype", ct.c_int32),
                ("dt_softplus", ct.c_int32)]


class Inputs(ct.Structure):
    _fields_ = [("x", ct.c_void_p), ("dt", ct.c_void_p), ("B", ct.c_void_p), ("C", ct.c_void_p),
                ("z", ct.c_void_p), ("A", ct.c_void_p), ("Dskip", ct.c_void_p)]


class Grads(ct.Structure):
    _fields_ = [("dx", ct.c_void_p), ("ddt", ct.c_void_p), ("dz", ct.c_void_p), ("dB", ct.c_void_p),
                ("dC", ct.c_void_p), ("dA", ct.c_void_p), ("dDskip", ct.c_void_p), ("dh0", ct.c_void_p)]


_vp = ct.c_void_p
_P = ct.POINTER
_lib.bdscan_train_blocks.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _vp, _vp]
_lib.bdscan_prefill.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _vp, _vp]
_lib.bdscan_block_step.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp]
_lib.bdscan_commit_block.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp]
_lib.bdscan_train_two_stream.argtypes = [_P(Dims), _P(Inputs), _P(Inputs), _vp, _vp, _vp, _vp, _vp, _vp]
_lib.bdscan_full_bidirectional.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _vp]
_lib.bdscan_prefill_chunked.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _vp, _vp, ct.c_size_t, _vp]
_lib.bdscan_prefill_chunked_noalloc.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _vp, _vp]
_lib.bdscan_train_blocks_backward.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp, _P(Grads), _vp, ct.c_size_t,
                                              _vp]
_lib.bdscan_train_blocks_backward_workspace.argtypes = [_P(Dims)]
_lib.bdscan_train_blocks_backward_workspace.restype = ct.c_size_t
_lib.bdscan_chunk_summary.argtypes = [_P(Dims), _P(Inputs), _vp, _vp, _vp]
_lib.bdscan_carry_fold.argtypes = [ct.c_int64, ct.c_int64, ct.c_int64, _vp, _vp, _vp, _vp, _vp]
_lib.bdscan_prefill_chunked_workspace.argtypes = [_P(Dims)]
_lib.bdscan_prefill_chunked_workspace.restype = ct.c_size_t
for _f in ("bdscan_train_blocks", "bdscan_prefill", "bdscan_block_step", "bdscan_commit_block",
           "bdscan_train_two_stream", "bdscan_full_bidirectional", "bdscan_prefill_chunked", "bdscan_prefill_chunked_noalloc",
           "bdscan_train_blocks_backward", "bdscan_chunk_summary", "bdscan_carry_fold", "bdscan_version"):
    getattr(_lib, _f).restype = ct.c_int
_lib.bdscan_status_string.argtypes = [ct.c_int]
_lib.bdscan_status_string.restype = ct.c_char_p
_lib.bdscan_last_cuda_error.restype = ct.c_char_p

LIBRARY_PATH = _LIB_PATH
version = _lib.bdscan_version

# The compiled per-step marshalling module (csrc/bdscan_fastpath.cpp): the same
# checks and the same C-ABI calls for block_step / commit_block / BlockStep,
# without the interpreter's per-attribute cost. It answers NOT_COMMON for any
# case outside the common one, which then takes the checked path below.
_FAST_PATH = os.path.join(os.path.dirname(_LIB_PATH), "_bdscan_fast" + sysconfig.get_config_var("EXT_SUFFIX"))
_fast = None
if os.path.exists(_FAST_PATH):
    _spec = importlib.util.spec_from_file_location("_bdscan_fast", _FAST_PATH)
    _fast = importlib.util.module_from_spec(_spec)
    _spec.loader.exec_module(_fast)
FASTPATH_LOADED = _fast is not None


class BdscanError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {_lib.bdscan_status_string(status).decode()}"
        if status == 5:
            msg += f" ({_lib.bdscan_last_cuda_error().decode()})"
        super().__init__(msg)
        self.status = status


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype, shape, device):
    # one combined test on the common path; the specific error only on failure
    if (isinstance(t, torch.Tensor) and t.dtype == dtype and t.shape == shape and t.is_contiguous()
            and t.device == device):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_DIMS = {}   # Dims structs by value (read-only once built; the library only reads them during a call)


def _dims_of(Bt, L, D, N, K, io, dt_softplus):
    key = (Bt, L, D, N, K, io, dt_softplus)
    d = _DIMS.get(key)
    if d is None:
        if len(_DIMS) >= 256:
            _DIMS.clear()
        d = _DIMS[key] = Dims(*key)
    return d


def _prepare(x, dt, A, B, C_, Dskip, block, z, dt_softplus):
    if not isinstance(x, torch.Tensor) or x.dim() != 3:
        raise ValueError("x must be a [batch, L, D] tensor")
    dev = x.device
    _check_device(dev)
    Bt, L, D = x.shape
    N = B.shape[-1] if isinstance(B, torch.Tensor) and B.dim() == 3 else -1
    io = x.dtype
    if io is not torch.float32 and io is not torch.bfloat16:
        raise TypeError("io dtype must be float32 or bfloat16")
    xs, bs, f32 = x.shape, (Bt, L, N), torch.float32
    # the common path: one pass of cheap tests; the specific error from _need otherwise
    T = torch.Tensor
    if not (x.is_contiguous()
            and isinstance(dt, T) and dt.dtype is io and dt.shape == xs and dt.is_contiguous() and dt.device == dev
            and isinstance(B, T) and B.dtype is io and B.shape == bs and B.is_contiguous() and B.device == dev
            and isinstance(C_, T) and C_.dtype is io and C_.shape == bs and C_.is_contiguous() and C_.device == dev
            and isinstance(A, T) and A.dtype is f32 and A.shape == (D, N) and A.is_contiguous() and A.device == dev
            and isinstance(Dskip, T) and Dskip.dtype is f32 and Dskip.shape == (D,) and Dskip.is_contiguous()
            and Dskip.device == dev):
        for t, name, dtp, shp in ((x, "x", io, (Bt, L, D)), (dt, "dt", io, (Bt, L, D)), (B, "B", io, bs),
                                  (C_, "C", io, bs), (A, "A", f32, (D, N)), (Dskip, "Dskip", f32, (D,))):
            _need(t, name, dtp, shp, dev)
    if z is not None:
        _need(z, "z", io, (Bt, L, D), dev)
    dims = _dims_of(Bt, L, D, N, int(block), BF16 if io is torch.bfloat16 else F32, 1 if dt_softplus else 0)
    ins = Inputs(x.data_ptr(), dt.data_ptr(), B.data_ptr(), C_.data_ptr(), None if z is None else z.data_ptr(),
                 A.data_ptr(), Dskip.data_ptr())
    return dims, ins, (Bt, L, D, N), io, dev


def _check_device(device):
    if device.type != "cuda":
        raise ValueError("bdscan runs on CUDA tensors only")


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(dev):
    """The current CUDA stream of dev as a raw handle (the call is queued there)."""
    if _raw_stream is not None:
        return _raw_stream(dev.index if dev.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(dev).cuda_stream


def _check(rc, where):
    if rc != 0:
        raise BdscanError(rc, where)


def train_blocks(x, dt, A, B, C, Dskip, block, z=None, h0=None, dt_softplus=True,
                 y=None, boundary=None, h_out=None, want_boundary=False, want_h_out=False):
    """Full-block pass over every block of every sequence: returns (y, boundary, h_out).

    boundary / h_out are returned when passed in or requested, else None.
    """
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    y = torch.empty((Bt, L, D), dtype=io, device=dev) if y is None else y
    _need(y, "y", io, (Bt, L, D), dev)
    if boundary is None and want_boundary:
        boundary = torch.empty((Bt, L // max(int(block), 1), D, N), dtype=torch.float32, device=dev)
    if boundary is not None:
        _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    if h_out is None and want_h_out:
        h_out = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
    if h_out is not None:
        _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    rc = _lib.bdscan_train_blocks(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(y), _ptr(boundary),
                                  _ptr(h_out), _stream(dev))
    _check(rc, "bdscan_train_blocks")
    return y, boundary, h_out


def prefill(x, dt, A, B, C, Dskip, block, z=None, h0=None, dt_softplus=True,
            want_y=True, y=None, h_out=None, boundary=None, want_boundary=False):
    """Forward-only scan of a clean context: returns (y or None, h_out, boundary or None)."""
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    if y is None and want_y:
        y = torch.empty((Bt, L, D), dtype=io, device=dev)
    if y is not None:
        _need(y, "y", io, (Bt, L, D), dev)
    h_out = torch.empty((Bt, D, N), dtype=torch.float32, device=dev) if h_out is None else h_out
    _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    if boundary is None and want_boundary:
        boundary = torch.empty((Bt, L // int(block), D, N), dtype=torch.float32, device=dev)
    if boundary is not None:
        _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    rc = _lib.bdscan_prefill(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(y), _ptr(h_out),
                             _ptr(boundary), _stream(dev))
    _check(rc, "bdscan_prefill")
    return y, h_out, boundary


def prefill_chunked_workspace_bytes(x, B, block, io_dtype=None):
    """Scratch bytes bdscan_prefill_chunked needs for these sizes on the current device."""
    Bt, L, D = x.shape
    dims = Dims(Bt, L, D, B.shape[-1], int(block), BF16 if x.dtype == torch.bfloat16 else F32, 1)
    return int(_lib.bdscan_prefill_chunked_workspace(ct.byref(dims)))


def prefill_chunked(x, dt, A, B, C, Dskip, block, z=None, h0=None, dt_softplus=True,
                    want_y=True, y=None, h_out=None, boundary=None, want_boundary=False, ws=None):
    """Time-chunked prefill (see include/bdscan.h): returns (y or None, h_out, boundary or None).

    ws: optional uint8 device tensor of at least prefill_chunked_workspace_bytes(); allocated here if None.
    """
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    if y is None and want_y:
        y = torch.empty((Bt, L, D), dtype=io, device=dev)
    if y is not None:
        _need(y, "y", io, (Bt, L, D), dev)
    h_out = torch.empty((Bt, D, N), dtype=torch.float32, device=dev) if h_out is None else h_out
    _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    if boundary is None and want_boundary:
        boundary = torch.empty((Bt, L // int(block), D, N), dtype=torch.float32, device=dev)
    if boundary is not None:
        _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    need = int(_lib.bdscan_prefill_chunked_workspace(ct.byref(dims)))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rc = _lib.bdscan_prefill_chunked(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(y), _ptr(h_out),
                                     _ptr(boundary), _ptr(ws), ws.numel() * ws.element_size(), _stream(dev))
    _check(rc, "bdscan_prefill_chunked")
    return y, h_out, boundary


def prefill_chunked_noalloc(x, dt, A, B, C, Dskip, block, y, h_out, z=None, h0=None, dt_softplus=True,
                            boundary=None):
    """Time-chunked prefill on the library's fixed 8 MiB device scratch: writes y, h_out and
    (if given) boundary, all caller-owned, and allocates nothing. Raises BdscanError
    (WORKSPACE) when the sizes need more scratch than that."""
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    _need(y, "y", io, (Bt, L, D), dev)
    _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    if boundary is not None:
        _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    rc = _lib.bdscan_prefill_chunked_noalloc(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(y), _ptr(h_out),
                                             _ptr(boundary), _stream(dev))
    _check(rc, "bdscan_prefill_chunked_noalloc")
    return y, h_out, boundary


def train_blocks_backward_workspace_bytes(x, B, block):
    """Scratch bytes bdscan_train_blocks_backward needs for these sizes."""
    Bt, L, D = x.shape
    dims = Dims(Bt, L, D, B.shape[-1], int(block), BF16 if x.dtype == torch.bfloat16 else F32, 1)
    return int(_lib.bdscan_train_blocks_backward_workspace(ct.byref(dims)))


def train_blocks_backward(x, dt, A, B, C, Dskip, block, dy, boundary, z=None, h0=None, dt_softplus=True,
                          want_dh0=True, grads=None, ws=None):
    """Gradients of train_blocks' y w.r.t. every input, given dy and the forward's boundary states.

    Returns dict(dx, ddt, dz (None without z), dB, dC, dA, dDskip, dh0 (None unless want_dh0)).
    grads: optional dict of preallocated outputs; ws: optional uint8 device scratch.
    """
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    _need(dy, "dy", io, (Bt, L, D), dev)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    if boundary is not None:
        _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    g = dict(grads or {})
    shapes = {"dx": ((Bt, L, D), io), "ddt": ((Bt, L, D), io), "dz": ((Bt, L, D), io), "dB": ((Bt, L, N), io),
              "dC": ((Bt, L, N), io), "dA": ((D, N), torch.float32), "dDskip": ((D,), torch.float32),
              "dh0": ((Bt, D, N), torch.float32)}
    for k, (shp, dtp) in shapes.items():
        if (k == "dz" and z is None) or (k == "dh0" and not want_dh0):
            g[k] = None
            continue
        if g.get(k) is None:
            g[k] = torch.empty(shp, dtype=dtp, device=dev)
        _need(g[k], k, dtp, shp, dev)
    need = int(_lib.bdscan_train_blocks_backward_workspace(ct.byref(dims)))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    gr = Grads(*[_ptr(g[k]) for k in ("dx", "ddt", "dz", "dB", "dC", "dA", "dDskip", "dh0")])
    rc = _lib.bdscan_train_blocks_backward(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(boundary), _ptr(dy),
                                           ct.byref(gr), _ptr(ws), ws.numel() * ws.element_size(), _stream(dev))
    _check(rc, "bdscan_train_blocks_backward")
    return g


def chunk_summary(x, dt, A, B, C, Dskip, block, dt_softplus=True, H=None, P=None):
    """(H, P) of the context: the state it reaches from zero and the product of its decays, [batch, D, N]."""
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, None, dt_softplus)
    H = torch.empty((Bt, D, N), dtype=torch.float32, device=dev) if H is None else H
    P = torch.empty((Bt, D, N), dtype=torch.float32, device=dev) if P is None else P
    _need(H, "H", torch.float32, (Bt, D, N), dev)
    _need(P, "P", torch.float32, (Bt, D, N), dev)
    rc = _lib.bdscan_chunk_summary(ct.byref(dims), ct.byref(ins), _ptr(H), _ptr(P), _stream(dev))
    _check(rc, "bdscan_chunk_summary")
    return H, P


def carry_fold(H_all, P_all, index, h0=None, out=None):
    """Start state of chunk `index` from the chunks' summaries H_all, P_all ([chunks, batch, D, N]) and h0."""
    if not isinstance(H_all, torch.Tensor) or H_all.dim() != 4:
        raise ValueError("H_all must be a [chunks, batch, D, N] tensor")
    _check_device(H_all.device)
    dev = H_all.device
    shape = tuple(H_all.shape)
    _need(H_all, "H_all", torch.float32, shape, dev)
    _need(P_all, "P_all", torch.float32, shape, dev)
    if h0 is not None:
        _need(h0, "h0", torch.float32, shape[1:], dev)
    out = torch.empty(shape[1:], dtype=torch.float32, device=dev) if out is None else out
    _need(out, "out", torch.float32, shape[1:], dev)
    count = shape[1] * shape[2] * shape[3]
    rc = _lib.bdscan_carry_fold(shape[0], int(index), count, _ptr(h0), _ptr(H_all), _ptr(P_all), _ptr(out),
                                _stream(dev))
    _check(rc, "bdscan_carry_fold")
    return out


def block_step(x, dt, A, B, C, Dskip, h_cache, z=None, dt_softplus=True, y=None):
    """One denoising step of the active block (L == block): returns y. h_cache is read only."""
    if _fast is not None:
        try:
            rc, yo = _fast.block_step(x, dt, A, B, C, Dskip, h_cache, z, bool(dt_softplus), y)
        except TypeError:   # an argument that is not a tensor: the checked path names it
            rc = _fast.NOT_COMMON
        if rc == 0:
            return yo
        if rc != _fast.NOT_COMMON:
            raise BdscanError(rc, "bdscan_block_step")
    block = x.shape[1]
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    _need(h_cache, "h_cache", torch.float32, (Bt, D, N), dev)
    y = torch.empty((Bt, L, D), dtype=io, device=dev) if y is None else y
    _need(y, "y", io, (Bt, L, D), dev)
    rc = _lib.bdscan_block_step(ct.byref(dims), ct.byref(ins), _ptr(h_cache), _ptr(y), _stream(dev))
    _check(rc, "bdscan_block_step")
    return y


class BlockStep:
    """A block step prepared for one shape, for denoising loops that call it
    many times: A, Dskip and the cache are checked once here, and each call
    checks only the step's own tensors (shape, dtype, device, contiguity) and
    marshals pointers. Calling it returns y = bdscan_block_step(x, dt, B, C)
    with the prepared A, Dskip, h_cache (read only) and gate flag; y may be
    passed in to avoid an allocation."""

    def __init__(self, A, Dskip, h_cache, block, dtype=torch.bfloat16, dt_softplus=True, gated=False):
        if not isinstance(h_cache, torch.Tensor) or h_cache.dim() != 3:
            raise ValueError("h_cache must be a [batch, D, N] tensor")
        _check_device(h_cache.device)
        Bt, D, N = h_cache.shape
        dev = h_cache.device
        if dtype not in (torch.float32, torch.bfloat16):
            raise TypeError("io dtype must be float32 or bfloat16")
        _need(h_cache, "h_cache", torch.float32, (Bt, D, N), dev)
        _need(A, "A", torch.float32, (D, N), dev)
        _need(Dskip, "Dskip", torch.float32, (D,), dev)
        self._keep = (A, Dskip, h_cache)   # the prepared pointers stay valid while this object lives
        self.dev, self.io, self.gated = dev, dtype, bool(gated)
        K = int(block)
        self.xshape, self.bshape = torch.Size((Bt, K, D)), torch.Size((Bt, K, N))
        self._dims = Dims(Bt, K, D, N, K, BF16 if dtype == torch.bfloat16 else F32, 1 if dt_softplus else 0)
        self._ins = Inputs(None, None, None, None, None, A.data_ptr(), Dskip.data_ptr())
        self._h = h_cache.data_ptr()
        self._dims_ref, self._ins_ref = ct.byref(self._dims), ct.byref(self._ins)
        self._fast_args = (Bt, K, D, N, dtype == torch.bfloat16, bool(dt_softplus), A.data_ptr(), Dskip.data_ptr(),
                           self._h)

    def __call__(self, x, dt, B, C, y=None, z=None):
        if _fast is not None and (z is not None) == self.gated:
            try:
                rc, yo = _fast.prepared_step(x, dt, B, C, z, y, *self._fast_args)
            except TypeError:
                rc = _fast.NOT_COMMON
            if rc == 0:
                return yo
            if rc != _fast.NOT_COMMON:
                raise BdscanError(rc, "bdscan_block_step")
        xs, bs, io, dev = self.xshape, self.bshape, self.io, self.dev
        for t, name, shp in ((x, "x", xs), (dt, "dt", xs), (B, "B", bs), (C, "C", bs)):
            _need(t, name, io, shp, dev)
        if self.gated:
            _need(z, "z", io, xs, dev)
        elif z is not None:
            raise ValueError("this BlockStep was prepared without a gate")
        if y is None:
            y = torch.empty(xs, dtype=io, device=dev)
        else:
            _need(y, "y", io, xs, dev)
        ins = self._ins
        ins.x, ins.dt, ins.B, ins.C = x.data_ptr(), dt.data_ptr(), B.data_ptr(), C.data_ptr()
        ins.z = z.data_ptr() if self.gated else None
        rc = _lib.bdscan_block_step(self._dims_ref, self._ins_ref, self._h, y.data_ptr(), _stream(dev))
        if rc != 0:
            raise BdscanError(rc, "bdscan_block_step")
        return y


def commit_block(x, dt, A, B, C, Dskip, h_cache, z=None, dt_softplus=True, want_y=False, y=None):
    """Commit a clean block (L == block): advances h_cache in place; returns y or None."""
    if _fast is not None:
        try:
            rc, yo = _fast.commit_block(x, dt, A, B, C, Dskip, h_cache, z, bool(dt_softplus), bool(want_y), y)
        except TypeError:
            rc = _fast.NOT_COMMON
        if rc == 0:
            return yo
        if rc != _fast.NOT_COMMON:
            raise BdscanError(rc, "bdscan_commit_block")
    block = x.shape[1]
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, block, z, dt_softplus)
    _need(h_cache, "h_cache", torch.float32, (Bt, D, N), dev)
    if y is None and want_y:
        y = torch.empty((Bt, L, D), dtype=io, device=dev)
    if y is not None:
        _need(y, "y", io, (Bt, L, D), dev)
    rc = _lib.bdscan_commit_block(ct.byref(dims), ct.byref(ins), _ptr(h_cache), _ptr(y), _stream(dev))
    _check(rc, "bdscan_commit_block")
    return y


def train_two_stream(clean, noisy, A, Dskip, block, h0=None, dt_softplus=True, want_y_clean=True,
                     y_clean=None, y_noisy=None, boundary=None, h_out=None, want_h_out=False):
    """Two-stream all-block training pass.

    clean, noisy: dicts with x, dt, B, C (and optionally z) tensors of one
    shape. Returns (y_clean or None, y_noisy, boundary, h_out or None).
    """
    dims, cin, (Bt, L, D, N), io, dev = _prepare(clean["x"], clean["dt"], A, clean["B"], clean["C"], Dskip, block,
                                                 clean.get("z"), dt_softplus)
    dims2, nin, shp2, io2, dev2 = _prepare(noisy["x"], noisy["dt"], A, noisy["B"], noisy["C"], Dskip, block,
                                           noisy.get("z"), dt_softplus)
    if (Bt, L, D, N) != shp2 or io != io2 or dev != dev2:
        raise ValueError("clean and noisy streams must have the same shapes, dtype and device")
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    if y_clean is None and want_y_clean:
        y_clean = torch.empty((Bt, L, D), dtype=io, device=dev)
    if y_clean is not None:
        _need(y_clean, "y_clean", io, (Bt, L, D), dev)
    y_noisy = torch.empty((Bt, L, D), dtype=io, device=dev) if y_noisy is None else y_noisy
    _need(y_noisy, "y_noisy", io, (Bt, L, D), dev)
    boundary = torch.empty((Bt, L // int(block), D, N), dtype=torch.float32, device=dev) if boundary is None else boundary
    _need(boundary, "boundary", torch.float32, (Bt, L // int(block), D, N), dev)
    if h_out is None and want_h_out:
        h_out = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
    if h_out is not None:
        _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    rc = _lib.bdscan_train_two_stream(ct.byref(dims), ct.byref(cin), ct.byref(nin), _ptr(h0), _ptr(y_clean),
                                      _ptr(y_noisy), _ptr(boundary), _ptr(h_out), _stream(dev))
    _check(rc, "bdscan_train_two_stream")
    return y_clean, y_noisy, boundary, h_out


def full_bidirectional(x, dt, A, B, C, Dskip, z=None, h0=None, dt_softplus=True, y=None, h_out=None,
                       want_h_out=False):
    """Forward and reverse scans over the whole sequence (no blocks): returns (y, h_out or None)."""
    L = x.shape[1]
    dims, ins, (Bt, L, D, N), io, dev = _prepare(x, dt, A, B, C, Dskip, max(L, 1), z, dt_softplus)
    if h0 is not None:
        _need(h0, "h0", torch.float32, (Bt, D, N), dev)
    y = torch.empty((Bt, L, D), dtype=io, device=dev) if y is None else y
    _need(y, "y", io, (Bt, L, D), dev)
    if h_out is None and want_h_out:
        h_out = torch.empty((Bt, D, N), dtype=torch.float32, device=dev)
    if h_out is not None:
        _need(h_out, "h_out", torch.float32, (Bt, D, N), dev)
    rc = _lib.bdscan_full_bidirectional(ct.byref(dims), ct.byref(ins), _ptr(h0), _ptr(y), _ptr(h_out), _stream(dev))
    _check(rc, "bdscan_full_bidirectional")
    return y, h_out


def raw_library():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib

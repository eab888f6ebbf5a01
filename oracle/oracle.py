"""ctypes front end of the C oracle (``bdscan_oracle.c``).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). Inputs are numpy arrays
in their storage type: ``uint16`` bf16 bit patterns or ``float32``. They are
widened exactly to float64 here and every result comes back as float64.
"""
from __future__ import annotations

import ctypes as C
import numpy as np

from . import build as _build

_LIBS: dict = {}
_dp = C.POINTER(C.c_double)
_i64 = C.c_int64


def load(mutant: int = 0):
    """Load (building first if needed) the oracle library, optionally a planted-mistake build."""
    if mutant not in _LIBS:
        lib = C.CDLL(_build.build(mutant))
        lib.oracle_forward.argtypes = [_i64] * 5 + [_dp, _dp, C.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_forward.restype = C.c_int
        lib.oracle_reverse_blocks.argtypes = [_i64] * 5 + [_dp, _dp, C.c_int, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_reverse_blocks.restype = C.c_int
        lib.oracle_combine.argtypes = [_i64, _dp, _dp, _dp, _dp]
        lib.oracle_combine.restype = None
        lib.oracle_bruteforce.argtypes = [_i64] * 5 + [_dp, _dp, C.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_bruteforce.restype = C.c_int
        lib.oracle_train_blocks_backward.argtypes = ([_i64] * 5 + [_dp, _dp, C.c_int] + [_dp] * 7
                                                     + [_dp] * 8)
        lib.oracle_train_blocks_backward.restype = C.c_int
        lib.oracle_softplus.argtypes = [C.c_double]
        lib.oracle_softplus.restype = C.c_double
        lib.oracle_mutant_id.restype = C.c_int
        _LIBS[mutant] = lib
    return _LIBS[mutant]


def decode(a) -> np.ndarray:
    """Exact widening to float64: uint16 arrays are bf16 bit patterns."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _dims(x, B):
    Bt, L, D = x.shape
    N = B.shape[-1]
    return Bt, L, D, N


def softplus(v: float, mutant: int = 0) -> float:
    return load(mutant).oracle_softplus(float(v))


def forward(x, dt, A, B, C_, Dskip, K, h0=None, dt_softplus=True, want_boundary=True, mutant=0):
    """Causal scan. Returns dict(y_fwd [Bt,L,D], h_out [Bt,D,N], boundary [Bt,L/K,D,N] or None)."""
    x, dt, A, B, C_, Dskip, h0 = map(decode, (x, dt, A, B, C_, Dskip, h0))
    Bt, L, D, N = _dims(x, B)
    y = np.zeros((Bt, L, D))
    h_out = np.zeros((Bt, D, N))
    bnd = np.zeros((Bt, L // K, D, N)) if want_boundary else None
    rc = load(mutant).oracle_forward(Bt, L, D, N, K, _p(x), _p(dt), int(dt_softplus), _p(A), _p(B), _p(C_),
                                     _p(Dskip), _p(h0), _p(y), _p(h_out), _p(bnd))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments")
    return {"y_fwd": y, "h_out": h_out, "boundary": bnd}


def reverse_blocks(x, dt, A, B, C_, Dskip, K, dt_softplus=True, mutant=0):
    """Block-confined reverse scan output y_rev [Bt, L, D] (includes Dskip*x)."""
    x, dt, A, B, C_, Dskip = map(decode, (x, dt, A, B, C_, Dskip))
    Bt, L, D, N = _dims(x, B)
    y = np.zeros((Bt, L, D))
    rc = load(mutant).oracle_reverse_blocks(Bt, L, D, N, K, _p(x), _p(dt), int(dt_softplus), _p(A), _p(B),
                                            _p(C_), _p(Dskip), _p(y))
    if rc != 0:
        raise ValueError("oracle_reverse_blocks rejected its arguments")
    return y


def _combine(y_fwd, y_rev, z, mutant=0):
    z = decode(z)
    out = np.zeros_like(y_fwd)
    load(mutant).oracle_combine(y_fwd.size, _p(y_fwd), _p(y_rev), _p(z), _p(out))
    return out


def train_blocks(x, dt, A, B, C_, Dskip, K, z=None, h0=None, dt_softplus=True, mutant=0):
    """All blocks at once: y = (y_fwd + y_rev) * gate, plus boundary and final states."""
    f = forward(x, dt, A, B, C_, Dskip, K, h0=h0, dt_softplus=dt_softplus, mutant=mutant)
    r = reverse_blocks(x, dt, A, B, C_, Dskip, K, dt_softplus=dt_softplus, mutant=mutant)
    return {"y": _combine(f["y_fwd"], r, z, mutant), "boundary": f["boundary"], "h_out": f["h_out"]}


def prefill(x, dt, A, B, C_, Dskip, K, z=None, h0=None, dt_softplus=True, mutant=0):
    """Forward-only scan of a clean context: y = y_fwd * gate, final and boundary states."""
    f = forward(x, dt, A, B, C_, Dskip, K, h0=h0, dt_softplus=dt_softplus, mutant=mutant)
    return {"y": _combine(f["y_fwd"], None, z, mutant), "boundary": f["boundary"], "h_out": f["h_out"]}


def block_step(x, dt, A, B, C_, Dskip, h_cache, z=None, dt_softplus=True, mutant=0):
    """One denoising step on the active block (L == K): forward from the cache plus in-block reverse."""
    K = np.asarray(x).shape[1]
    return train_blocks(x, dt, A, B, C_, Dskip, K, z=z, h0=h_cache, dt_softplus=dt_softplus, mutant=mutant)["y"]


def commit_block(x, dt, A, B, C_, Dskip, h_cache, z=None, dt_softplus=True, mutant=0):
    """Commit a clean block: returns (new cache state, y as block_step would give on the clean block)."""
    K = np.asarray(x).shape[1]
    r = train_blocks(x, dt, A, B, C_, Dskip, K, z=z, h0=h_cache, dt_softplus=dt_softplus, mutant=mutant)
    return r["h_out"], r["y"]


def bruteforce(x, dt, A, B, C_, Dskip, K, z=None, h0=None, dt_softplus=True, mutant=0):
    """Closed-form matrix evaluation (long double) for L <= 64: returns dict(y, boundary)."""
    x, dt, A, B, C_, Dskip, z, h0 = map(decode, (x, dt, A, B, C_, Dskip, z, h0))
    Bt, L, D, N = _dims(x, B)
    y = np.zeros((Bt, L, D))
    bnd = np.zeros((Bt, L // K, D, N))
    rc = load(mutant).oracle_bruteforce(Bt, L, D, N, K, _p(x), _p(dt), int(dt_softplus), _p(A), _p(B), _p(C_),
                                        _p(Dskip), _p(z), _p(h0), _p(y), _p(bnd))
    if rc != 0:
        raise ValueError("oracle_bruteforce rejected its arguments")
    return {"y": y, "boundary": bnd}


def two_stream(clean, noisy, A, Dskip, K, h0=None, z_noisy=None, dt_softplus=True, mutant=0):
    """All-block training with separate clean and noisy streams.

    clean / noisy: dicts with x, dt, B, C ([Bt, L, ...] each). The clean stream
    is scanned forward only (the prefix operator): its outputs y_clean and the
    state after every block, the caches. Noisy block j resumes the forward scan
    from the clean cache at its start (h0 for j = 0) and adds its block-confined
    reverse scan: y_noisy = (y_fwd + y_rev) * gate. Returns dict(y_clean,
    y_noisy, boundary, h_out).
    """
    f = forward(clean["x"], clean["dt"], A, clean["B"], clean["C"], Dskip, K, h0=h0,
                dt_softplus=dt_softplus, mutant=mutant)
    Bt, L = np.asarray(noisy["x"]).shape[:2]
    D = np.asarray(noisy["x"]).shape[2]
    N = np.asarray(noisy["B"]).shape[2]
    y_noisy = np.zeros((Bt, L, D))
    for j in range(L // K):
        sl = slice(j * K, (j + 1) * K)
        hj = (np.zeros((Bt, D, N)) if h0 is None else decode(h0)) if j == 0 else f["boundary"][:, j - 1]
        blk = {k: np.ascontiguousarray(np.asarray(noisy[k])[:, sl]) for k in ("x", "dt", "B", "C")}
        zj = None if z_noisy is None else np.ascontiguousarray(np.asarray(z_noisy)[:, sl])
        y_noisy[:, sl] = block_step(blk["x"], blk["dt"], A, blk["B"], blk["C"], Dskip, hj, z=zj,
                                    dt_softplus=dt_softplus, mutant=mutant)
    return {"y_clean": _combine(f["y_fwd"], None, None, mutant), "y_noisy": y_noisy,
            "boundary": f["boundary"], "h_out": f["h_out"]}


def train_blocks_backward(x, dt, A, B, C_, Dskip, K, dy, z=None, h0=None, dt_softplus=True, mutant=0):
    """Gradients of train_blocks' y with respect to every input, given dy.

    Returns dict(dx, ddt, dz (None without z), dB, dC, dA, dDskip, dh0), all float64.
    """
    x, dt, A, B, C_, Dskip, z, h0, dy = map(decode, (x, dt, A, B, C_, Dskip, z, h0, dy))
    Bt, L, D, N = _dims(x, B)
    out = {"dx": np.zeros((Bt, L, D)), "ddt": np.zeros((Bt, L, D)),
           "dz": np.zeros((Bt, L, D)) if z is not None else None,
           "dB": np.zeros((Bt, L, N)), "dC": np.zeros((Bt, L, N)), "dA": np.zeros((D, N)),
           "dDskip": np.zeros(D), "dh0": np.zeros((Bt, D, N))}
    rc = load(mutant).oracle_train_blocks_backward(
        Bt, L, D, N, K, _p(x), _p(dt), int(dt_softplus), _p(A), _p(B), _p(C_), _p(Dskip), _p(z), _p(h0), _p(dy),
        *[_p(out[k]) for k in ("dx", "ddt", "dz", "dB", "dC", "dA", "dDskip", "dh0")])
    if rc != 0:
        raise ValueError("oracle_train_blocks_backward rejected its arguments")
    return out

"""C-ABI library: loads, exports what the header declares, and rejects bad
arguments before touching the GPU (runs without a GPU)."""
import ctypes as C
import os
import re

import pytest

from selective_ssm_scan_mamba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    return C.CDLL(B.build())


def declared_functions():
    names = []
    for h in sorted(os.listdir(HEADER_DIR)):
        if h.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(bdscan_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_four_operations():
    names = declared_functions()
    for op in ("bdscan_train_blocks", "bdscan_prefill", "bdscan_block_step", "bdscan_commit_block"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


class Dims(C.Structure):
    _fields_ = [("batch", C.c_int64), ("seqlen", C.c_int64), ("d_inner", C.c_int64),
                ("d_state", C.c_int64), ("block", C.c_int64), ("io_dtype", C.c_int32),
                ("dt_softplus", C.c_int32)]


class Inputs(C.Structure):
    _fields_ = [("x", C.c_void_p), ("dt", C.c_void_p), ("B", C.c_void_p), ("C", C.c_void_p),
                ("z", C.c_void_p), ("A", C.c_void_p), ("Dskip", C.c_void_p)]


# fake, never dereferenced: every call below fails validation before any launch
P = 0x100000


def _ins(**kw):
    d = dict(x=P, dt=P + 0x100, B=P + 0x200, C=P + 0x300, z=None, A=P + 0x400, Dskip=P + 0x500)
    d.update(kw)
    return Inputs(**d)


def _train(lib, dims, ins, y=P + 0x600):
    lib.bdscan_train_blocks.argtypes = [C.POINTER(Dims), C.POINTER(Inputs)] + [C.c_void_p] * 5
    return lib.bdscan_train_blocks(C.byref(dims) if dims else None, C.byref(ins) if ins else None,
                                   None, y, None, None, None)


@pytest.mark.parametrize("dims,ins,want", [
    (None, _ins(), 1),
    (Dims(2, 64, 64, 32, 16, 1, 1), _ins(), 2),            # N unsupported
    (Dims(2, 60, 64, 16, 16, 1, 1), _ins(), 1),            # L % K != 0
    (Dims(2, 64, 60, 16, 16, 1, 1), _ins(), 2),            # bf16 needs D % 8 == 0
    (Dims(2, 64, 62, 16, 16, 0, 1), _ins(), 2),            # fp32 needs D % 4 == 0
    (Dims(2, 64, 64, 16, 0, 1, 1), _ins(), 1),             # K < 1
    (Dims(2, 64, 64, 16, 16, 7, 1), _ins(), 1),            # bad dtype
    (Dims(-1, 64, 64, 16, 16, 1, 1), _ins(), 1),           # negative batch
    (Dims(2, 64, 64, 16, 16, 1, 1), _ins(x=None), 1),      # missing x
    (Dims(2, 64, 64, 16, 16, 1, 1), _ins(B=P + 8), 3),     # misaligned B
    (Dims(2, 4096, 64, 16, 4096, 1, 1), _ins(), 2),        # block too long for the long-block path
])
def test_train_blocks_rejects(lib, dims, ins, want):
    assert _train(lib, dims, ins) == want


def test_train_blocks_requires_y(lib):
    assert _train(lib, Dims(2, 64, 64, 16, 16, 1, 1), _ins(), y=None) == 1


def test_step_and_commit_require_one_block(lib):
    lib.bdscan_block_step.argtypes = [C.POINTER(Dims), C.POINTER(Inputs)] + [C.c_void_p] * 3
    lib.bdscan_commit_block.argtypes = [C.POINTER(Dims), C.POINTER(Inputs)] + [C.c_void_p] * 3
    d = Dims(2, 64, 64, 16, 32, 1, 1)   # L != K
    assert lib.bdscan_block_step(C.byref(d), C.byref(_ins()), P + 0x700, P + 0x800, None) == 1
    assert lib.bdscan_commit_block(C.byref(d), C.byref(_ins()), P + 0x700, None, None) == 1
    d = Dims(2, 32, 64, 16, 32, 1, 1)
    assert lib.bdscan_block_step(C.byref(d), C.byref(_ins()), None, P + 0x800, None) == 1   # no cache
    assert lib.bdscan_commit_block(C.byref(d), C.byref(_ins()), None, None, None) == 1


def test_prefill_requires_final_state(lib):
    lib.bdscan_prefill.argtypes = [C.POINTER(Dims), C.POINTER(Inputs)] + [C.c_void_p] * 5
    d = Dims(2, 64, 64, 16, 16, 1, 1)
    assert lib.bdscan_prefill(C.byref(d), C.byref(_ins()), None, None, None, None, None) == 1


def test_status_strings(lib):
    lib.bdscan_status_string.restype = C.c_char_p
    assert lib.bdscan_status_string(0) == b"BDSCAN_OK"
    assert lib.bdscan_status_string(3) == b"BDSCAN_ERR_ALIGNMENT"
    assert lib.bdscan_status_string(99) == b"BDSCAN_UNKNOWN_STATUS"
    assert lib.bdscan_version() >= 100

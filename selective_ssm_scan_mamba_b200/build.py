"""Build ``_lib/libbdscan.so`` in-tree with nvcc for sm_100a only, and the
compiled per-step marshalling module ``_lib/_bdscan_fast`` beside it.

Run ``python -m selective_ssm_scan_mamba_b200.build`` (or ``__graft_entry__.build()``).
The CUDA runtime is linked statically so the library does not depend on the
runtime version that PyTorch ships. The marshalling module is a PyTorch C++
extension (host code only) linked against libbdscan.so through its own
directory; it calls the same C-ABI entry points as the ctypes binding.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
import sysconfig

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIBDIR = os.path.join(HERE, "_lib")
LIB = os.path.join(LIBDIR, "libbdscan.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


FAST_SRC = os.path.join(CSRC, "bdscan_fastpath.cpp")
FAST = os.path.join(LIBDIR, "_bdscan_fast" + sysconfig.get_config_var("EXT_SUFFIX"))
CXX = os.environ.get("CXX", "g++")


def build_fastpath(force: bool = False) -> str:
    """Compile the per-step marshalling module (needs libbdscan.so first)."""
    deps = [FAST_SRC, LIB, os.path.join(ROOT, "include", "bdscan.h")]
    if not force and os.path.exists(FAST) and os.path.getmtime(FAST) >= max(os.path.getmtime(p) for p in deps):
        return FAST
    import torch
    from torch.utils import cpp_extension as ce
    incs = ce.include_paths("cuda") + [sysconfig.get_paths()["include"], os.path.join(ROOT, "include")]
    libdirs = ce.library_paths("cuda")
    tmp = FAST + f".tmp{os.getpid()}"
    cmd = [CXX, "-O2", "-std=c++17", "-fPIC", "-shared", "-DTORCH_EXTENSION_NAME=_bdscan_fast",
           "-DTORCH_API_INCLUDE_EXTENSION_H", f"-D_GLIBCXX_USE_CXX11_ABI={int(torch._C._GLIBCXX_USE_CXX11_ABI)}",
           *[f"-I{p}" for p in incs], FAST_SRC, "-o", tmp, *[f"-L{p}" for p in libdirs],
           "-lc10", "-lc10_cuda", "-ltorch", "-ltorch_cpu", "-ltorch_python",
           f"-L{LIBDIR}", "-lbdscan", "-Wl,-rpath,$ORIGIN"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, FAST)
    return FAST


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        os.makedirs(LIBDIR, exist_ok=True)
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *sources()]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    build_fastpath(force)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))

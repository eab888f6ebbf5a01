"""Seeded synthetic inputs for the block-confined bidirectional selective scan.

This module is the one piece shared by the CUDA path's tests/bench and the CPU
oracle: it only draws random numbers and rounds them to the storage dtype. It
holds none of the scan's arithmetic.

Workloads follow the five configurations of the block-diffusion Mamba-H mixer
workloads (value distributions of the mixer inputs):

* ``x ~ N(0, 1)``                    ``[batch, L, D]``   (io dtype)
* ``dt_raw ~ N(-2, 0.5)``            ``[batch, L, D]``   (io dtype; the kernel
  applies ``softplus`` itself, so the stored operand is the raw value)
* ``A = -exp(U(log 1, log 16))``     ``[D, N]``          fp32
* ``B, C ~ N(0, 1) / sqrt(N)``       ``[batch, L, N]``   (io dtype)
* ``Dskip ~ N(0, 1)``                ``[D]``             fp32
* ``z ~ N(0, 1)``                    ``[batch, L, D]``   (optional gate)

Random streams are keyed, not sequential: every (array, stream, batch row,
4096-token chunk) draws from its own ``PCG64(SeedSequence([seed, ...key]))``.
Any token range of any batch row is therefore reproducible on its own, which
lets a test regenerate a slice of a 262,144-token context without holding the
whole context in host memory, and lets the oracle see exactly the values the
GPU saw. bf16 values are produced by round-to-nearest-even from the fp32 draw
and returned as their raw ``uint16`` bit patterns.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 4096  # tokens per independently seeded chunk

_ARRAY_IDS = {"x": 1, "dt": 2, "B": 3, "C": 4, "z": 5, "A": 6, "Dskip": 7}
# streams name independent sequences inside one workload
_STREAM_IDS = {"seq": 0, "context": 1, "noisy": 2, "clean": 3, "layer": 4}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 to bf16 (round to nearest, ties to even); returns uint16 bits.

    The 32-bit sum cannot wrap for finite inputs: the largest finite pattern
    0xFF7FFFFF plus 0x8000 stays below 2**32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= 16
    return r.astype(np.uint16)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, key)])))


def _stream_key(stream) -> tuple:
    if isinstance(stream, str):
        stream = (stream,)
    name, *rest = stream
    return (_STREAM_IDS[name], *[int(r) for r in rest])


def _draw_chunk(seed, array, stream, b, c, width, mean, std):
    g = _rng(seed, _ARRAY_IDS[array], *_stream_key(stream), b, c)
    blk = g.standard_normal((CHUNK, width), dtype=np.float32)
    if std != 1.0:
        blk *= np.float32(std)
    if mean != 0.0:
        blk += np.float32(mean)
    return blk


def _chunk_range(t0, t1):
    return range(t0 // CHUNK, (t1 - 1) // CHUNK + 1) if t1 > t0 else range(0)


def _cast(a32: np.ndarray, io: str) -> np.ndarray:
    if io == "bf16":
        return f32_to_bf16_bits(a32)
    if io == "f32":
        return np.ascontiguousarray(a32, dtype=np.float32)
    raise ValueError(f"io dtype {io!r}")


def make_sequence(seed: int, batch: int, L: int, D: int, N: int, io: str,
                  stream="seq", t0: int = 0, gated: bool = False,
                  channels=None) -> dict:
    """Per-token inputs x, dt, B, C (and z) for tokens [t0, t0+L) of `stream`.

    ``channels`` optionally restricts x/dt/z to a subset of channel indices
    (B and C are shared by all channels and always returned whole).
    """
    t1 = t0 + L
    specs = [("x", D, 0.0, 1.0), ("dt", D, -2.0, 0.5), ("B", N, 0.0, 1.0 / np.sqrt(N)),
             ("C", N, 0.0, 1.0 / np.sqrt(N))] + ([("z", D, 0.0, 1.0)] if gated else [])
    store = np.uint16 if io == "bf16" else np.float32
    res = {}
    for name, width, _, _ in specs:
        w_out = len(channels) if (channels is not None and name in ("x", "dt", "z")) else width
        res[name] = np.empty((batch, L, w_out), dtype=store)

    def job(name, width, mean, std, b, c):
        blk = _draw_chunk(seed, name, stream, b, c, width, mean, std)
        lo, hi = max(t0, c * CHUNK), min(t1, (c + 1) * CHUNK)
        part = blk[lo - c * CHUNK:hi - c * CHUNK]
        if channels is not None and name in ("x", "dt", "z"):
            part = part[:, channels]
        res[name][b, lo - t0:hi - t0] = _cast(part, io)

    jobs = [(name, width, mean, std, b, c) for name, width, mean, std in specs
            for b in range(batch) for c in _chunk_range(t0, t1)]
    if len(jobs) > 2 and batch * L * D >= (1 << 22):
        with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
            list(ex.map(lambda j: job(*j), jobs))
    else:
        for j in jobs:
            job(*j)
    return res


def make_params(seed: int, D: int, N: int, layer: int = 0) -> dict:
    """Per-channel parameters: A [D, N] fp32 (negative) and Dskip [D] fp32."""
    g = _rng(seed, _ARRAY_IDS["A"], _STREAM_IDS["layer"], layer)
    u = g.uniform(np.log(1.0), np.log(16.0), size=(D, N))
    A = (-np.exp(u)).astype(np.float32)
    g = _rng(seed, _ARRAY_IDS["Dskip"], _STREAM_IDS["layer"], layer)
    Dskip = g.standard_normal(D).astype(np.float32)
    return {"A": np.ascontiguousarray(A), "Dskip": np.ascontiguousarray(Dskip)}


def make_state(seed: int, batch: int, D: int, N: int, scale: float = 1.0) -> np.ndarray:
    """A generic fp32 initial state [batch, D, N] ~ N(0, scale^2) for tests."""
    g = _rng(seed, 99, batch, D, N)
    return (g.standard_normal((batch, D, N)) * scale).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One of the five mixer workloads (sizes, block length, dtype, seed)."""
    name: str
    batch: int
    L: int            # tokens scanned by the main call (train / prefill)
    D: int
    N: int
    K: int            # block length
    io: str
    seed: int
    steps: int = 0    # denoising steps per block (inference workloads)
    blocks: int = 0   # committed blocks (inference workloads)
    layers: int = 1
    note: str = ""


WORKLOADS = {
    "pr1": Workload("pr1", batch=1, L=256, D=64, N=16, K=16, io="f32", seed=0,
                    note="one mixer, 16 block-boundary states, fp32"),
    "train": Workload("train", batch=8, L=4096, D=1536, N=16, K=16, io="bf16", seed=1,
                      note="full-block training objective, all blocks in one launch"),
    "step65k": Workload("step65k", batch=1, L=65536, D=1536, N=16, K=32, io="bf16", seed=2,
                        steps=32, blocks=1, note="block step at a 65,536-token context"),
    "step262k": Workload("step262k", batch=4, L=262144, D=2048, N=16, K=32, io="bf16", seed=3,
                         steps=64, blocks=8, note="block steps at a 262,144-token context"),
    "stack350m": Workload("stack350m", batch=16, L=8192, D=2048, N=64, K=16, io="bf16", seed=4,
                          layers=24, note="24 mixer layers, block sizes {4,16,64,256}"),
}
STACK_BLOCK_SIZES = (4, 16, 64, 256)

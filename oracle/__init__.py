"""CPU oracle for the block-confined bidirectional selective scan.

TEST INFRASTRUCTURE ONLY: a plain, sequential fp64 C restatement of what the
mixer computes, used to check the CUDA path. Only ``tests/``, the package's
``smoke()`` check and ``bench.py``'s CPU-baseline / reference legs may import
it. It shares no code with the CUDA path and the CUDA path never calls it.

Parity status: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (hand-derived example, closed forms, brute-force
matrix form, invariants, planted-mistake checks); the backward pass by
central differences of the pinned forward, the closed-form matrix in x and
the Euler identities of y's homogeneities.
"""
from .oracle import (  # noqa: F401
    decode, forward, reverse_blocks, train_blocks, prefill, block_step,
    commit_block, bruteforce, softplus, load, two_stream, train_blocks_backward,
)

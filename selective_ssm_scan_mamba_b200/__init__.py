"""B200-native block-confined bidirectional selective scan (BDLM Mamba-H mixer).

``inputs``            seeded synthetic workloads (numpy only)
``bdscan``            Python binding of the C-ABI library ``libbdscan.so`` (CUDA, sm_100a):
                      training pass and its backward, prefill (sequential, time-chunked,
                      allocation-free), block step, commit, two-stream training, the
                      full-sequence comparator, chunk summaries for context parallelism
``context_parallel``  prefill of one context split over the ranks of a process group
``build``             compiles ``libbdscan.so`` in-tree

Import the submodules explicitly, e.g. ``from selective_ssm_scan_mamba_b200 import bdscan``.
"""

"""B200-native block-confined bidirectional selective scan (BDLM Mamba-H mixer).

``inputs``  seeded synthetic workloads (numpy only)
``bdscan``  Python binding of the C-ABI library ``libbdscan.so`` (CUDA, sm_100a)
"""
__all__ = ["inputs", "bdscan"]


def __getattr__(name):
    if name == "bdscan":
        from . import bdscan as _b
        return _b
    raise AttributeError(name)

"""B200-native block-confined bidirectional selective scan (BDLM Mamba-H mixer).

``inputs``  seeded synthetic workloads (numpy only)
``bdscan``  Python binding of the C-ABI library ``libbdscan.so`` (CUDA, sm_100a);
            import it explicitly: ``from selective_ssm_scan_mamba_b200 import bdscan``
"""

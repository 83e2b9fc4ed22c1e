"""LongCat Sparse Attention (LSA) hot path for B200 (sm_100a).

The compute lives in liblsa.so (C-ABI, include/lsa.h); `lsa` is its Python
binding and `device_inputs` draws the synthetic workloads on the device.
"""

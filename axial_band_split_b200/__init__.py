"""Mel-Band RoFormer core forward on NVIDIA B200 (sm_100a), behind the C ABI of libmrf.

The package holds the CUDA sources (csrc/), their build script (build.py), the ctypes
binding (mrf.py) and the FLOP/byte accounting used for roofline reports (accounting.py).
"""

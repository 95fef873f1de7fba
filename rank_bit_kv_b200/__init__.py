"""kvc: compressed-KV single-token decode attention for B200 (sm_100a).

The CUDA library (``libkvc.so``, C ABI declared in ``include/kvc.h``) is loaded
lazily on first use by :mod:`rank_bit_kv_b200.kvc`; importing the package or
its ``synth`` module does not touch the GPU.
"""

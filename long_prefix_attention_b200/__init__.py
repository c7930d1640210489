"""Attention State Memory (ASM) hot path for NVIDIA B200 (sm_100a).

The compute lives in ``libasm_b200.so`` (CUDA kernels behind the C ABI of
``include/asm.h``); :mod:`long_prefix_attention_b200.ops` is its Python
binding and :mod:`long_prefix_attention_b200.inputs` draws the seeded
synthetic workloads.  Importing the package loads nothing; the library is
loaded on the first call.
"""
__all__ = ["ops", "inputs", "build"]

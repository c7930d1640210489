"""ctypes loader for ``libasm_b200.so`` (the C ABI of include/asm.h).

Loading fails loudly when the library has not been built: there is no other
implementation of these calls in this package.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libasm_b200.so")

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/asm.h
SIGNATURES = {
    "asm_build_states": (I, [P, P, P, I, I, I, I, I, F, I, I, P, P, P]),
    "asm_merge_states": (I, [P, P, P, P, ctypes.c_int64, I, I, P]),
    "asm_kmeanspp_workspace_size": (SZ, [I, I, I, I]),
    "asm_kmeanspp_seed": (I, [P, I, I, I, I, P, I, P, P, SZ, P]),
    "asm_kmeanspp_batched_workspace_size": (SZ, [I, I, I, I, I]),
    "asm_kmeanspp_seed_batched": (I, [P, I, I, I, I, I, P, I, I, P, P, SZ, P]),
    "asm_kmeans_assign": (I, [P, P, I, I, I, I, I, I, P, P, SZ, P]),
    "asm_kmeans_update": (I, [P, P, I, I, I, I, I, P, P, P, P, P, P, SZ, P]),
    "asm_kmeans_workspace_size": (SZ, [I, I, I, I]),
    "asm_kmeans": (I, [P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P]),
    "asm_aggregate": (I, [P, P, P, P, I, I, I, I, I, I, P, P, P]),
    "asm_decode_workspace_size": (SZ, [I, I, I, I, I, I, I]),
    "asm_decode_step": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P, P, ctypes.c_uint, P, SZ, P]),
    "asm_decode_step_launches": (I, [I, I, I, I, I, I, I]),
    "asm_decode_step_noalloc": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P, P, ctypes.c_uint, P]),
    "asm_decode_noalloc_error": (I, [ctypes.POINTER(ctypes.c_int), P]),
    "asm_flash_decode_workspace_size": (SZ, [I, I, I, I, I, I, I]),
    "asm_flash_decode": (I, [P, P, P, I, P, P, P, I, I, I, I, I, F, I, P, P, P, SZ, P]),
    "asm_index_reorder": (I, [P, I, I, I, I, P, P, P, P, P, P, P]),
    "asm_decode_indexed_workspace_size": (SZ, [I, I, I, I, I, I, I, I, I]),
    "asm_decode_step_indexed": (I, [P, P, P, I, I, I, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P, P, P,
                                    SZ, P]),
    "asm_whitening_workspace_size": (SZ, [I, I]),
    "asm_whitening": (I, [P, I, I, I, I, F, P, P, P, SZ, P]),
    "asm_whiten": (I, [P, I, I, I, I, ctypes.c_int64, ctypes.c_int64, P, P, P, ctypes.c_int64, ctypes.c_int64, P]),
    "asm_decode_step_search": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P, P, ctypes.c_uint, P,
                                   SZ, P]),
    "asm_workspace_init": (I, [P, SZ, P]),
    "asm_workspace_error": (I, [P, SZ, ctypes.POINTER(ctypes.c_int), P]),
    "asm_wait_spin_limit": (ctypes.c_uint32, []),
    "asm_wait_selftest": (I, [I, P, SZ, ctypes.POINTER(ctypes.c_uint64), P]),
    "asm_status_string": (ctypes.c_char_p, [I]),
    "asm_last_cuda_error": (ctypes.c_char_p, []),
    "asm_version": (ctypes.c_char_p, []),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m long_prefix_attention_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib

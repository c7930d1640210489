"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/asm.h declares, and rejects invalid arguments with
the documented status before any CUDA call is made."""
import ctypes
import os
import re

import pytest

from long_prefix_attention_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "asm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(asm_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ["asm_build_states", "asm_kmeanspp_seed", "asm_kmeans", "asm_kmeans_assign",
              "asm_kmeans_update", "asm_aggregate", "asm_decode_step", "asm_flash_decode",
              "asm_decode_workspace_size", "asm_workspace_init", "asm_status_string"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    for s in range(6):
        assert lib.asm_status_string(s)
    assert lib.asm_version().decode().count(".") == 2
    # no CUDA call has failed on this thread
    assert lib.asm_last_cuda_error().decode() == "no error"


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p(0x10008)       # 8-byte aligned only
NULL = None


def decode(lib, **kw):
    a = dict(q=FAKE, c=FAKE, ab=FAKE, lz=FAKE, kc=FAKE, vc=FAKE, ll=FAKE, B=1, Hq=32, Hkv=8,
             K=1024, Tmax=2048, d=128, scale=0.088, metric=0, dt=1, out=FAKE, lse=NULL, idx=NULL,
             flags=0, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.asm_decode_step(a["q"], a["c"], a["ab"], a["lz"], a["kc"], a["vc"], a["ll"], a["B"],
                               a["Hq"], a["Hkv"], a["K"], a["Tmax"], a["d"], a["scale"],
                               a["metric"], a["dt"], a["out"], a["lse"], a["idx"], a["flags"],
                               a["ws"], a["wsb"], None)


def test_decode_validation(lib):
    assert decode(lib, d=96) == UNSUPPORTED
    assert decode(lib, Hq=32, Hkv=5) == INVALID
    assert decode(lib, Hq=48, Hkv=3) == UNSUPPORTED    # group of 16
    assert decode(lib, q=NULL) == INVALID
    assert decode(lib, c=ODD) == INVALID
    assert decode(lib, K=0) == INVALID
    assert decode(lib, B=0) == INVALID
    assert decode(lib, metric=7) == INVALID
    assert decode(lib, dt=3) == INVALID
    assert decode(lib, wsb=16) == WORKSPACE
    assert decode(lib, ws=NULL) == WORKSPACE
    assert decode(lib, scale=float("nan")) == INVALID
    assert decode(lib, flags=6) == INVALID


def test_workspace_sizes_grow_with_the_problem(lib):
    s1 = lib.asm_decode_workspace_size(1, 32, 8, 1024, 2048, 128, 1)
    s2 = lib.asm_decode_workspace_size(16, 32, 8, 8192, 4096, 128, 1)
    assert 0 < s1 < s2 and s1 % 256 == 0
    assert lib.asm_decode_workspace_size(0, 32, 8, 1024, 2048, 128, 1) == 0
    assert lib.asm_flash_decode_workspace_size(1, 32, 8, 32768, 2048, 128, 1) > 0
    assert lib.asm_kmeans_workspace_size(32, 65536, 128, 8192) > 0
    assert lib.asm_kmeanspp_workspace_size(32, 65536, 128, 8192) > 0
    assert 0 < lib.asm_kmeanspp_batched_workspace_size(2, 4096, 128, 256, 32) < \
        lib.asm_kmeanspp_batched_workspace_size(32, 65536, 128, 8192, 128)


def test_build_and_kmeans_validation(lib):
    P = FAKE
    # build states: bad group / d
    assert lib.asm_build_states(P, P, P, 32, 6, 16, 16, 128, 0.1, 1, 0, P, P, None) == INVALID
    assert lib.asm_build_states(P, P, P, 32, 8, 16, 16, 80, 0.1, 1, 0, P, P, None) == UNSUPPORTED
    assert lib.asm_build_states(P, P, P, 32, 8, 0, 16, 128, 0.1, 1, 0, P, P, None) == 0  # N=0: no-op
    # k-means++: K > N, small workspace
    assert lib.asm_kmeanspp_seed(P, 2, 10, 64, 11, P, 0, P, P, 1 << 30, None) == INVALID
    assert lib.asm_kmeanspp_seed(P, 2, 10, 64, 4, P, 0, P, P, 8, None) == WORKSPACE
    # batched k-means++: batch 0 or above 256, no draws, K > N, N above 2^21, small workspace
    sb = lib.asm_kmeanspp_batched_workspace_size(2, 10, 64, 4, 2)
    assert sb > 0 and lib.asm_kmeanspp_batched_workspace_size(2, 10, 64, 4, 0) == 0
    assert lib.asm_kmeanspp_batched_workspace_size(2, 10, 64, 4, 257) == 0
    assert lib.asm_kmeanspp_seed_batched(P, 2, 10, 64, 4, 0, P, 8, 0, P, P, 1 << 30, None) == INVALID
    assert lib.asm_kmeanspp_seed_batched(P, 2, 10, 64, 4, 257, P, 8, 0, P, P, 1 << 30, None) == UNSUPPORTED
    assert lib.asm_kmeanspp_seed_batched(P, 2, 10, 64, 4, 2, P, 0, 0, P, P, 1 << 30, None) == INVALID
    assert lib.asm_kmeanspp_seed_batched(P, 2, 10, 64, 11, 2, P, 8, 0, P, P, 1 << 30, None) == INVALID
    assert lib.asm_kmeanspp_seed_batched(P, 1, (1 << 21) + 1, 64, 4, 2, P, 8, 0, P, P, 1 << 40,
                                         None) == UNSUPPORTED
    assert lib.asm_kmeanspp_seed_batched(P, 2, 10, 64, 4, 2, P, 8, 0, P, P, sb - 1, None) == WORKSPACE
    # k-means: iters < 1, bad metric
    assert lib.asm_kmeans(P, 2, 10, 64, 4, 0, 0, 0, P, P, P, P, P, P, P, P, 1 << 30, None) == INVALID
    assert lib.asm_kmeans(P, 2, 10, 64, 4, 3, 5, 0, P, P, P, P, P, P, P, P, 1 << 30, None) == INVALID
    # aggregate: bad z mode
    assert lib.asm_aggregate(P, P, P, P, 2, 10, 64, 4, 9, 0, P, P, None) == INVALID
    # flash decode: nothing to attend
    assert lib.asm_flash_decode(P, P, P, 0, P, P, P, 1, 32, 8, 0, 128, 0.1, 1, P, NULL, P,
                                1 << 30, None) == INVALID


def indexed(lib, **kw):
    a = dict(q=FAKE, s=FAKE, so=FAKE, K1=64, P=8, ms=40, c=FAKE, ab=FAKE, lz=FAKE, kc=FAKE, vc=FAKE, ll=FAKE, B=1,
             Hq=32, Hkv=8, K=2048, Tmax=256, d=128, scale=0.088, metric=0, dt=1, out=FAKE, lse=NULL, idx=NULL,
             ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.asm_decode_step_indexed(a["q"], a["s"], a["so"], a["K1"], a["P"], a["ms"], a["c"], a["ab"], a["lz"],
                                       a["kc"], a["vc"], a["ll"], a["B"], a["Hq"], a["Hkv"], a["K"], a["Tmax"], a["d"],
                                       a["scale"], a["metric"], a["dt"], a["out"], a["lse"], a["idx"], a["ws"],
                                       a["wsb"], None)


def test_indexed_decode_rejects_bad_arguments_before_any_launch(lib):
    assert indexed(lib, P=0) == 1                 # no cluster kept
    assert indexed(lib, P=65) == 1                # more kept than clusters
    assert indexed(lib, K1=64, P=33) == 1         # more than 32 kept
    assert indexed(lib, K1=5000, K=8192) == 1     # more than 4096 clusters
    assert indexed(lib, ms=0) == 1                # empty largest cluster
    assert indexed(lib, s=ODD) == 1               # misaligned super-centres
    assert indexed(lib, dt=0) == 2                # fp32 storage: unsupported
    assert indexed(lib, d=96) == 2                # head dim
    assert indexed(lib, wsb=256) == 3             # workspace too small
    need = lib.asm_decode_indexed_workspace_size(1, 32, 8, 64, 8, 40, 256, 128, 1)
    assert need > 0 and indexed(lib, wsb=need - 16) == 3
    assert lib.asm_decode_indexed_workspace_size(1, 32, 8, 64, 8, 40, 256, 128, 0) == 0  # fp32


def test_index_reorder_rejects_bad_arguments(lib):
    args = [FAKE, 4, 100, 128, 1, FAKE, FAKE, FAKE, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000),
            ctypes.c_void_p(0x40000), None]
    bad = list(args)
    bad[0] = NULL
    assert lib.asm_index_reorder(*bad) == 1       # no permutation
    bad = list(args)
    bad[8] = FAKE
    assert lib.asm_index_reorder(*bad) == 1       # output aliases its input
    bad = list(args)
    bad[3] = 80
    assert lib.asm_index_reorder(*bad) == 2       # head dim


def test_whitening_and_search_decode_reject_bad_arguments(lib):
    P = FAKE
    ws_need = lib.asm_whitening_workspace_size(32, 128)
    assert ws_need > 0 and lib.asm_whitening_workspace_size(32, 96) == 0
    # asm_whitening(x, H, N, d, dt, eps_rel, mu, W, ws, ws_bytes, stream)
    assert lib.asm_whitening(P, 32, 65536, 96, 1, 1e-5, P, P, P, ws_need, None) == UNSUPPORTED
    assert lib.asm_whitening(NULL, 32, 65536, 128, 1, 1e-5, P, P, P, ws_need, None) == INVALID
    assert lib.asm_whitening(P, 32, 0, 128, 1, 1e-5, P, P, P, ws_need, None) == INVALID
    assert lib.asm_whitening(P, 32, 100, 128, 1, -1.0, P, P, P, ws_need, None) == INVALID
    assert lib.asm_whitening(P, 32, 100, 128, 1, float("nan"), P, P, P, ws_need, None) == INVALID
    assert lib.asm_whitening(P, 32, 100, 128, 1, 1e-5, P, P, P, ws_need - 1, None) == WORKSPACE
    # asm_whiten(x, H, R, d, dt, sh, sr, mu, W, y, ysh, ysr, stream)
    assert lib.asm_whiten(P, 2, 10, 128, 1, 1280, -128, P, P, P, 1280, 128, None) == INVALID
    assert lib.asm_whiten(P, 2, 10, 100, 1, 1000, 100, P, P, P, 1000, 100, None) == UNSUPPORTED
    assert lib.asm_whiten(P, 2, 10, 128, 1, 1280, 128, P, P, NULL, 1280, 128, None) == INVALID
    assert lib.asm_whiten(P, 2, 0, 128, 1, 1280, 128, P, P, P, 1280, 128, None) == 0  # nothing to do
    # asm_decode_step_search: a missing search query is rejected first
    assert lib.asm_decode_step_search(P, NULL, P, P, P, P, P, P, 1, 32, 8, 1024, 2048, 128, 0.088, 0, 1, P,
                                      NULL, NULL, 0, P, 1 << 30, None) == INVALID
    assert lib.asm_decode_step_search(P, ODD, P, P, P, P, P, P, 1, 32, 8, 1024, 2048, 128, 0.088, 0, 1, P,
                                      NULL, NULL, 0, P, 1 << 30, None) == INVALID
    assert lib.asm_decode_step_search(P, P, P, P, P, P, P, P, 1, 32, 8, 1024, 2048, 128, 0.088, 0, 1, P,
                                      NULL, NULL, 0, P, 8, None) == WORKSPACE


def test_whiten_binding_needs_an_unambiguous_layout():
    """The Python binding infers [H, R, d] or [R, H, d] from mu's head count and
    refuses to guess when both dimensions equal it (no library call is made)."""
    import torch
    from long_prefix_attention_b200 import ops
    mu = torch.zeros(4, 64)
    W = torch.zeros(4, 64, 64)
    x = torch.zeros(4, 4, 64)
    with pytest.raises(ops.AsmError):
        ops.asm_whiten(x, mu, W, torch.zeros_like(x))
    with pytest.raises(ops.AsmError):  # the named layout must match the shape
        ops.asm_whiten(torch.zeros(5, 3, 64), mu, W, torch.zeros(5, 3, 64), layout="heads")
    with pytest.raises(ops.AsmError):  # shape and dtype of y must match x
        ops.asm_whiten(torch.zeros(4, 7, 64), mu, W, torch.zeros(4, 7, 64, dtype=torch.bfloat16))

"""asm_decode_step_noalloc: the decode step for callers that cannot allocate
device memory where they decode (it uses the library's built-in 8 MiB scratch
instead of a caller workspace).  Its outputs must match those of
asm_decode_step on the same inputs, call after call.

This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from long_prefix_attention_b200 import _lib, inputs, ops

pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 storage, as in the other decode parity tests


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_decode_twice():
    lib = _lib.load()
    cfg = dict(inputs.CONFIGS[1])
    ins = inputs.decode_inputs(cfg, B=2, K=700, T=300, local_len=[300, 177])
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in ins.items()}
    B, Hq, D = d["q"].shape
    Hkv, T = d["k_cache"].shape[1:3]
    K = d["centroids"].shape[1]
    # reference: the entry point with a caller workspace
    ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, D, d["q"].dtype), "cuda")
    ref = torch.empty_like(d["q"])
    ref_lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    ops.asm_decode_step(d["q"], d["centroids"], d["a_bar"], d["logz_bar"], d["k_cache"], d["v_cache"],
                        d["local_len"], d["scale"], ref, ws, lse_out=ref_lse)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(d["q"], float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((B, Hq), -1, dtype=torch.int32, device="cuda")
        st = lib.asm_decode_step_noalloc(
            _p(d["q"]), _p(d["centroids"]), _p(d["a_bar"]), _p(d["logz_bar"]), _p(d["k_cache"]),
            _p(d["v_cache"]), _p(d["local_len"]), B, Hq, Hkv, K, T, D, d["scale"], ops.ASM_L2,
            ops.ASM_BF16, _p(out), _p(lse), _p(idx), 0, stream)
        assert st == 0, ops.status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert (out.float() - ref.float()).abs().max().item() <= TOL, f"call {call}"
        assert (lse - ref_lse).abs().max().item() <= TOL, f"call {call}"
        assert (idx >= 0).all() and (idx < K).all()


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib.load()
    need = lib.asm_decode_workspace_size(64, 32, 8, 8192, 32768, 128, ops.ASM_BF16)
    assert need > 8 << 20
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = _p(x)
    st = lib.asm_decode_step_noalloc(p, p, p, p, p, p, p, 64, 32, 8, 8192, 32768, 128, 0.088,
                                     ops.ASM_L2, ops.ASM_BF16, p, None, None, 0, None)
    assert st == 3  # ASM_ERR_WORKSPACE: nothing was launched

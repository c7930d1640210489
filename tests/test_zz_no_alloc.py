"""asm_decode_step_noalloc: the decode step for callers that cannot allocate
device memory where they decode -- a plug-in whose host framework owns every
device allocation, or a latency-critical loop where cudaMalloc is ruled out
because it may synchronise the device.  It uses the library's built-in 8 MiB
scratch array instead of a caller workspace.  It runs the same kernels with
the same launch shape as asm_decode_step, so its outputs (out, lse and the
retrieved index) must equal those of asm_decode_step bit for bit, call after
call, although the scratch keeps the previous call's contents.

This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from long_prefix_attention_b200 import _lib, inputs, ops

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _check_twice(ins, dt_code):
    lib = _lib.load()
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in ins.items()}
    B, Hq, D = d["q"].shape
    Hkv, T = d["k_cache"].shape[1:3]
    K = d["centroids"].shape[1]
    # reference: the entry point with a caller workspace
    ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, D, d["q"].dtype), "cuda")
    ref = torch.empty_like(d["q"])
    ref_lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    ref_idx = torch.empty(B, Hq, dtype=torch.int32, device="cuda")
    ops.asm_decode_step(d["q"], d["centroids"], d["a_bar"], d["logz_bar"], d["k_cache"], d["v_cache"],
                        d["local_len"], d["scale"], ref, ws, lse_out=ref_lse, idx_out=ref_idx)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(d["q"], float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((B, Hq), -1, dtype=torch.int32, device="cuda")
        st = lib.asm_decode_step_noalloc(
            _p(d["q"]), _p(d["centroids"]), _p(d["a_bar"]), _p(d["logz_bar"]), _p(d["k_cache"]),
            _p(d["v_cache"]), _p(d["local_len"]), B, Hq, Hkv, K, T, D, d["scale"], ops.ASM_L2,
            dt_code, _p(out), _p(lse), _p(idx), 0, stream)
        assert st == 0, ops.status_string(st)
        torch.cuda.synchronize()
        assert ops.asm_decode_noalloc_error() == 0, f"call {call}: device-side timeout"
        assert torch.equal(out, ref), f"call {call}: out differs"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs"
        assert torch.equal(idx, ref_idx), f"call {call}: idx differs"


def test_noalloc_matches_workspace_decode_twice():
    """bf16 at the LLaMA layer shape (8 KV heads), two ragged rows."""
    ins = inputs.decode_inputs(dict(inputs.CONFIGS[1]), B=2, K=700, T=300, local_len=[300, 177])
    _check_twice(ins, ops.ASM_BF16)


def test_noalloc_fp32_counters_start_from_zero():
    """fp32 at the tiny config's shapes (d = 64): its kernel keeps per-(b, g)
    arrival counters in the scratch, which each call must find at zero."""
    cfg = dict(inputs.CONFIGS[0], logz_lo=5.0, logz_hi=10.0)
    ins = inputs.decode_inputs(cfg, seed=inputs.BASE_SEED + 300, B=3, K=cfg["K"], T=cfg["T"],
                               local_len=[cfg["T"], 0, 5])
    _check_twice(ins, ops.ASM_F32)


def test_noalloc_rejects_bad_calls_before_touching_the_stream():
    lib = _lib.load()
    need = lib.asm_decode_workspace_size(64, 32, 8, 8192, 32768, 128, ops.ASM_BF16)
    assert need > 8 << 20
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = _p(x)
    st = lib.asm_decode_step_noalloc(p, p, p, p, p, p, p, 64, 32, 8, 8192, 32768, 128, 0.088,
                                     ops.ASM_L2, ops.ASM_BF16, p, None, None, 0, None)
    assert st == ops.ASM_ERR_WORKSPACE  # beyond the built-in scratch: nothing was launched
    # an invalid argument is rejected before the scratch is cleared
    st = lib.asm_decode_step_noalloc(p, p, p, p, p, p, None, 1, 32, 8, 1024, 2048, 128, 0.088,
                                     ops.ASM_L2, ops.ASM_BF16, p, None, None, 0, None)
    assert st == ops.ASM_ERR_INVALID_ARG

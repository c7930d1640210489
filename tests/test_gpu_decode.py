"""Parity of asm_decode_step and asm_flash_decode (CUDA, through the C ABI)
with the fp64 oracle on seeded inputs.

Decode step: "Fase de Inferencia Online" of "Context Memorization for
Efficient Long Context Generation" (Recuperacion: nearest centroid; Fusion:
online-softmax merge of its stored state with attention over the local
tokens).
"""
import math

import numpy as np
import pytest
import torch

from long_prefix_attention_b200 import inputs, ops
from oracle import asm_oracle as O

from gpu_common import TOL, check_indices, dev, f64, host, max_abs

pytestmark = pytest.mark.gpu


def run_decode(ins, metric=ops.ASM_L2, with_lse=True, with_idx=True, calls=1, flags=0):
    q, C, Ab, lz = (dev(ins[k]) for k in ("q", "centroids", "a_bar", "logz_bar"))
    kc, vc, ll = dev(ins["k_cache"]), dev(ins["v_cache"]), dev(ins["local_len"])
    B, Hq, d = q.shape
    K = C.shape[1]
    _, Hkv, Tmax, _ = kc.shape
    ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, Tmax, d, q.dtype), q.device)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if with_lse else None
    idx = torch.empty(B, Hq, dtype=torch.int32, device=q.device) if with_idx else None
    for _ in range(calls):
        out.fill_(float("nan"))
        ops.asm_decode_step(q, C, Ab, lz, kc, vc, ll, ins["scale"], out, ws, lse_out=lse,
                            idx_out=idx, metric=metric, flags=flags)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    return out, lse, idx


def check_decode(ins, metric=ops.ASM_L2, calls=1, flags=0):
    out, lse, idx = run_decode(ins, metric, calls=calls, flags=flags)
    o_out, o_lse, o_idx, o_gap = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"],
                                          ins["k_cache"], ins["v_cache"], ins["local_len"],
                                          ins["scale"], metric)
    g_idx = host(idx).numpy()
    bad = check_indices(g_idx, o_idx, o_gap)
    if bad.any():  # near-ties: compare against the oracle on the GPU's choice
        o_out, o_lse, _, _ = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"],
                                      ins["k_cache"], ins["v_cache"], ins["local_len"],
                                      ins["scale"], metric, idx_in=g_idx)
    tol = TOL[ins["q"].dtype]
    assert max_abs(f64(out), o_out) <= tol
    assert max_abs(f64(lse), o_lse) <= tol
    return out


def small_case(dt, B=2, Hq=8, Hkv=2, K=100, T=45, d=128, local_len=None, seed=7):
    cfg = dict(inputs.CONFIGS[1])
    cfg.update(dtype=dt, Hq=Hq, Hkv=Hkv, d=d, n_mix=16)
    return inputs.decode_inputs(cfg, seed=seed, B=B, K=K, T=T, local_len=local_len)


def test_decode_tiny_fp32_config():
    """The tiny fp32 workload: 8 independent batch-1 steps, local length 16."""
    cfg = inputs.CONFIGS[0]
    for i in range(cfg["n_decode"]):
        ins = inputs.decode_inputs(dict(cfg, logz_lo=5.0, logz_hi=10.0), seed=inputs.BASE_SEED + 100 + i,
                                   B=1, K=cfg["K"], T=cfg["T"])
        check_decode(ins)


def test_decode_llama_layer_k1024_t2048_b1():
    check_decode(inputs.decode_inputs(inputs.CONFIGS[1]), calls=3)


def test_decode_llama_layer_prefetching_centroids():
    """ASM_DECODE_PREFETCH_CENTROIDS streams centroid units before the
    dependency wait; the results are those of the plain call."""
    check_decode(inputs.decode_inputs(inputs.CONFIGS[1]), calls=2, flags=ops.ASM_DECODE_PREFETCH_CENTROIDS)
    check_decode(small_case("bf16", B=3, K=700, T=90, local_len=[90, 0, 45]),
                 flags=ops.ASM_DECODE_PREFETCH_CENTROIDS)


def test_decode_llama_layer_k8192_t4096_b16():
    check_decode(inputs.decode_inputs(inputs.CONFIGS[2]))


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_shapes(dt, d, G):
    Hkv = 2
    ins = small_case(dt, B=3, Hq=G * Hkv, Hkv=Hkv, K=131, T=77, d=d, local_len=[77, 33, 1], seed=G * d)
    check_decode(ins)


def test_decode_ragged_and_empty_local():
    ins = small_case("bf16", B=4, K=64, T=100, local_len=[0, 100, 31, 64])
    out = check_decode(ins)
    # row 0 has no local tokens: the output is the retrieved state itself
    o_out, o_lse, o_idx, _ = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"],
                                      ins["k_cache"], ins["v_cache"], ins["local_len"], ins["scale"])
    ab = f64(ins["a_bar"])
    for h in range(ins["q"].shape[1]):
        np.testing.assert_allclose(f64(out)[0, h], ab[h, o_idx[0, h]], atol=1e-2)


def test_decode_no_local_cache_and_single_centroid():
    ins = small_case("f32", B=2, K=1, T=0)
    check_decode(ins)


def test_decode_cosine_metric():
    check_decode(small_case("bf16", B=2, K=300, T=50), metric=ops.ASM_COSINE)


def test_decode_empty_memory_state_is_local_attention():
    ins = small_case("f32", B=2, K=5, T=40)
    ins["logz_bar"] = torch.full_like(ins["logz_bar"], -math.inf)
    out = check_decode(ins)
    ref, ref_lse = O.full_attention(ins["q"], np.zeros((2, 0, 128)), np.zeros((2, 0, 128)),
                                    ins["k_cache"], ins["v_cache"], ins["local_len"], ins["scale"])
    assert max_abs(f64(out), ref) <= 1e-4


def test_decode_optional_outputs_absent():
    ins = small_case("bf16")
    out, _, _ = run_decode(ins, with_lse=False, with_idx=False)
    o_out, _, _, _ = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"],
                              ins["k_cache"], ins["v_cache"], ins["local_len"], ins["scale"])
    assert max_abs(f64(out), o_out) <= 2e-2


def test_decode_counters_reset_across_calls():
    """Self-resetting arrival counters: repeated calls on one workspace agree."""
    ins = small_case("bf16", B=3, K=500, T=300)
    out1, _, _ = run_decode(ins, calls=1)
    out5, _, _ = run_decode(ins, calls=5)
    assert torch.equal(out1, out5)


# ------------------------------------------- LLaMA-like KV-head counts --
#
# 8 or more KV heads (the LLaMA-3.1-8B layer has 8): every group size and
# head dim, ragged and empty local windows, partial centroid tiles, the
# largest batch, long windows and the longest batch-1 window of the sweep.

def fused_case(B, G, d, K, T, local_len=None, Hkv=8, seed=11):
    return small_case("bf16", B=B, Hq=G * Hkv, Hkv=Hkv, K=K, T=T, d=d, local_len=local_len, seed=seed)


def assert_two_launches(ins):
    B, Hq, d = ins["q"].shape
    K = ins["centroids"].shape[1]
    _, Hkv, T, _ = ins["k_cache"].shape
    assert ops.asm_decode_step_launches(B, Hq, Hkv, K, T, d, torch.bfloat16) == 2


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_llama_heads_shapes(d, G):
    ins = fused_case(5, G, d, K=300, T=200, local_len=[200, 0, 1, 129, 64], seed=G * d + 1)
    assert_two_launches(ins)
    check_decode(ins, calls=2)


@pytest.mark.parametrize("B,K,T,lens", [
    (1, 1, 0, None),                  # no local cache, one centre
    (1, 129, 1, None),                # one token; a partial second centroid tile
    (64, 1000, 70, "ragged"),         # a large batch with ragged rows, some empty
    (33, 4097, 65, None),             # an odd batch; a one-row last centroid unit
    (2, 5000, 3000, [3000, 1500]),    # long windows: many partials per row
])
def test_decode_llama_heads_edges(B, K, T, lens):
    if lens == "ragged":
        lens = [(7 * b) % (T + 1) for b in range(B)]
    ins = fused_case(B, 4, 128, K=K, T=T, local_len=lens, seed=B + K)
    assert_two_launches(ins)
    check_decode(ins)


@pytest.mark.parametrize("Hkv,G", [(16, 2), (32, 1)])
def test_decode_llama_heads_more_kv_heads(Hkv, G):
    ins = fused_case(3, G, 128, K=700, T=150, local_len=[150, 77, 0], Hkv=Hkv, seed=Hkv)
    assert_two_launches(ins)
    check_decode(ins)


def test_decode_llama_heads_long_window_b1():
    """The longest batch-1 window of the throughput sweep: K = 8192, T = 32768."""
    ins = inputs.decode_inputs(inputs.CONFIGS[1], seed=inputs.BASE_SEED + 77, B=1, K=8192, T=32768)
    assert_two_launches(ins)
    check_decode(ins)


def test_decode_llama_heads_cosine_prefetch_and_repeat():
    ins = fused_case(3, 4, 128, K=900, T=333, local_len=[333, 5, 200], seed=5)
    check_decode(ins, metric=ops.ASM_COSINE, flags=ops.ASM_DECODE_PREFETCH_CENTROIDS)
    # nothing carries over between calls: one call and five calls agree bit for bit
    out1, lse1, idx1 = run_decode(ins, calls=1)
    out5, lse5, idx5 = run_decode(ins, calls=5, flags=ops.ASM_DECODE_PREFETCH_CENTROIDS)
    assert torch.equal(out1, out5) and torch.equal(lse1, lse5) and torch.equal(idx1, idx5)


def test_decode_llama_heads_search_query():
    """asm_decode_step_search: the search uses its own query, the local
    attention and the merge use q."""
    ins = fused_case(2, 4, 128, K=500, T=100, seed=9)
    qs_ins = fused_case(2, 4, 128, K=500, T=100, seed=10)
    q, qs = dev(ins["q"]), dev(qs_ins["q"])
    C, Ab, lz = dev(ins["centroids"]), dev(ins["a_bar"]), dev(ins["logz_bar"])
    kc, vc, ll = dev(ins["k_cache"]), dev(ins["v_cache"]), dev(ins["local_len"])
    B, Hq, d = q.shape
    ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, 8, 500, 100, d, q.dtype), "cuda")
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, Hq, dtype=torch.int32, device="cuda")
    ops.asm_decode_step_search(q, qs, C, Ab, lz, kc, vc, ll, ins["scale"], out, ws, lse_out=lse, idx_out=idx)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    _, _, s_idx, s_gap = O.decode(qs_ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"],
                                  ins["k_cache"], ins["v_cache"], ins["local_len"], ins["scale"])
    g_idx = host(idx).numpy()
    check_indices(g_idx, s_idx, s_gap)
    o_out, o_lse, _, _ = O.decode(ins["q"], ins["centroids"], ins["a_bar"], ins["logz_bar"], ins["k_cache"],
                                  ins["v_cache"], ins["local_len"], ins["scale"], idx_in=g_idx)
    assert max_abs(f64(out), o_out) <= TOL[torch.bfloat16]
    assert max_abs(f64(lse), o_lse) <= TOL[torch.bfloat16]


# ------------------------------------------------------------ flash decode --

def run_flash(q, kp, vp, kc, vc, ll, scale):
    B, Hq, d = q.shape
    Hkv, Lp, _ = kp.shape
    Tmax = kc.shape[2]
    ws = ops.alloc_workspace(ops.asm_flash_decode_workspace_size(B, Hq, Hkv, Lp, Tmax, d, q.dtype),
                             q.device)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    ops.asm_flash_decode(q, kp, vp, kc, vc, ll, scale, out, ws, lse_out=lse)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("dt,Lp,T,B", [("bf16", 4096, 256, 2), ("f32", 333, 17, 3), ("bf16", 0, 64, 1),
                                      ("bf16", 100, 0, 2)])
def test_flash_decode_matches_full_attention(dt, Lp, T, B):
    ins = small_case(dt, B=B, K=4, T=T, local_len=[T] * B)
    kp = inputs.normal(99, "kp", (2, Lp, 128), dt)
    vp = inputs.normal(99, "vp", (2, Lp, 128), dt)
    out, lse = run_flash(dev(ins["q"]), dev(kp), dev(vp), dev(ins["k_cache"]), dev(ins["v_cache"]),
                         dev(ins["local_len"]), ins["scale"])
    ref, ref_lse = O.full_attention(ins["q"], kp, vp, ins["k_cache"], ins["v_cache"], ins["local_len"],
                                    ins["scale"])
    tol = TOL[ins["q"].dtype]
    assert max_abs(f64(out), ref) <= tol
    assert max_abs(f64(lse), ref_lse) <= tol


def test_flash_decode_batch_rows_share_the_prefix():
    """Five rows with ragged local lengths over one explicit prefix whose
    length is not a multiple of the tile: the rows that read a prefix tile
    run together, each with its own local window."""
    lens = [130, 0, 64, 129, 1]
    ins = small_case("bf16", B=5, K=4, T=130, local_len=lens)
    kp = inputs.normal(7, "kp", (2, 700, 128), "bf16")
    vp = inputs.normal(7, "vp", (2, 700, 128), "bf16")
    out, lse = run_flash(dev(ins["q"]), dev(kp), dev(vp), dev(ins["k_cache"]), dev(ins["v_cache"]),
                         dev(ins["local_len"]), ins["scale"])
    ref, ref_lse = O.full_attention(ins["q"], kp, vp, ins["k_cache"], ins["v_cache"], ins["local_len"],
                                    ins["scale"])
    assert max_abs(f64(out), ref) <= 2e-2
    assert max_abs(f64(lse), ref_lse) <= 2e-2


def test_identity_memory_recovers_full_attention():
    """K = N memory built on the GPU (states of the calibration queries
    themselves, singleton clusters): a decode query equal to calibration
    query i retrieves i and the merged output equals attention over
    prefix + local ("Fusion" bullet: exact as if the prefix were present)."""
    dt = torch.bfloat16
    Hq, Hkv, N, L, d, B, T = 8, 2, 256, 1024, 128, 4, 200
    cfg = dict(inputs.CONFIGS[3], Hq=Hq, Hkv=Hkv, n_mix=32)
    bi = inputs.build_inputs(cfg, seed=5, N=N, L=L, K=N)
    q_cal, kp, vp = dev(bi["q"]), dev(bi["k"]), dev(bi["v"])
    a = torch.empty_like(q_cal)
    logz = torch.empty(Hq, N, dtype=torch.float32, device="cuda")
    ops.asm_build_states(q_cal, kp, vp, bi["scale"], a, logz)
    perm = torch.arange(N, dtype=torch.int32, device="cuda").repeat(Hq, 1).contiguous()
    seg = torch.arange(N + 1, dtype=torch.int32, device="cuda").repeat(Hq, 1).contiguous()
    a_bar = torch.empty_like(a)
    lz_bar = torch.empty_like(logz)
    ops.asm_aggregate(a, logz, perm, seg, a_bar, lz_bar)
    g = torch.Generator().manual_seed(3)
    pick = torch.randint(0, N, (B, Hq), generator=g)
    qd = torch.stack([bi["q"][torch.arange(Hq), pick[b]] for b in range(B)]).contiguous()
    kc = inputs.normal(11, "kc", (B, Hkv, T, d), "bf16")
    vc = inputs.normal(11, "vc", (B, Hkv, T, d), "bf16")
    ll = torch.tensor([200, 0, 57, 128], dtype=torch.int32)
    ins = dict(q=qd, centroids=bi["q"], a_bar=host(a_bar), logz_bar=host(lz_bar), k_cache=kc,
               v_cache=vc, local_len=ll, scale=bi["scale"])
    out, lse, idx = run_decode(ins)
    assert torch.equal(host(idx).long(), pick)
    ref, ref_lse = O.full_attention(qd, bi["k"], bi["v"], kc, vc, ll, bi["scale"])
    assert max_abs(f64(out), ref) <= 2e-2
    assert max_abs(f64(lse), ref_lse) <= 2e-2

"""Parity of the two-level (hierarchical) memory with the fp64 oracle.

The retrieval the pages describe is hierarchical ("Complejidad" in "Context
Memorization for Efficient Long Context Generation"); the index is built with
the library's own k-means on the centres, the memory is laid out by cluster,
and the decode keeps the P best clusters and retrieves the best member.
"""
import numpy as np
import pytest
import torch

from long_prefix_attention_b200 import inputs, ops
from oracle import asm_oracle as O

from gpu_common import GAP, dev, f64, host, max_abs

pytestmark = pytest.mark.gpu


def structured_memory(Hq=4, Hkv=2, K=1500, d=128, n_mix=64, seed=21):
    """Centres drawn from a Gaussian mixture (clustered, like k-means centres
    of real queries), random states, and decode queries from the same mixture."""
    cfg = dict(inputs.CONFIGS[1], Hq=Hq, Hkv=Hkv, d=d, n_mix=n_mix, sigma=0.3)
    cen = inputs.mixture(seed, "calib_q", Hq, K, d, n_mix, 0.3, "bf16")
    return cfg, cen


def build_index(cen, K1, iters=4):
    """Super-centres, members and the ordered memory, all on the GPU."""
    H, K, d = cen.shape
    x = dev(cen)
    u = dev(inputs.kmeanspp_uniforms(inputs.BASE_SEED + 77, H, K1))
    init = torch.empty(H, K1, dtype=torch.int32, device="cuda")
    ws_s = ops.alloc_workspace(ops.asm_kmeanspp_workspace_size(H, K, d, K1), "cuda", zero=False)
    ops.asm_kmeanspp_seed(x, u, init, ws_s)
    c = torch.empty(H, K1, d, dtype=torch.float32, device="cuda")
    sdt = torch.empty(H, K1, d, dtype=x.dtype, device="cuda")
    assign = torch.empty(H, K, dtype=torch.int32, device="cuda")
    counts = torch.empty(H, K1, dtype=torch.int32, device="cuda")
    perm = torch.empty(H, K, dtype=torch.int32, device="cuda")
    seg = torch.empty(H, K1 + 1, dtype=torch.int32, device="cuda")
    ws = ops.alloc_workspace(ops.asm_kmeans_workspace_size(H, K, d, K1), "cuda")
    ops.asm_kmeans(x, init, iters, c, sdt, assign, counts, perm, seg, ws)
    torch.cuda.synchronize()
    return x, sdt, perm, seg, int(host(counts).max())


def ordered(x, perm, seed=5):
    H, K, d = x.shape
    a_bar = dev(inputs.normal(seed, "a_bar", (H, K, d), "bf16"))
    lz = dev(inputs.uniform(seed, "logz_bar", (H, K), 5.0, 10.0))
    c_o, a_o = torch.empty_like(x), torch.empty_like(a_bar)
    lz_o = torch.empty_like(lz)
    ops.asm_index_reorder(perm, x, a_bar, lz, c_o, a_o, lz_o)
    torch.cuda.synchronize()
    return a_bar, lz, c_o, a_o, lz_o


def decode_inputs(cfg, B, T, Hq, Hkv, d, K, seed=9):
    ins = inputs.decode_inputs(dict(cfg, Hq=Hq, Hkv=Hkv, d=d), seed=seed, B=B, K=4, T=T)
    # decode queries: further draws from the mixture the centres came from
    q = inputs.mixture(21, "calib_q", Hq, K + 100 + B, d, cfg["n_mix"], 0.3, "bf16")[:, K + 100:]
    ins["q"] = q.transpose(0, 1).contiguous()
    return ins


def run_indexed(ins, sdt, seg, P, max_seg, c_o, a_o, lz_o):
    q = dev(ins["q"])
    B, Hq, d = q.shape
    kc, vc = dev(ins["k_cache"]), dev(ins["v_cache"])
    Hkv, T = kc.shape[1], kc.shape[2]
    K1 = sdt.shape[1]
    ws = ops.alloc_workspace(ops.asm_decode_indexed_workspace_size(B, Hq, Hkv, K1, P, max_seg, T, d, q.dtype),
                             "cuda")
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, Hq, dtype=torch.int32, device="cuda")
    ops.asm_decode_step_indexed(q, sdt, seg, P, max_seg, c_o, a_o, lz_o, kc, vc, dev(ins["local_len"]),
                                ins["scale"], out, ws, lse_out=lse, idx_out=idx)
    torch.cuda.synchronize()
    assert ops.asm_workspace_error(ws) == 0
    return out, lse, idx


def test_index_reorder_is_an_exact_gather():
    cfg, cen = structured_memory(K=700)
    x, sdt, perm, seg, max_seg = build_index(cen, 20)
    a_bar, lz, c_o, a_o, lz_o = ordered(x, perm)
    pr = perm.long()
    hh = torch.arange(x.shape[0], device="cuda")[:, None]
    assert torch.equal(c_o, x[hh, pr]) and torch.equal(a_o, a_bar[hh, pr]) and torch.equal(lz_o, lz[hh, pr])
    # members of every cluster are contiguous and ascending
    s = host(seg).numpy()
    assert (s[:, 0] == 0).all() and (s[:, -1] == 700).all() and (np.diff(s, axis=1) >= 0).all()


@pytest.mark.parametrize("K,K1,P", [(1500, 40, 4), (1500, 40, 1), (1024, 5, 2), (600, 30, 30)])
def test_indexed_decode_matches_the_two_level_oracle(K, K1, P):
    Hq, Hkv, d, B, T = 4, 2, 128, 3, 100
    cfg, cen = structured_memory(Hq=Hq, Hkv=Hkv, K=K, d=d)
    x, sdt, perm, seg, max_seg = build_index(cen, K1)
    a_bar, lz, c_o, a_o, lz_o = ordered(x, perm)
    ins = decode_inputs(cfg, B, T, Hq, Hkv, d, K)
    out, lse, idx = run_indexed(ins, sdt, seg, P, max_seg, c_o, a_o, lz_o)
    o_idx, o_sel, gap_sel, gap_idx = O.index_search(ins["q"], f64(sdt), host(seg).numpy(), f64(c_o), P)
    g_idx = host(idx).numpy()
    bad = g_idx != o_idx
    # a mismatch is accepted only where the oracle's own choice is a near-tie
    assert not (bad & (gap_sel >= GAP) & (gap_idx >= GAP)).any(), f"{int(bad.sum())} mismatches"
    # the retrieved row is valid: a member of one of the oracle's kept clusters
    # (or of a near-tied one), and the output is the oracle's at that row
    ref, ref_lse, _, _ = O.decode(ins["q"], f64(c_o), f64(a_o), host(lz_o).numpy(), ins["k_cache"],
                                  ins["v_cache"], ins["local_len"], ins["scale"], idx_in=g_idx)
    assert max_abs(f64(out), ref) <= 2e-2
    assert max_abs(f64(lse), ref_lse) <= 2e-2
    if P == K1:
        # every cluster kept: the flat search over the ordered memory
        flat = torch.empty_like(idx)
        ws = ops.alloc_workspace(ops.asm_decode_workspace_size(B, Hq, Hkv, K, T, d, torch.bfloat16), "cuda")
        o2 = torch.empty_like(out)
        ops.asm_decode_step(dev(ins["q"]), c_o, a_o, lz_o, dev(ins["k_cache"]), dev(ins["v_cache"]),
                            dev(ins["local_len"]), ins["scale"], o2, ws, idx_out=flat)
        torch.cuda.synchronize()
        fo, fgap = zip(*[O.assign(ins["q"][:, h], f64(c_o)[h]) for h in range(Hq)])
        fgap = np.stack(fgap, 1)
        diff = host(flat).numpy() != g_idx
        assert not (diff & (fgap >= GAP)).any()

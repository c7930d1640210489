"""Split of the memory build over several GPUs (one process per GPU).

Every query head is built independently, and the prefix seen by one KV
group can be cut into chunks whose attention states combine by the
online-softmax identity ("Context Memorization for Efficient Long Context
Generation", Metodologia, "Eficiencia").  Two splits follow from that:

* ``head_shard``: each rank builds whole KV groups of the query heads
  (states, clustering, aggregation); nothing crosses GPUs.
* ``chunk_shard`` and ``build_states_split``: each rank encodes a contiguous
  run of the prefix chunks with ``asm_build_states`` (merging its own chunks
  in order), the ranks all-gather their (a, logZ) states, and every rank
  folds them in chunk order with ``asm_merge_states``.  The gathered states
  arrive in rank order, which is chunk order.

The collective goes through ``torch.distributed`` (NCCL between GPUs); the
attention and merge arithmetic run in the library's kernels.  ``encode`` and
``merge`` can be replaced, which the CPU tests of the plumbing use.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops


def head_shard(Hq: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """Query heads [h0, h1) of rank `rank`: whole KV groups (the Hq / Hkv
    query heads sharing a KV head stay together), as even as the groups
    allow; a rank gets none when world > Hkv."""
    G = Hq // Hkv
    g0, g1 = rank * Hkv // world, (rank + 1) * Hkv // world
    return g0 * G, g1 * G


def chunk_shard(n_chunks: int, world: int, rank: int) -> tuple[int, int]:
    """Prefix chunks [c0, c1) that rank `rank` encodes: contiguous runs in
    rank order, as even as possible; a rank gets none when world > n_chunks."""
    return rank * n_chunks // world, (rank + 1) * n_chunks // world


def build_states_split(q, k_chunks, v_chunks, scale: float, a, logz, group=None, encode=None, merge=None):
    """States of q over the concatenation of the prefix chunks, with the
    chunks split over the ranks of `group`.

    q [Hq, N, d]; k_chunks / v_chunks: the prefix chunks in order, each
    [Hkv, L_i, d] (every rank passes all of them, or at least its own);
    a [Hq, N, d] and logz [Hq, N] receive the states over the whole prefix,
    on every rank.  encode(q, k, v, scale, a, logz, accumulate) and
    merge(a, logz, a_in, logz_in) default to asm_build_states and
    asm_merge_states.
    """
    encode = encode or (lambda q_, k_, v_, s_, a_, z_, acc: ops.asm_build_states(q_, k_, v_, s_, a_, z_, accumulate=acc))
    merge = merge or ops.asm_merge_states
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    c0, c1 = chunk_shard(len(k_chunks), world, rank)
    if c1 == c0:
        # no chunk here: the empty state (a = 0, logZ = -inf), the merge's identity
        k0 = k_chunks[0][:, :0]
        encode(q, k0, v_chunks[0][:, :0], scale, a, logz, False)
    for i in range(c0, c1):
        encode(q, k_chunks[i], v_chunks[i], scale, a, logz, i > c0)
    if world == 1:
        return a, logz
    parts_a = [torch.empty_like(a) for _ in range(world)]
    parts_z = [torch.empty_like(logz) for _ in range(world)]
    dist.all_gather(parts_a, a, group=group)
    dist.all_gather(parts_z, logz, group=group)
    a.copy_(parts_a[0])
    logz.copy_(parts_z[0])
    for j in range(1, world):
        merge(a, logz, parts_a[j], parts_z[j])
    return a, logz

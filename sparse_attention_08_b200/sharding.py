"""Splitting one long prefill over several GPUs (strong scaling).

Query rows are independent once a GPU holds the key side they read ("DeepSeek
V3.2 and the lightning indexer", section "How the lightning indexer works": a
query's scores, selection and attention use only its own row and the keys).
So one sequence of L queries is cut into 2·world equal blocks and rank r takes
blocks r and 2·world−1−r: block b costs about (b + ½)·(L/2w)² causal pairs, so
every rank gets the same total (zig-zag).  When the key-side cache is sharded
by position (rank r holds keys [r·L/w, (r+1)·L/w)), one all-gather per tensor
gives every rank the whole cache; that exchange is the only collective.

A block [q0, q1) runs as a chunk under the library's varlen convention: one
sequence with len_q = q1 − q0 queries against len_k = q1 keys, so its local
query i sits at position q0 + i.
"""
from __future__ import annotations


def zigzag_blocks(L: int, world: int, rank: int) -> list[tuple[int, int]]:
    """The two query blocks [q0, q1) of rank `rank` (L divisible by 2·world)."""
    if world < 1 or not 0 <= rank < world or L % (2 * world) != 0:
        raise ValueError("zigzag_blocks: L must split into 2*world equal blocks")
    n = L // (2 * world)
    a, b = rank, 2 * world - 1 - rank
    return [(a * n, (a + 1) * n), (b * n, (b + 1) * n)]


def key_shard(L: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [k0, k1) of the position-sharded key cache held by `rank`."""
    if world < 1 or not 0 <= rank < world or L % world != 0:
        raise ValueError("key_shard: L must split into world equal shards")
    n = L // world
    return rank * n, (rank + 1) * n


def block_args(q0: int, q1: int) -> dict:
    """Varlen arguments of block [q0, q1) run as a chunk: its query rows, the
    key rows it reads, cu_seqlens and maxima."""
    if not 0 <= q0 < q1:
        raise ValueError("block_args: empty block")
    return {"q_rows": slice(q0, q1), "key_rows": slice(0, q1), "cu_q": [0, q1 - q0],
            "cu_k": [0, q1], "max_len_q": q1 - q0, "max_len_k": q1}


def all_gather_rows(local, group=None):
    """Concatenates every rank's equal-sized row shard (dim 0) in rank order."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, local.contiguous(), group=group)
    else:
        dist.all_gather(list(out.chunk(world)), local.contiguous(), group=group)
    return out

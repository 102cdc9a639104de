"""Head-group sharding of the layer over GPUs (the pages' tensor-parallel deployment: the
model's attention heads split across GPUs, [P5] "Deploy ...": --tensor-parallel-size).

Rank r of `world` owns KV heads [r Hkv/world, (r+1) Hkv/world) and their Q heads (the GQA
group of KV head g is Q heads [g G, (g+1) G)). The estimator works per KV group and the
selection per Q head, so a shard computes exactly the rows of its heads: there is no exchange
inside attention. The only collective is the all-gather of the output over heads after it
(outside the attention kernels; in a model the output projection's reduction would take its
place).
"""
from __future__ import annotations


def head_shard(n_q_heads: int, n_kv_heads: int, rank: int, world: int):
    """((h0, h1), (g0, g1)): the Q-head and KV-head ranges of `rank`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    if n_kv_heads % world:
        raise ValueError(f"{n_kv_heads} KV heads do not split over {world} ranks")
    G = n_q_heads // n_kv_heads
    per = n_kv_heads // world
    g0, g1 = rank * per, (rank + 1) * per
    return (g0 * G, g1 * G), (g0, g1)


def shard_workload(w, rank: int, world: int):
    """The per-rank layer: the same workload with the rank's head counts."""
    (h0, h1), (g0, g1) = head_shard(w.n_q_heads, w.n_kv_heads, rank, world)
    return w.with_(n_q_heads=h1 - h0, n_kv_heads=g1 - g0)


def shard_inputs(x: dict, w, rank: int, world: int) -> dict:
    """The rank's contiguous slices of q [N][Hq][D], k, v [N][Hkv][D]."""
    (h0, h1), (g0, g1) = head_shard(w.n_q_heads, w.n_kv_heads, rank, world)
    return {"q": x["q"][:, h0:h1].contiguous(), "k": x["k"][:, g0:g1].contiguous(),
            "v": x["v"][:, g0:g1].contiguous()}


def gather_heads(local, world: int, group=None):
    """All-gather of the ranks' outputs [N][Hq/world][D] into [N][Hq][D] (rank order =
    head order), through torch.distributed (NCCL on GPUs, gloo on CPU)."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts, dim=1)

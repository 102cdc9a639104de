"""Head-group sharding: the shard arithmetic, and a 2-rank gloo run on CPU in which each rank
computes its heads with the fp64 oracle and the all-gather over heads reproduces the
unsharded oracle output exactly (the shards do not exchange anything inside attention)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_prefill_dca_b200 import parallel as P
from synth import configs as C


def test_head_shard_ranges():
    assert P.head_shard(28, 4, 0, 2) == ((0, 14), (0, 2))
    assert P.head_shard(28, 4, 1, 2) == ((14, 28), (2, 4))
    assert P.head_shard(40, 8, 3, 4) == ((30, 40), (6, 8))
    assert P.head_shard(28, 4, 0, 1) == ((0, 28), (0, 4))
    with pytest.raises(ValueError):
        P.head_shard(28, 4, 0, 3)          # 4 KV heads over 3 ranks
    with pytest.raises(ValueError):
        P.head_shard(28, 4, 2, 2)
    w = P.shard_workload(C.L7B_1M, 1, 4)
    assert (w.n_q_heads, w.n_kv_heads) == (7, 1) and w.seq_len == C.L7B_1M.seq_len


def _rank(rank, world, port, w, q, k, v, ref, ok):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import dca_vs as O
        x = P.shard_inputs({"q": q, "k": k, "v": v}, w, rank, world)
        ws = P.shard_workload(w, rank, world)
        out, _, _ = O.Oracle(x["q"], x["k"], x["v"], ws).run()
        local = torch.from_numpy(np.stack([out[h] for h in range(ws.n_q_heads)], axis=1))
        full = P.gather_heads(local, world)
        ok[rank] = bool(torch.equal(full, ref))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_gather_equals_unsharded():
    from oracle import dca_vs as O
    w = C.SMALL_SPARSE.with_(seq_len=700, n_q_heads=4, n_kv_heads=2, prefill_chunk=384)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(w.seq_len, w.n_q_heads, w.head_dim, generator=g, dtype=torch.float64)
    k = torch.randn(w.seq_len, w.n_kv_heads, w.head_dim, generator=g, dtype=torch.float64)
    v = torch.randn(w.seq_len, w.n_kv_heads, w.head_dim, generator=g, dtype=torch.float64)
    out, _, _ = O.Oracle(q, k, v, w).run()
    ref = torch.from_numpy(np.stack([out[h] for h in range(w.n_q_heads)], axis=1))
    ctx = mp.get_context("spawn")
    ok = ctx.Manager().dict()
    port = 29000 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, w, q, k, v, ref, ok)) for r in range(2)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(timeout=300)
    assert all(p_.exitcode == 0 for p_ in procs)
    assert ok.get(0) and ok.get(1)

"""Head-group sharding on one GPU: each rank's shard of the layer (its KV groups and their Q
heads) run in turn, one after the other, through the product entry point; the shards
concatenated over heads match the fp64 oracle of the whole layer and the unsharded run.
(The ranks exchange nothing inside attention, so running them in sequence is the same
computation as running them on separate GPUs.)"""
import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import parallel as P
from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Layer
from oracle import dca_vs as O
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_layer_matches_oracle(world):
    w = C.SMALL_SPARSE.with_(n_q_heads=8, n_kv_heads=4)
    x = I.generate(w)
    parts = []
    for r in range(world):
        xs = P.shard_inputs(x, w, r, world)
        ws = P.shard_workload(w, r, world)
        g = {k: t.cuda() for k, t in xs.items()}
        parts.append(Layer(ws)(g["q"], g["k"], g["v"]))
    torch.cuda.synchronize()
    q1m.check_status()
    got = torch.cat(parts, dim=1).cpu().numpy()
    g = {k: t.cuda() for k, t in x.items()}
    whole = Layer(w)(g["q"], g["k"], g["v"]).cpu().numpy()
    out, _, _ = O.Oracle(x["q"], x["k"], x["v"], w).run()
    ref = np.stack([out[h] for h in range(w.n_q_heads)], axis=1)
    err = np.abs(got - ref)
    rel = float(np.sum(err) / np.sum(np.abs(ref)))
    print(f"world {world}: max-abs {err.max():.2e} mean-rel {rel:.2e}, "
          f"max |sharded - whole| {np.abs(got - whole).max():.2e}")
    assert err.max() <= 2e-2 and rel <= 1e-3
    assert np.abs(got - whole).max() <= 2e-2

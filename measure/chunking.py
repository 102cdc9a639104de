"""Per-chunk timing of the chunked prefill with fixed-size chunks and with equal-cost chunks
(the pages' sizing of chunks by attention cost, here on one GPU).

    python -m measure.chunking --workload 7b-1m --chunks 8

For each mode, runs every prefill chunk through the stage kernels (the same ones the layer
runs) on the seeded synthetic inputs, times each chunk and its attention kernel with CUDA
events, counts the attended pairs from the chunk's own block masks, and prints one JSON line:
per-chunk ms, the max/mean ratio of the chunk times, and the layer total.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_prefill_dca_b200 import q1m  # noqa: E402
from long_context_prefill_dca_b200.accounting import dense_pairs, pairs_from_counts  # noqa: E402
from long_context_prefill_dca_b200.layer import Stages  # noqa: E402


def run(w, g, out):
    st = Stages(w, "bf16")
    rows = []
    for s0, e in q1m.prefill_bounds(w):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        st.keys(g["k"], g["v"], s0, e)
        st.queries(g["q"], s0, e)
        mask = resid = cnt = None
        if not w.dense:
            vert, slash = st.estimate(g["q"], s0, e)
            V, S = st.select(vert, slash, e)
            mask, resid, cnt = st.masks(V, S, s0, e)
        ev[1].record()
        st.attn(s0, e, mask, resid, cnt)
        ev[2].record()
        st.merge(s0, e, out)
        torch.cuda.synchronize()
        q1m.check_status()
        rows.append({"rows": [s0, e], "ms": ev[0].elapsed_time(ev[2]), "attn_ms": ev[1].elapsed_time(ev[2]),
                     "pairs": dense_pairs(s0, e, w.n_q_heads) if cnt is None
                     else pairs_from_counts(cnt.cpu().numpy(), s0, e)})
        del mask, resid, cnt
    del st
    torch.cuda.empty_cache()
    ms = [r["ms"] for r in rows]
    return {"chunks": rows, "total_ms": sum(ms), "max_over_mean": max(ms) / (sum(ms) / len(ms))}


def main():
    from synth import configs as C
    from synth import inputs as I
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="7b-1m")
    ap.add_argument("--chunks", type=int, default=8)
    args = ap.parse_args()
    w0 = C.BY_NAME[args.workload]
    x = I.generate(w0)
    g = {k: t.cuda() for k, t in x.items()}
    out = torch.empty(w0.seq_len, w0.n_q_heads, w0.head_dim, dtype=torch.bfloat16, device="cuda")
    fixed = w0.with_(prefill_chunk=128 * -(-w0.seq_len // (128 * args.chunks)))
    for name, w in (("fixed", fixed), ("equal-cost", w0.with_(equal_cost_chunks=args.chunks))):
        run(w, g, out)                       # warm-up (also builds the rope table)
        r = run(w, g, out)
        print(json.dumps({"workload": w0.name, "mode": name, "n_chunks": len(r["chunks"]), **r}), flush=True)


if __name__ == "__main__":
    main()

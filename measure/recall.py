"""Attention recall of the vertical-slash selection, per Q head and prefill chunk, and budget
sweeps (the measurement behind the pages' sparsity refinement: keep the sparse config's
accuracy loss small).

    python -m measure.recall --workload small-sparse [--sweep 0.5,1,2]

Runs the layer twice through the C ABI, sparse and dense, and reports
recall_i = exp(lse_sparse_i - lse_dense_i) (q1m_attention_recall): the share of each row's
dense softmax mass that its attended set keeps. Inputs are the seeded synthetic workloads.
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
from long_context_prefill_dca_b200.layer import Layer  # noqa: E402


def recall(w, g) -> torch.Tensor:
    """[Hq, N] recall of workload w on device inputs g."""
    lse_s = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    lse_d = torch.empty_like(lse_s)
    Layer(w)(g["q"], g["k"], g["v"], lse=lse_s)
    Layer(w.with_(vs_vertical=0, vs_slash=0))(g["q"], g["k"], g["v"], lse=lse_d)
    r = torch.empty_like(lse_s)
    q1m.attention_recall(lse_s, lse_d, r)
    torch.cuda.synchronize()
    q1m.check_status()
    return r


def summarize(w, r: torch.Tensor) -> dict:
    out = {"workload": w.name, "budget": [w.vs_vertical, w.vs_slash], "per_chunk": []}
    for s0, e in q1m.prefill_bounds(w):
        c = r[:, s0:e]
        out["per_chunk"].append({"rows": [s0, e], "mean": c.mean().item(), "min": c.min().item(),
                                 "per_head_mean": [round(x, 6) for x in c.mean(1).tolist()]})
    out["mean"] = r.mean().item()
    out["p01"] = torch.quantile(r.flatten()[:: max(1, r.numel() // 1_000_000)], 0.01).item()
    return out


def main():
    from synth import configs as C
    from synth import inputs as I
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="small-sparse")
    ap.add_argument("--sweep", default="1", help="comma-separated budget multipliers")
    args = ap.parse_args()
    w0 = C.BY_NAME[args.workload]
    x = I.generate(w0)
    g = {k: t.cuda() for k, t in x.items()}
    for mult in [float(v) for v in args.sweep.split(",")]:
        w = w0.with_(vs_vertical=max(0, int(w0.vs_vertical * mult)),
                     vs_slash=max(w0.vs_force_local, int(w0.vs_slash * mult)))
        print(json.dumps(summarize(w, recall(w, g))), flush=True)


if __name__ == "__main__":
    main()

"""Timing of one DCA decode step (q1m_dca_decode) at long context on the seeded inputs.

    python -m measure.decode_bench --workload 7b-1m --steps 20

Builds the fp16 cache of the first n - 1 tokens with the prefill's key rotation, then times
the decode step of the token at n - 1 (append, query views, decode kernel, merge) for a few
context lengths, called eagerly and replayed from a CUDA graph. The decode kernel is HBM-bound: its algorithmic bytes are the K and V rows
it reads, 2 x (pos + 1) x Hkv x D x 2; the roofline is the measured copy bandwidth. The K/V
read per step (2.1 GB at 1M) is far larger than L2, so no flush is needed. One JSON line per
context length.
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
from long_context_prefill_dca_b200.layer import Stages  # noqa: E402


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def main():
    from synth import configs as C
    from synth import inputs as I
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="7b-1m")
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    w = C.BY_NAME[args.workload].with_(vs_vertical=0, vs_slash=0)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    n = w.seq_len
    st = Stages(w)
    st.keys(g["k"], g["v"], 0, n - 1)
    torch.cuda.synchronize()
    peak, src = hbm_peak()
    out = torch.empty(w.n_q_heads, w.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(w.n_q_heads, device="cuda")
    for pos in sorted({n - 1, min(n - 1, 262143), min(n - 1, 131071), min(n - 1, 32767)}):
        def step():
            # the token at pos; the cache holds the prefill's rotation of rows [0, pos)
            st.decode(g["q"][pos], g["k"][pos], g["v"][pos], pos, out, lse)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        q1m.profile_enable(True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
        q1m.check_status()
        prof = q1m.profile_read()
        q1m.profile_enable(False)
        step_us = e0.elapsed_time(e1) / args.steps * 1e3
        # the same step replayed from a CUDA graph: the device-side step time without the
        # host's per-call work (argument marshalling, four launches), which dominates at
        # short contexts; a serving loop would capture the step the same way
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            step()
        torch.cuda.current_stream().wait_stream(gs)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(args.steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        q1m.check_status()
        graph_us = e0.elapsed_time(e1) / args.steps * 1e3
        del graph
        k_ms, k_n = prof["decode"]
        kern_us = k_ms / k_n * 1e3
        byts = 2.0 * (pos + 1) * w.n_kv_heads * w.head_dim * 2
        gbs = byts / (kern_us * 1e-6) / 1e9
        print(json.dumps({"workload": w.name, "context": pos + 1, "step_us": step_us,
                          "step_graph_us": graph_us, "decode_kernel_us": kern_us,
                          "kv_bytes": byts,
                          "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                                       "frac": gbs / peak, "peak_source": src},
                          "tokens_per_s_per_layer": 1e6 / step_us,
                          "tokens_per_s_per_layer_graph": 1e6 / graph_us}), flush=True)
    # restore the cache row n - 1 is not needed: the cache is discarded


if __name__ == "__main__":
    main()

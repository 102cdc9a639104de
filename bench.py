#!/usr/bin/env python
"""Benchmark of the DCA + vertical-slash chunked-prefill attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one whole layer: every prefill chunk of the 7B-shape 1,048,576-token workload
(28 Q / 4 KV heads, D = 128, bf16 inputs, RoPE base 1e7, dca_chunk 262,144, local window
4,096, YaRN s = 4, prefill chunk 131,072, budgets 2,000 columns + 12,000 diagonals) through
q1m_dca_sparse_prefill, with inputs resident in HBM (they are far larger than L2, so no
flush is needed). Prints one JSON line.

value = effective TFLOP/s of the layer: 4 * D * (number of attended (query, key) pairs, i.e.
sum of |A(i)| over rows and heads, from the layer's own block masks) / layer time.
With N GPUs every rank runs an independent replica (the layer does not shard); value is the
work of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DCA+sparse prefill attn ms/layer & effective TFLOP/s at 1M tok; % BF16 peak"
UNIT = "TFLOP/s"


KERNEL_SOURCES = ("attn_tc.cuh", "q1m_device.cuh", "exp2_poly.h")
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "block_sparse_attn_dram_7b-1m.md")


def kernel_source_hash() -> str:
    """sha256 of the attention kernel's sources with comments and blank space removed, so
    that it follows code changes only."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "long_context_prefill_dca_b200", "csrc")
    text = "".join(open(os.path.join(csrc, f)).read() for f in KERNEL_SOURCES)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha256(text.encode()).hexdigest()


def kernel_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary of the 7B@1M layer, or
    None when the workload differs or the kernel's code changed since the capture (the hash
    of its sources is recorded beside the figure)."""
    if workload != "7b-1m" or not os.path.exists(TRAFFIC_PROFILE):
        return None
    rec = {}
    for line in open(TRAFFIC_PROFILE):
        if ":" in line and line.split(":", 1)[0] in ("traffic_per_launch_bytes", "kernel_source_sha256"):
            k, v = line.split(":", 1)
            rec[k] = v.strip()
    if rec.get("kernel_source_sha256") != kernel_source_hash() or "traffic_per_launch_bytes" not in rec:
        return None
    return float(rec["traffic_per_launch_bytes"])


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="7b-1m")
    ap.add_argument("--out-dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="with N > 1 GPUs: independent replicas of the layer (weak scaling), or "
                         "the layer's KV-head groups split over the ranks (strong scaling; no "
                         "exchange inside attention, an all-gather of the output after it)")
    ap.add_argument("--equal-cost-chunks", type=int, default=0,
                    help="K > 0: K prefill chunks of equal dense attention cost instead of the "
                         "workload's fixed prefill chunk")
    return ap.parse_args()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's value (all ranks call this in the same order)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput of replicas: the work of every rank over the slowest rank's step
    time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def sum_over_ranks(value: float, world: int, device=None) -> float:
    """The sum of every rank's value (all ranks call this in the same order)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["bf16_tflops"], m["bf16_tflops_sustained"], m["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


# ---------------------------------------------------------------------------------------
# attended pairs (the work the metric counts), from the layer's own block masks
# ---------------------------------------------------------------------------------------
def attended_pairs(w, g, device):
    """(total pairs, computed-block density, per-chunk pairs) from the layer's own masks."""
    from long_context_prefill_dca_b200.accounting import attended_pairs as count
    return count(w, g, device)


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_sample(w, x, dense_pairs_total, n_rows=4):
    """Time the fp64 oracle on a bounded sample of the layer and extrapolate to the whole
    layer. Returns (seconds per layer, description, total pairs estimate)."""
    import numpy as np
    from oracle import dca_vs as O
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    h = w.n_q_heads - 1
    g = h // w.group
    chunks = list(O.prefill_chunks(w))
    s0, e = chunks[-1]
    t0 = time.perf_counter()
    orc.krot(g)
    t_krot = time.perf_counter() - t0
    t_est, density = 0.0, 1.0
    sel = O.ChunkSelection(s0, e)
    if not w.dense:
        R = O.estimator_rows(s0, e, w)
        t0 = time.perf_counter()
        vt, sl, _ = O.estimate_head(orc.q_rows(R, h), R, orc.krot(g), e, w)
        V, S = O.select_head(vt, sl, w)
        t_est = time.perf_counter() - t0
        sel.V = [None] * w.n_q_heads
        sel.S = [None] * w.n_q_heads
        sel.V[h], sel.S[h] = V, S
        nb = (e + 127) // 128
        dens = [O.computed_blocks(S, b, e)[: b + 1].mean() for b in range(s0 // 128, nb, 64)]
        density = float(np.mean(dens))
    rows = np.arange(e - n_rows, e)
    t0 = time.perf_counter()
    orc.attend_rows(rows, h, sel)
    t_att = time.perf_counter() - t0
    pairs_sample = float(sum(int(orc.attended(int(i), h, sel).sum()) for i in rows))
    pairs_total = dense_pairs_total * density
    est_rows_keys = sum(w.n_q_heads * ee for _, ee in chunks)
    t_layer = (t_att / pairs_sample * pairs_total + t_est / e * est_rows_keys +
               t_krot * w.n_kv_heads)
    desc = (f"fp64 oracle, head {h}: key rotation of 1 KV head ({t_krot:.1f}s), estimator of "
            f"the last chunk ({t_est:.1f}s), attention of the last {n_rows} rows "
            f"({t_att:.1f}s, {pairs_sample:.3g} pairs); extrapolated to the layer by pairs "
            f"(density {density:.3f}), estimator rows x keys and KV heads")
    return t_layer, desc, pairs_total


def estimator_work(w) -> dict:
    """Algorithmic work of the vertical-slash estimator over all prefill chunks: bytes (two
    passes over the fp16 key prefix, the estimator query rows, the fp32 scores written),
    tensor FLOPs (two passes of 2 * rows * keys * D per KV-group row set) and exponentials."""
    from long_context_prefill_dca_b200 import q1m
    D, hq, hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    byts = flops = exps = 0.0
    for s0, e in q1m.prefill_bounds(w):
        rows = min(w.vs_last_q, e - s0)
        byts += 2 * e * hkv * D * 2 + rows * hq * D * 2 + 2 * hq * e * 4
        flops += 2 * 2.0 * rows * hq * e * D
        exps += 2.0 * rows * hq * e
    return {"bytes": byts, "flops": flops, "exps": exps}


# ex2 results per clock per SM on the multi-function units (measured on B200 with all SMs
# busy: 15.99)
MUFU_EXP_PER_CLK_PER_SM = 16


def estimator_bounds(ew: dict, t_est: float, hbm_gbs: float, tensor_tflops: float, sms: int,
                     sm_mhz: float) -> dict:
    """The estimator's three bounds for its measured time t_est (s): HBM bytes, tensor FLOPs
    and MUFU exponentials (peak = MUFU_EXP_PER_CLK_PER_SM x SMs x SM clock), each achieved and
    as a fraction of its peak, and the HBM fraction the stage would reach if it ran exactly
    at its exponential bound: the ceiling its arithmetic sets on the HBM fraction."""
    exp_peak = MUFU_EXP_PER_CLK_PER_SM * sms * sm_mhz * 1e6      # exponentials per second
    t_exp = ew["exps"] / exp_peak
    return {"gbs": ew["bytes"] / t_est / 1e9,
            "frac_hbm": ew["bytes"] / t_est / 1e9 / hbm_gbs,
            "tflops": ew["flops"] / t_est / 1e12,
            "frac_tensor": ew["flops"] / t_est / 1e12 / tensor_tflops,
            "gexp_per_s": ew["exps"] / t_est / 1e9,
            "exp_peak_gexp_per_s": exp_peak / 1e9,
            "frac_exp": t_exp / t_est,
            "frac_hbm_at_exp_bound": ew["bytes"] / t_exp / 1e9 / hbm_gbs}


def dense_pairs(w) -> float:
    n = float(w.seq_len)
    return n * (n + 1) / 2 * w.n_q_heads


def run_reference(args):
    """The reference arm: the oracle as it stands on the host cores, bounded samples."""
    from synth import configs as C
    from synth import inputs as I
    w = C.BY_NAME[args.workload].with_(equal_cost_chunks=args.equal_cost_chunks)
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = I.generate(w)
    dp = dense_pairs(w)
    times = []
    desc, pairs = "", dp
    for it in range(args.warmup + args.steps):
        t_layer, desc, pairs = oracle_sample(w, x, dp)
        if it >= args.warmup:
            times.append(t_layer)
    t = sum(times) / len(times)
    flops = 4.0 * w.head_dim * pairs
    value = flops / t / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) + planted sinks/bands)",
            "config": {"workload": w.name, "seq_len": w.seq_len, "n_q_heads": w.n_q_heads,
                       "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import numpy as np
    import torch
    import torch.distributed as dist
    from long_context_prefill_dca_b200 import q1m
    from long_context_prefill_dca_b200.layer import HostLayer, Layer
    from synth import configs as C
    from synth import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=device)
    w = C.BY_NAME[args.workload].with_(out_dtype=args.out_dtype,
                                        equal_cost_chunks=args.equal_cost_chunks)
    q1m.library()
    sharded = args.shard == "heads" and world > 1
    w_full = w
    x = I.generate(w)
    if sharded:
        from long_context_prefill_dca_b200 import parallel as P
        x = P.shard_inputs(x, w, rank, world)
        w = P.shard_workload(w, rank, world)
    g = {k: t.to(device) for k, t in x.items()}
    pairs, density, per_chunk = attended_pairs(w, g, device)
    flops = 4.0 * w.head_dim * pairs
    layer = Layer(w, args.out_dtype, device)
    out = torch.empty(w.seq_len, w.n_q_heads, w.head_dim,
                      dtype=torch.bfloat16 if args.out_dtype == "bf16" else torch.float32,
                      device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        layer(g["q"], g["k"], g["v"], out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    q1m.check_status(stream)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.5)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    q1m.profile_enable(True)
    n0 = q1m.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    launches = q1m.launch_count() - n0
    prof = q1m.profile_read()
    q1m.profile_enable(False)
    clk = clocks.stop()
    q1m.check_status(stream)
    ms_step = max_over_ranks(ev0.elapsed_time(ev1), world, device) / args.steps
    job_flops = sum_over_ranks(flops, world, device)   # replicas: world x flops
    value = job_flops / (ms_step * 1e-3) / 1e12
    allgather_ms = None
    if sharded:
        # the only collective of the sharded layer, after attention: out over heads
        from long_context_prefill_dca_b200 import parallel as P
        dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        full = P.gather_heads(out, world)
        a1.record(stream)
        torch.cuda.synchronize(device)
        allgather_ms = max_over_ranks(a0.elapsed_time(a1), world, device)
        del full

    # e2e: the same layer through the host-buffer entry point, copies included
    e2e = None
    if args.e2e_steps > 0:
        del layer
        torch.cuda.empty_cache()
        hl = HostLayer(w, args.out_dtype, device)
        pin = {k: v.pin_memory() for k, v in x.items()}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hl(pin["q"], pin["k"], pin["v"], out_h, stream=stream)       # warm-up
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            hl(pin["q"], pin["k"], pin["v"], out_h, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, device)
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        e2e = {"value": job_flops / (ms_e2e * 1e-3) / 1e12, "unit": UNIT,
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": out_h.numel() * out_h.element_size(), "steps": args.e2e_steps}
        del hl, pin, out_h

    burst, sustained, hbm, src = peaks()
    attn_ms, attn_n = prof["attn"]
    # per launch: the timed region's attention FLOPs over its attention-kernel launches,
    # divided by the average launch duration (events on the launching stream)
    achieved = (flops * args.steps / attn_n) / (attn_ms / attn_n * 1e-3) / 1e12 if attn_n else None
    roofline = {"bound": "tensor", "kernel": "block_sparse_attn_kernel<128>",
                "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                "frac": achieved / sustained if achieved else None, "traffic": kernel_traffic(w.name),
                "traffic_unit": "DRAM bytes per launch (ncu, profiles/block_sparse_attn_dram_7b-1m.md)",
                "peak_source": f"{src} bf16 sustained (MEASURED_PEAKS.json); fp16 operands run at the bf16 rate",
                "frac_of_burst": achieved / burst if achieved else None,
                "layer_frac": value / world / sustained}
    stages = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
              for k, v in prof.items()}
    estimator = None
    if not w.dense and prof["estimate"][0] > 0:
        ew = estimator_work(w)
        t_est = prof["estimate"][0] / args.steps * 1e-3
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        estimator = {"ms_per_step": t_est * 1e3, "algorithmic_bytes": ew["bytes"],
                     **estimator_bounds(ew, t_est, hbm, sustained, sms, float(mhz)),
                     "note": "two tcgen05 passes over the key prefix; at D=128 with 7 Q heads "
                             "per KV head the exponentials, not HBM, bound it: "
                             "frac_hbm_at_exp_bound is the most HBM it can reach"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_layer, desc, cpu_pairs = oracle_sample(w, x, dense_pairs(w))
        cpu = {"value": 4.0 * w.head_dim * pairs / t_layer / 1e12, "unit": UNIT,
               "cores": blas_threads(), "kind": "oracle", "sample": desc,
               "seconds_per_layer_extrapolated": t_layer}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic (seeded N(0,1) + planted sinks/bands, bf16)",
            "config": {"workload": w.name, "seq_len": w.seq_len, "n_q_heads": w_full.n_q_heads,
                       "n_kv_heads": w_full.n_kv_heads, "head_dim": w.head_dim,
                       "heads_per_rank": [w.n_q_heads, w.n_kv_heads],
                       "dca_chunk": w.dca_chunk, "local_window": w.local_window,
                       "yarn_s": w.yarn_s, "prefill_chunk": w.prefill_chunk,
                       "chunking": (f"equal-cost x{w.equal_cost_chunks}" if w.equal_cost_chunks
                                    else "fixed"),
                       "prefill_chunks": [list(b) for b in q1m.prefill_bounds(w)],
                       "vs_budget": [w.vs_vertical, w.vs_slash], "inputs": "bf16",
                       "mma": "f16 x f16 -> f32", "out": args.out_dtype,
                       "parallelism": (f"KV-head groups split over {world} GPUs" if sharded else
                                       f"replicas x{world}" if world > 1 else "single GPU"),
                       "allgather_ms": allgather_ms,
                       "l2": "inputs (9.6 GB) far larger than L2 (126 MB); no flush",
                       "attended_pairs": job_flops / (4.0 * w.head_dim), "block_density": density,
                       "ms_per_layer": ms_step},
            "roofline": roofline, "estimator": estimator, "stages": stages,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

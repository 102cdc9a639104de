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

# DRAM traffic of one attention launch, from a one-launch ncu capture of a small case
# (dram__bytes_read.sum + dram__bytes_write.sum), with the sha256 of the kernel's sources at
# capture time: the figure is reported only while the sources still hash to it. The capture
# is the 7B-shape 131,072-token workload's last prefill chunk; the 1M-token layer is not
# captured (its launches run for seconds with tens of GB resident), so its traffic is null.
SMALL_CASE_TRAFFIC = {
    "workload": "7b-128k", "chunk": 3,
    "bytes_per_launch": 6412883000 + 1387854000,     # dram read + write, GB rounded to kB
    "kernel_source_sha256": "69979cbce8382b1df522f55bb0cd5eb94bfeec79dbde3cb0a88a5c9dd693f556",
}


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


def small_case_traffic():
    """The small case's DRAM bytes per attention launch while the kernel is unchanged since
    its capture, else None."""
    t = SMALL_CASE_TRAFFIC
    if t["bytes_per_launch"] is None or t["kernel_source_sha256"] != kernel_source_hash():
        return None
    return t["bytes_per_launch"]


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


FULL_ORACLE_ROWS = 1 << 14    # rows x heads up to which the oracle runs the whole layer


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, x, dense_pairs_total, n_heads=4, rows_per_head=16, orc=None, t_krot=None):
    """Time the fp64 oracle, as it stands, on a bounded sample of the layer and extrapolate to
    the whole layer. The sample: the key rotation of the last KV group, the estimator and
    selection of the last prefill chunk for `n_heads` Q heads of that group, and the attention
    of the last `rows_per_head` rows of each of those heads. The layer estimate scales the
    attention time by attended pairs (the sampled heads' block density applied to every row),
    the estimator time by estimator rows x keys over all chunks, and the rotation by KV heads.
    `orc` / `t_krot` reuse an oracle whose rotated keys are already computed and the time that
    took (the reference arm's later steps). Returns a dict."""
    import numpy as np
    from oracle import dca_vs as O
    if w.seq_len * w.n_q_heads <= FULL_ORACLE_ROWS:
        # small enough for the whole layer: no extrapolation
        t0 = time.perf_counter()
        O.Oracle(x["q"], x["k"], x["v"], w).run()
        t = time.perf_counter() - t0
        return {"t_layer": t, "sample_s": t, "pairs_total": dense_pairs_total if w.dense else None,
                "desc": f"fp64 oracle (numpy), the whole layer: every row of every head ({t:.1f} s)",
                "orc": None, "t_krot": None, "extrapolated": False}
    g = w.n_kv_heads - 1
    heads = [g * w.group + i for i in range(min(n_heads, w.group))]
    sample_t0 = time.perf_counter()
    if orc is None:
        orc = O.Oracle(x["q"], x["k"], x["v"], w)
    if t_krot is None:
        t0 = time.perf_counter()
        orc.krot(g)
        t_krot = time.perf_counter() - t0
    chunks = list(O.prefill_chunks(w))
    s0, e = chunks[-1]
    t_est, density = 0.0, 1.0
    sel = O.ChunkSelection(s0, e)
    if not w.dense:
        R = O.estimator_rows(s0, e, w)
        sel.V = [None] * w.n_q_heads
        sel.S = [None] * w.n_q_heads
        dens = []
        t0 = time.perf_counter()
        for h in heads:
            vt, sl, _ = O.estimate_head(orc.q_rows(R, h), R, orc.krot(g), e, w)
            sel.V[h], sel.S[h] = O.select_head(vt, sl, w)
        t_est = time.perf_counter() - t0
        nb = (e + 127) // 128
        for h in heads:
            dens += [O.computed_blocks(sel.S[h], b, e)[: b + 1].mean() for b in range(s0 // 128, nb, 64)]
        density = float(np.mean(dens))
    rows = np.arange(e - rows_per_head, e)
    t0 = time.perf_counter()
    for h in heads:
        orc.attend_rows(rows, h, sel)
    t_att = time.perf_counter() - t0
    sample_s = time.perf_counter() - sample_t0
    pairs_sample = float(sum(int(orc.attended(int(i), h, sel).sum()) for h in heads for i in rows))
    pairs_total = dense_pairs_total * density
    est_rows_keys = sum(w.n_q_heads * ee for _, ee in chunks)
    t_layer = (t_att / pairs_sample * pairs_total + t_est / (len(heads) * e) * est_rows_keys +
               t_krot * w.n_kv_heads)
    desc = (f"fp64 oracle (numpy; BLAS matmuls threaded, the rest on one core), KV group {g}: key "
            f"rotation ({t_krot:.1f} s), estimator + selection of the last prefill chunk for Q "
            f"heads {heads} ({t_est:.1f} s), attention of the last {rows_per_head} rows of each "
            f"({t_att:.1f} s, {pairs_sample:.3g} pairs); extrapolated to the layer by attended "
            f"pairs (block density {density:.3f}), estimator rows x keys and KV heads")
    return {"t_layer": t_layer, "sample_s": sample_s, "desc": desc, "pairs_total": pairs_total,
            "orc": orc, "t_krot": t_krot, "pairs_sample": pairs_sample, "extrapolated": True}


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


L2_FLUSH_BYTES = 512 << 20    # written between timed steps when the inputs are smaller


def config_of(w, args, world=1, w_full=None, sharded=False) -> dict:
    """The workload description both arms print."""
    from long_context_prefill_dca_b200 import q1m
    w_full = w_full or w
    in_bytes = (w.seq_len * (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim *
                (2 if w.in_dtype == "bf16" else 4))
    return {"workload": w.name, "seq_len": w.seq_len, "n_q_heads": w_full.n_q_heads,
            "n_kv_heads": w_full.n_kv_heads, "head_dim": w.head_dim,
            "heads_per_rank": [w.n_q_heads, w.n_kv_heads],
            "dca_chunk": w.dca_chunk, "local_window": w.local_window,
            "yarn_s": w.yarn_s, "prefill_chunk": w.prefill_chunk,
            "chunking": (f"equal-cost x{w.equal_cost_chunks}" if w.equal_cost_chunks else "fixed"),
            "prefill_chunks": [list(b) for b in q1m.prefill_bounds(w)],
            "vs_budget": [w.vs_vertical, w.vs_slash], "inputs": w.in_dtype,
            "mma": "f16 x f16 -> f32 (rotated, scaled Q and K beyond +-65,504 are refused "
                   "with Q1M_ERR_RANGE)",
            "out": args.out_dtype,
            "parallelism": (f"KV-head groups split over {world} GPUs" if sharded else
                            f"replicas x{world}" if world > 1 else "single GPU"),
            "l2": (f"inputs ({in_bytes / 1e9:.2f} GB) larger than L2 (126 MB); no flush"
                   if in_bytes >= L2_FLUSH_BYTES else
                   f"inputs ({in_bytes / 1e6:.1f} MB) within L2: a {L2_FLUSH_BYTES >> 20} MiB "
                   "buffer is written between timed steps, each step timed on its own")}


def run_reference(args):
    """The reference arm: the oracle as it stands on the host cores. Each step times one
    bounded sample of the workload (the first step also rotates the sampled KV group's keys,
    which later steps reuse); value is the layer's attention FLOPs over the layer time
    extrapolated from that sample."""
    from synth import configs as C
    from synth import inputs as I
    w = C.BY_NAME[args.workload].with_(equal_cost_chunks=args.equal_cost_chunks,
                                        out_dtype=args.out_dtype)
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = I.generate(w)
    dp = dense_pairs(w)
    layer_s, sample_s = [], []
    orc, t_krot, res = None, None, None
    for it in range(args.warmup + args.steps):
        res = oracle_sample(w, x, dp, n_heads=1, rows_per_head=4, orc=orc, t_krot=t_krot)
        orc, t_krot = res["orc"], res["t_krot"]
        if it >= args.warmup:
            layer_s.append(res["t_layer"])
            sample_s.append(res["sample_s"])
    t = sum(layer_s) / len(layer_s)
    if res["pairs_total"] is None:   # the whole sparse layer ran: count its attended pairs
        from oracle import dca_vs as O
        orc = O.Oracle(x["q"], x["k"], x["v"], w)
        res["pairs_total"] = float(sum(int(orc.attended(i, h, sel).sum())
                                       for sel in (orc.select_chunk(a, b) for a, b in O.prefill_chunks(w))
                                       for h in range(w.n_q_heads) for i in range(sel.s0, sel.e)))
    flops = 4.0 * w.head_dim * res["pairs_total"]
    value = flops / t / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sum(sample_s) / len(sample_s) * 1e3,
            "ms_per_layer_extrapolated": t * 1e3 if res["extrapolated"] else None,
            "extrapolated": res["extrapolated"],
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) + planted sinks/bands)",
            "config": config_of(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "host_cores": host_cores(), "kind": "oracle",
                             "extrapolated": res["extrapolated"],
                             "sample_seconds": sum(sample_s) / len(sample_s),
                             "sample": res["desc"] + "; ms_per_step is one sample's measured time"},
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
    in_bytes = sum(t.numel() * t.element_size() for t in g.values())
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device) if in_bytes < L2_FLUSH_BYTES else None

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
    if flush is None:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(device)
        ms_total = ev0.elapsed_time(ev1)
    else:
        # inputs that fit in L2: each step is timed on its own, after a write of a buffer
        # larger than L2 that evicts the previous step's data
        evs = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(device)
        ms_total = sum(a.elapsed_time(b) for a, b in evs)
    if world > 1:
        dist.barrier()
    launches = q1m.launch_count() - n0
    prof = q1m.profile_read()
    q1m.profile_enable(False)
    clk = clocks.stop()
    q1m.check_status(stream)
    ms_step = max_over_ranks(ms_total, world, device) / args.steps
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
    t_small = small_case_traffic()
    roofline = {"bound": "tensor", "kernel": f"block_sparse_attn_kernel<{w.head_dim}>",
                "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                "frac": achieved / sustained if achieved else None,
                "traffic": t_small if w.name == SMALL_CASE_TRAFFIC["workload"] else None,
                "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + "
                                "dram__bytes_write.sum, one launch of the small case)",
                "traffic_small_case": {"workload": SMALL_CASE_TRAFFIC["workload"],
                                       "prefill_chunk": SMALL_CASE_TRAFFIC["chunk"],
                                       "bytes_per_launch": t_small},
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
        res = oracle_sample(w, x, dense_pairs(w))
        cpu = {"value": 4.0 * w.head_dim * pairs / res["t_layer"] / 1e12, "unit": UNIT,
               "cores": blas_threads(), "host_cores": host_cores(), "kind": "oracle",
               "extrapolated": res["extrapolated"], "sample_seconds": res["sample_s"],
               "sample": res["desc"], "seconds_per_layer": res["t_layer"]}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic (seeded N(0,1) + planted sinks/bands, bf16)",
            "config": {**config_of(w, args, world, w_full, sharded),
                       "allgather_ms": allgather_ms,
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

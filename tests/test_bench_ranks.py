"""The benchmark's multi-rank logic on CPU: two gloo ranks, max-over-ranks timing and the
whole-job throughput; the reference arm prints only on rank 0."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    ms = [120.0, 95.0][rank]               # rank 0 is the slower one
    slow = bench.max_over_ranks(ms, world)
    # head-sharded runs: each rank counts its own shard's work; the job sums them
    shard_flops = [3e14, 5e14][rank]
    q.put((rank, slow, bench.job_tflops(1e15, world, slow), bench.sum_over_ranks(shard_flops, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slow, tf, total in res:
        assert slow == 120.0
        assert tf == pytest.approx(1e15 * 2 / 0.120 / 1e12)
        assert total == pytest.approx(8e14)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_tflops(2e12, 1, 1000.0) == pytest.approx(2.0)
    assert bench.sum_over_ranks(3.5, 1) == 3.5


def test_reference_arm_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny-dense-2k", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "small-sparse", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_small_case_traffic_tracks_the_capture(monkeypatch):
    """The roofline traffic figure is the small case's capture, reported only while the
    attention kernel's sources hash to the value recorded with it."""
    import bench
    monkeypatch.setitem(bench.SMALL_CASE_TRAFFIC, "bytes_per_launch", 123.0)
    monkeypatch.setitem(bench.SMALL_CASE_TRAFFIC, "kernel_source_sha256", "00")
    assert bench.small_case_traffic() is None
    monkeypatch.setitem(bench.SMALL_CASE_TRAFFIC, "kernel_source_sha256", bench.kernel_source_hash())
    assert bench.small_case_traffic() == 123.0
    monkeypatch.setitem(bench.SMALL_CASE_TRAFFIC, "bytes_per_launch", None)
    assert bench.small_case_traffic() is None


def test_estimator_bounds_identities_and_ceiling():
    """The estimator's reported bounds are consistent (frac_hbm = frac_exp x the HBM
    fraction at the exponential bound; frac_exp = achieved / peak exponential rate), and at
    the 7B shape its exponentials cap its HBM fraction near 0.45: per key and chunk it reads
    2 passes x 4 KV heads x 128 x 2 bytes = 2,048 bytes and writes 2 x 28 x 4 = 224 bytes of
    scores, and computes 2 x 64 x 28 = 3,584 exponentials; 16 exponentials per clock on 148
    SMs at 1,965 MHz against 6,538.9 GB/s give 2272 / 3584 x 4.653e12 / 6.5389e12 = 0.451."""
    import bench
    from synth import configs as C
    ew = bench.estimator_work(C.L7B_1M)
    b = bench.estimator_bounds(ew, 27.3e-3, 6538.9, 1402.6, 148, 1965.0)
    assert abs(b["frac_hbm"] - b["frac_exp"] * b["frac_hbm_at_exp_bound"]) < 1e-12
    assert abs(b["frac_exp"] - b["gexp_per_s"] / b["exp_peak_gexp_per_s"]) < 1e-12
    assert abs(b["exp_peak_gexp_per_s"] - 16 * 148 * 1.965) < 1e-6
    assert 0.445 < b["frac_hbm_at_exp_bound"] < 0.455, b["frac_hbm_at_exp_bound"]
    assert 0.0 < b["frac_exp"] < 1.0 and 0.0 < b["frac_hbm"] < b["frac_hbm_at_exp_bound"]

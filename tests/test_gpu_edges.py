"""Edge cases of the CUDA path against the fp64 oracle: sequences shorter than one tile,
one prefill chunk or 128-row chunks, a zero local window, one Q head per KV head, budgets at
or above the candidate count, a slash-only budget, few estimator rows, s < 1, ragged tails;
the host-buffer entry point; the device-side range check."""
import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import HostLayer, Layer
from oracle import dca_vs as O
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_REL = 2e-2, 1e-3

BASE = C.Workload(name="edge", seq_len=700, n_q_heads=4, n_kv_heads=2, head_dim=128,
                  in_dtype="bf16", rope_base=1e4, dca_chunk=384, local_window=128, yarn_s=2.0,
                  prefill_chunk=256, vs_vertical=20, vs_slash=70, sinks=4, bands=2,
                  band_hi=300, seed=0x5EED0100)

EDGES = [
    BASE.with_(name="seq1-dense", seq_len=1, vs_vertical=0, vs_slash=0, sinks=0, bands=0),
    BASE.with_(name="seq5-sparse", seq_len=5, sinks=0, bands=0),
    BASE.with_(name="seq100-sparse", seq_len=100, sinks=2, bands=0),
    BASE.with_(name="seq128-exact", seq_len=128, bands=0),
    BASE.with_(name="one-chunk", prefill_chunk=1024),
    BASE.with_(name="chunk128", prefill_chunk=128),
    BASE.with_(name="window0", local_window=0, dca_chunk=256),
    BASE.with_(name="mha-d64", n_q_heads=3, n_kv_heads=3, head_dim=64, in_dtype="f32"),
    BASE.with_(name="gqa7", n_q_heads=7, n_kv_heads=1, seq_len=520),
    BASE.with_(name="full-budget", vs_vertical=10**6, vs_slash=10**6),
    BASE.with_(name="slash-only", vs_vertical=0, vs_slash=40),
    BASE.with_(name="last-q-16", vs_last_q=16, vs_force_local=8),
    BASE.with_(name="no-yarn", yarn_s=0.5),
    BASE.with_(name="ragged-many", seq_len=1111, prefill_chunk=384),
    BASE.with_(name="equal-cost-4", seq_len=1500, equal_cost_chunks=4),
    BASE.with_(name="equal-cost-dense", seq_len=900, equal_cost_chunks=3, vs_vertical=0, vs_slash=0),
]


def oracle_out(w, x):
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    out, lse, _ = orc.run()
    return (np.stack([out[h] for h in range(w.n_q_heads)], axis=1),
            np.stack([lse[h] for h in range(w.n_q_heads)], axis=0))


def rel(a, b):
    return float(np.sum(np.abs(a - b)) / max(np.sum(np.abs(b)), 1e-30))


@pytest.mark.parametrize("w", EDGES, ids=lambda w: w.name)
def test_edge_case_matches_oracle(w):
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    lse = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    out = Layer(w)(g["q"], g["k"], g["v"], lse=lse)
    torch.cuda.synchronize()
    q1m.check_status()
    ref, ref_lse = oracle_out(w, x)
    got = out.cpu().numpy()
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref)
    print(f"{w.name}: max-abs {err.max():.2e} mean-rel {rel(got, ref):.2e}")
    assert err.max() <= MAX_ABS and rel(got, ref) <= MEAN_REL
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


HOST_CASES = [BASE, BASE.with_(name="host-ragged-many", seq_len=1111, prefill_chunk=128),
              BASE.with_(name="host-equal-cost", seq_len=1500, equal_cost_chunks=3),
              BASE.with_(name="host-one-chunk", prefill_chunk=1024)]


@pytest.mark.parametrize("w", HOST_CASES, ids=lambda w: w.name)
def test_host_buffer_entry_point_matches_device_entry_point(deterministic, w):
    """The host-buffer path uploads and downloads chunk by chunk on its own copy streams;
    its out and lse equal the device path's bit for bit."""
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    lse_d = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    dev = Layer(w)(g["q"], g["k"], g["v"], lse=lse_d).cpu()
    pin = {k: v.pin_memory() for k, v in x.items()}
    out_h = torch.full(dev.shape, float("nan"), dtype=dev.dtype).pin_memory()
    lse_h = torch.full((w.n_q_heads, w.seq_len), float("nan")).pin_memory()
    HostLayer(w)(pin["q"], pin["k"], pin["v"], out_h, lse_h)
    assert torch.equal(out_h, dev)
    assert torch.equal(lse_h, lse_d.cpu())
    # a second call on a side stream, with other inputs queued on it first, gives the same
    x2 = I.generate(w.with_(seed=w.seed + 1))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        junk = torch.empty(64 << 20, dtype=torch.uint8, device="cuda").fill_(7)   # queued work
        HostLayer(w)(*(x2[k].pin_memory() for k in ("q", "k", "v")), out_h, lse_h,
                     stream=s.cuda_stream)
    ref2 = Layer(w)(*(x2[k].cuda() for k in ("q", "k", "v"))).cpu()
    assert torch.equal(out_h, ref2)
    del junk


def test_fp16_range_overflow_is_reported():
    """Keys far beyond fp16 range latch Q1M_ERR_RANGE in the rotation stage."""
    w = BASE.with_(vs_vertical=0, vs_slash=0)
    x = I.generate(w)
    x["k"][3, 0, 5] = 1e30 if w.in_dtype == "f32" else torch.tensor(3e38).to(torch.bfloat16)
    g = {k: t.cuda() for k, t in x.items()}
    Layer(w)(g["q"], g["k"], g["v"])
    assert q1m.status_poll() == -6
    assert q1m.status_poll() == 0          # the latch clears on read


def test_nan_score_is_reported():
    w = BASE
    vert = torch.rand(w.n_q_heads, 300, device="cuda")
    slash = torch.rand(w.n_q_heads, 300, device="cuda")
    vert[1, 17] = float("nan")
    V = torch.empty(w.n_q_heads, w.vs_vertical, dtype=torch.int32, device="cuda")
    S = torch.empty(w.n_q_heads, w.vs_slash, dtype=torch.int32, device="cuda")
    q1m.vs_select(vert, slash, 300, 300, w.n_q_heads, q1m.params(w), V, S)
    assert q1m.status_poll() == -6
    assert q1m.status_poll() == 0


def test_prefill_resumed_at_chunk_granularity(deterministic):
    """Chunks [0, 2) then [2, end) on the same workspace equal one call, bit for bit."""
    w = BASE.with_(seq_len=1111, prefill_chunk=256)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    layer = Layer(w)
    whole = layer(g["q"], g["k"], g["v"]).clone()
    lse_whole = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    layer(g["q"], g["k"], g["v"], lse=lse_whole)
    out = torch.full_like(whole, float("nan"))
    lse = torch.full_like(lse_whole, float("nan"))
    layer2 = Layer(w)
    layer2.chunks(g["q"], g["k"], g["v"], 0, 2, out, lse)
    torch.cuda.synchronize()
    assert torch.isnan(out[512:]).all() and not torch.isnan(out[:512]).any()
    layer2.chunks(g["q"], g["k"], g["v"], 2, 1 << 40, out, lse)
    torch.cuda.synchronize()
    q1m.check_status()
    assert torch.equal(out, whole) and torch.equal(lse, lse_whole)


def test_repeated_runs_default_and_deterministic():
    """Deterministic mode: repeated runs are bit-identical. Default mode (key-block walks
    aligned to a global tile count): repeated runs agree at the level of the fp16 rounding
    of P (the running maximum it is rounded against follows the tile order), and with the
    deterministic run."""
    w = BASE.with_(seq_len=1500)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    q1m.set_deterministic(True)
    try:
        a = Layer(w)(g["q"], g["k"], g["v"])
        b = Layer(w)(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        assert torch.equal(a, b)
    finally:
        q1m.set_deterministic(False)
    c = Layer(w)(g["q"], g["k"], g["v"])
    d = Layer(w)(g["q"], g["k"], g["v"])
    torch.cuda.synchronize()
    q1m.check_status()
    # one fp16 ulp of a P element that carries half of a row's mass moves an output by up to
    # ~5e-4 |v - out|, so the run-to-run bound is 5e-3 absolute (a quarter of the parity
    # tolerance) and 5e-4 relative in sum
    for u in (d, a):
        diff = (c - u).abs()
        assert diff.max().item() <= 5e-3 and diff.sum().item() <= 5e-4 * c.abs().sum().item()


def test_host_path_bf16_out_without_lse_and_pageable_buffers(deterministic):
    """bf16 output with lse left out, from pinned and from pageable host buffers."""
    w = BASE.with_(seq_len=900)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    dev = Layer(w, "bf16")(g["q"], g["k"], g["v"]).cpu()
    for pinned in (True, False):
        src = {k: (t.pin_memory() if pinned else t.clone()) for k, t in x.items()}
        out_h = torch.zeros(dev.shape, dtype=torch.bfloat16)
        if pinned:
            out_h = out_h.pin_memory()
        HostLayer(w, "bf16")(src["q"], src["k"], src["v"], out_h, None)
        assert torch.equal(out_h, dev), pinned


def test_layer_replays_from_a_cuda_graph(deterministic):
    """The whole layer (every prefill chunk's stages) captured into one CUDA graph: a replay
    equals an eager call bit for bit, and new inputs copied into the captured buffers give
    the new result."""
    w = BASE.with_(seq_len=1111, prefill_chunk=256)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    layer = Layer(w)
    eager = layer(g["q"], g["k"], g["v"]).clone()
    out = torch.empty_like(eager)
    lse = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer(g["q"], g["k"], g["v"], out=out, lse=lse)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        layer(g["q"], g["k"], g["v"], out=out, lse=lse)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    q1m.check_status()
    assert torch.equal(out, eager)
    x2 = I.generate(w.with_(seed=w.seed + 7))
    for k in ("q", "k", "v"):
        g[k].copy_(x2[k].cuda())
    graph.replay()
    torch.cuda.synchronize()
    q1m.check_status()
    ref2 = Layer(w)(g["q"], g["k"], g["v"])
    assert torch.equal(out, ref2)
    del graph

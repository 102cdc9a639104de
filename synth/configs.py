"""Workload definitions for the DCA + vertical-slash chunked-prefill attention layer.

These are plain data: the shapes, RoPE/DCA/YaRN settings, prefill chunk and sparse
budgets of each synthetic workload, plus the small parity cases used by the tests.
No arithmetic of the method lives here.

The five named workloads follow the layer shapes the Qwen2.5-1M pages give
(Qwen2.5-1M Technical Report review, section 三 "model architecture" table:
7B = 28 Q / 4 KV heads, 14B = 40 Q / 8 KV heads; RoPE base schedule 1e4 -> 1e7;
deployment page "Deploy Qwen2.5-1M Models Locally": max model length 1,010,000 and
a chunked-prefill chunk of 131,072 tokens; "Sparse Attention": chunk 32,768).
"""
from __future__ import annotations

from dataclasses import dataclass, replace, asdict


@dataclass(frozen=True)
class Workload:
    name: str
    seq_len: int          # N
    n_q_heads: int        # Hq
    n_kv_heads: int       # Hkv
    head_dim: int         # D
    in_dtype: str         # "bf16" or "f32"
    rope_base: float
    dca_chunk: int        # c: the trained length; a DCA chunk holds c - w tokens
    local_window: int     # w
    yarn_s: float         # inference / training length ratio (<= 1: no scaling)
    prefill_chunk: int    # P: query rows per chunked-prefill step
    vs_vertical: int      # vertical (column) budget per head; 0 and 0 => dense
    vs_slash: int         # slash (diagonal) budget per head
    vs_last_q: int = 64   # estimator rows: the last rows of each prefill chunk
    vs_force_local: int = 64  # diagonals 0 .. vs_force_local-1 always kept
    sinks: int = 0        # planted sink columns per KV head
    bands: int = 0        # planted diagonal bands per KV head
    band_lo: int = 128    # band offsets drawn uniformly in [band_lo, band_hi)
    band_hi: int = 65536
    seed: int = 0
    out_dtype: str = "f32"
    equal_cost_chunks: int = 0  # K > 0: K prefill chunks of equal dense attention cost

    @property
    def dense(self) -> bool:
        return self.vs_vertical == 0 and self.vs_slash == 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def as_dict(self) -> dict:
        return asdict(self)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


SEED_BASE = 0x5EED0000

# The five workloads of the benchmark suite, in order.
TINY_2K = Workload(
    name="tiny-dense-2k", seq_len=2048, n_q_heads=2, n_kv_heads=1, head_dim=64,
    in_dtype="f32", rope_base=1e4, dca_chunk=512, local_window=128, yarn_s=1.0,
    prefill_chunk=2048, vs_vertical=0, vs_slash=0, seed=SEED_BASE + 0)

L7B_128K = Workload(
    name="7b-128k", seq_len=131072, n_q_heads=28, n_kv_heads=4, head_dim=128,
    in_dtype="bf16", rope_base=1e6, dca_chunk=32768, local_window=1024, yarn_s=4.0,
    prefill_chunk=32768, vs_vertical=1000, vs_slash=6096, sinks=16, bands=0,
    seed=SEED_BASE + 1)

L14B_256K = Workload(
    name="14b-256k", seq_len=262144, n_q_heads=40, n_kv_heads=8, head_dim=128,
    in_dtype="bf16", rope_base=1e7, dca_chunk=65536, local_window=2048, yarn_s=4.0,
    prefill_chunk=32768, vs_vertical=1000, vs_slash=6096, sinks=16, bands=8,
    seed=SEED_BASE + 2)

L7B_1M = Workload(
    name="7b-1m", seq_len=1048576, n_q_heads=28, n_kv_heads=4, head_dim=128,
    in_dtype="bf16", rope_base=1e7, dca_chunk=262144, local_window=4096, yarn_s=4.0,
    prefill_chunk=131072, vs_vertical=2000, vs_slash=12000, sinks=16, bands=8,
    seed=SEED_BASE + 3)

L14B_1M = Workload(
    name="14b-1.01m", seq_len=1010000, n_q_heads=40, n_kv_heads=8, head_dim=128,
    in_dtype="bf16", rope_base=1e7, dca_chunk=262144, local_window=4096, yarn_s=3.85,
    prefill_chunk=131072, vs_vertical=2000, vs_slash=12000, sinks=16, bands=8,
    seed=SEED_BASE + 4)

SUITE = [TINY_2K, L7B_128K, L14B_256K, L7B_1M, L14B_1M]
BY_NAME = {w.name: w for w in SUITE}

# Small parity cases: sizes the oracle finishes in seconds that still span several
# 128-row tiles, several DCA chunks, several prefill chunks and a ragged tail.
SMALL_SPARSE = Workload(
    name="small-sparse", seq_len=3000, n_q_heads=4, n_kv_heads=2, head_dim=128,
    in_dtype="bf16", rope_base=1e6, dca_chunk=1024, local_window=128, yarn_s=2.93,
    prefill_chunk=1024, vs_vertical=80, vs_slash=110, sinks=16, bands=4,
    band_hi=1500, seed=SEED_BASE + 10)

SMALL_DENSE_D128 = Workload(
    name="small-dense-d128", seq_len=1700, n_q_heads=3, n_kv_heads=1, head_dim=128,
    in_dtype="bf16", rope_base=1e4, dca_chunk=640, local_window=128, yarn_s=2.66,
    prefill_chunk=768, vs_vertical=0, vs_slash=0, sinks=4, seed=SEED_BASE + 11)

SMALL_SPARSE_D64 = Workload(
    name="small-sparse-d64", seq_len=2500, n_q_heads=6, n_kv_heads=2, head_dim=64,
    in_dtype="f32", rope_base=1e4, dca_chunk=768, local_window=256, yarn_s=3.26,
    prefill_chunk=1280, vs_vertical=40, vs_slash=90, sinks=8, bands=2,
    band_hi=1200, seed=SEED_BASE + 12)

SMALL = [SMALL_SPARSE, SMALL_DENSE_D128, SMALL_SPARSE_D64]
for _w in SMALL:
    BY_NAME[_w.name] = _w

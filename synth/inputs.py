"""Seeded synthetic inputs (q, k, v) for one attention layer.

This module only draws random numbers; it holds none of the method's arithmetic.
Both the CUDA path (tests, bench) and the fp64 oracle take their inputs from here.

Recipe (the pages measure on passkey / RULER / LV-Eval, which need trained weights
and datasets; these seeded inputs stand in for them):

* base values: q [N, Hq, D], k and v [N, Hkv, D] i.i.d. N(0, 1), drawn in float32
  from counter-based Philox streams (one stream per tensor and 8192-token block, so
  blocks can be drawn in parallel and any block can be redrawn on its own);
* sinks: per KV head g, ``sinks`` distinct columns j_m uniform over [0, N) and a unit
  vector u_g; k[j_m, g] += 4 u_g and q[i, h] += u_g for every row i and every Q head
  h of group g (all before RoPE);
* bands: per KV head g, ``bands`` distinct offsets o_b uniform in [band_lo, band_hi)
  and per-position unit vectors r_{g,i}; q[i, h in g] += r_{g,i} and
  k[i - o_b, g] += 4 r_{g,i} for every i >= o_b;
* the float32 result is rounded to nearest-even into the workload's input dtype.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

BLOCK_TOKENS = 8192
_TAG = {"q": 1, "k": 2, "v": 3, "sink": 4, "band": 5, "bandvec": 6, "rows": 7}


def _rng(seed: int, tag: str, sub: int = 0) -> np.random.Generator:
    # Philox-4x64 (Salmon et al., SC'11) keyed by (seed, tag, sub): independent streams.
    key = [np.uint64(seed) & np.uint64(0xFFFFFFFFFFFFFFFF),
           np.uint64((_TAG[tag] << 40) | (sub & 0xFFFFFFFFFF))]
    return np.random.Generator(np.random.Philox(key=key))


def _unit_rows(g: np.random.Generator, n: int, d: int) -> np.ndarray:
    x = g.standard_normal((n, d), dtype=np.float64)
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    return x.astype(np.float32)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _normal_tensor(seed: int, tag: str, n: int, h: int, d: int) -> np.ndarray:
    out = np.empty((n, h, d), dtype=np.float32)
    nblk = (n + BLOCK_TOKENS - 1) // BLOCK_TOKENS

    def fill(b: int) -> None:
        t0, t1 = b * BLOCK_TOKENS, min(n, (b + 1) * BLOCK_TOKENS)
        out[t0:t1] = _rng(seed, tag, b).standard_normal((t1 - t0, h, d), dtype=np.float32)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(nblk)))
    return out


def plants(w) -> dict:
    """The planted structure of workload ``w`` (sink columns, band offsets)."""
    res = {"sink_cols": [], "band_offsets": []}
    for g in range(w.n_kv_heads):
        if w.sinks:
            r = _rng(w.seed, "sink", g)
            res["sink_cols"].append(np.sort(r.choice(w.seq_len, size=w.sinks, replace=False)))
        if w.bands:
            r = _rng(w.seed, "band", g)
            hi = min(w.band_hi, w.seq_len)
            res["band_offsets"].append(
                np.sort(r.choice(np.arange(w.band_lo, hi), size=w.bands, replace=False)))
    return res


def generate(w, rows: slice | None = None) -> dict:
    """Return {"q", "k", "v"} as CPU torch tensors in the workload's input dtype.

    q is [N, Hq, D]; k and v are [N, Hkv, D]; all token-major and contiguous.
    """
    n, hq, hkv, d, G = w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.group
    q = _normal_tensor(w.seed, "q", n, hq, d)
    k = _normal_tensor(w.seed, "k", n, hkv, d)
    v = _normal_tensor(w.seed, "v", n, hkv, d)
    pl = plants(w)
    for g in range(hkv):
        hs = slice(g * G, (g + 1) * G)
        if w.sinks:
            u = _unit_rows(_rng(w.seed, "sink", 1000 + g), 1, d)[0]
            k[pl["sink_cols"][g], g, :] += 4.0 * u
            q[:, hs, :] += u[None, None, :]
        if w.bands:
            r = np.empty((n, d), dtype=np.float32)
            nblk = (n + BLOCK_TOKENS - 1) // BLOCK_TOKENS

            def fill(b: int, g=g, r=r) -> None:
                t0, t1 = b * BLOCK_TOKENS, min(n, (b + 1) * BLOCK_TOKENS)
                r[t0:t1] = _unit_rows(_rng(w.seed, "bandvec", (g << 24) | b), t1 - t0, d)

            with ThreadPoolExecutor(_threads()) as ex:
                list(ex.map(fill, range(nblk)))
            q[:, hs, :] += r[:, None, :]
            for o in pl["band_offsets"][g]:
                o = int(o)
                k[: n - o, g, :] += 4.0 * r[o:, :]
            del r
    dt = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    out = {}
    for name, arr in (("q", q), ("k", k), ("v", v)):
        t = torch.from_numpy(arr)
        out[name] = t.to(dt) if dt != torch.float32 else t
    return out


def sample_rows(w, count: int, seed: int = 0x51A3) -> np.ndarray:
    """(token, head) pairs for sampled parity checks at full size.

    ``count`` tokens uniform without replacement, each with one Q head drawn uniformly,
    plus the first and the last row of every prefill chunk (head chosen the same way).
    Returned sorted by (head, token) as an int64 array of shape [M, 2].
    """
    g = _rng(seed, "rows", w.seq_len)
    count = min(count, w.seq_len)
    toks = g.choice(w.seq_len, size=count, replace=False)
    edges = []
    for s0 in range(0, w.seq_len, w.prefill_chunk):
        e = min(w.seq_len, s0 + w.prefill_chunk)
        edges += [s0, e - 1]
    toks = np.concatenate([toks, np.array(edges, dtype=np.int64)])
    heads = g.integers(0, w.n_q_heads, size=toks.shape[0])
    pairs = np.unique(np.stack([heads, toks], axis=1), axis=0)
    return pairs[:, [1, 0]][np.lexsort((pairs[:, 1], pairs[:, 0]))].astype(np.int64)

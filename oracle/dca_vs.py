"""fp64 CPU oracle: Dual Chunk Attention + YaRN scaling + vertical-slash sparse attention
under chunked prefill, for one GQA attention layer.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this module. It shares no code with the CUDA
library and imports nothing from it. Plain numpy float64; a matmul is the only library
step; no blocking, fusion or reordering beyond the definitions below.

Sources (page title, section):
  [P2]  "Qwen2.5-1M Technical Report" paper review (xllm-io), section 三 model architecture
        (GQA head counts, RoPE), section 四 inference and deployment optimisation:
        "Dual Chunk Attention (DCA)" (three patterns, Figure 2 caption: relative positions
        remapped to small values), "YaRN 注意力缩放" (the logit-scale formula),
        "稀疏注意力机制" (MInference vertical-slash, Figure 4 caption: key tokens chosen
        per prefill chunk, continuous relative positions).
  [P5]  "Qwen2.5-1M リリース" (agentlenshq), "Sparse Attention" (chunked prefill, chunk
        32,768) and "Deploy Qwen2.5-1M Models Locally" (chunk 131,072 via
        --max-num-batched-tokens).
Readings where the pages leave a step open are marked READING.

Every function here is pinned by tests in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

INTRA, SUCC, INTER = 0, 1, 2
BLOCK = 128  # mask block size (READING: 128 x 128 blocks)


# ----------------------------------------------------------------------------------------
# YaRN logit scale  [P2 section 四, "YaRN 注意力缩放": softmax(q^T k / (t sqrt(D))) with
# sqrt(1/t) = 0.1 ln(s) + 1, s = inference length / training length]
# ----------------------------------------------------------------------------------------
def yarn_inv_t(s: float) -> float:
    """1/t for length ratio s. READING: s <= 1 means no extrapolation, so 1/t = 1."""
    if s <= 1.0:
        return 1.0
    r = 0.1 * math.log(s) + 1.0
    return r * r


def logit_scale(cfg) -> float:
    """Factor applied to <q, k>: (1/t) / sqrt(D)."""
    return yarn_inv_t(cfg.yarn_s) / math.sqrt(cfg.head_dim)


# ----------------------------------------------------------------------------------------
# RoPE  [P2 section 三: rotary position embedding]. READING: the rotate-half pairing
# (f, f + D/2) with theta_f = base^(-2f/D), as in the Qwen2 model family.
# ----------------------------------------------------------------------------------------
def rope_theta(d: int, base: float) -> np.ndarray:
    f = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * f / d)


def rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate vectors x[..., D] (fp64) by integer positions pos[...] (broadcast)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------------------
# DCA position remap  [P2 section 四 "Dual Chunk Attention": intra-chunk, inter-chunk and
# successive-chunk attention; Figure 2: relative positions stay within the trained range].
# READING: c = dca_chunk is the trained length, a DCA chunk holds L = c - w tokens,
# keys sit at j mod L, the query sits at
#   intra (same chunk):           i mod L
#   successive (previous chunk):  min(i mod L + L, c - 1)
#   inter (two or more back):     c - 1
# ----------------------------------------------------------------------------------------
def dca_len(cfg) -> int:
    return cfg.dca_chunk - cfg.local_window


def dca_pattern(i, j, cfg) -> np.ndarray:
    L = dca_len(cfg)
    ci = np.asarray(i) // L
    cj = np.asarray(j) // L
    return np.where(ci == cj, INTRA, np.where(cj == ci - 1, SUCC, INTER))


def dca_key_position(j, cfg) -> np.ndarray:
    return np.asarray(j) % dca_len(cfg)


def dca_query_position(i, pattern: int, cfg) -> np.ndarray:
    L, c = dca_len(cfg), cfg.dca_chunk
    t = np.asarray(i) % L
    if pattern == INTRA:
        return t
    if pattern == SUCC:
        return np.minimum(t + L, c - 1)
    return np.full_like(t, c - 1)


def rotated_keys(k_g: np.ndarray, cfg) -> np.ndarray:
    """R(j mod L) k_j for the keys k_g[J, D] of one KV head, j = 0 .. J-1."""
    j = np.arange(k_g.shape[0])
    return rope(k_g, dca_key_position(j, cfg), cfg.rope_base)


def dca_logits(q_rows: np.ndarray, i_rows: np.ndarray, krot: np.ndarray, js: np.ndarray,
               cfg) -> np.ndarray:
    """Scaled DCA logits l(i, j) for query rows q_rows[n, D] at positions i_rows[n] (one Q
    head) against keys js[J] whose rotated values are krot[J, D]. Each pair uses the query
    position of its own pattern."""
    i_rows = np.asarray(i_rows)
    pat = dca_pattern(i_rows[:, None], np.asarray(js)[None, :], cfg).astype(np.int8)
    out = np.zeros(pat.shape, dtype=np.float64)
    for p in (INTRA, SUCC, INTER):
        if not np.any(pat == p):
            continue
        qv = rope(q_rows, dca_query_position(i_rows, p, cfg), cfg.rope_base)
        out = np.where(pat == p, qv @ krot.T, out)
    return out * logit_scale(cfg)


# ----------------------------------------------------------------------------------------
# Chunked prefill  [P5 "Sparse Attention" and "Deploy ...": prefill in query chunks of
# 32,768 / 131,072 tokens; each chunk attends the growing key prefix].
# ----------------------------------------------------------------------------------------
def prefill_chunks(cfg):
    """Yield (s0, e): query rows [s0, e) of each prefill chunk; keys are [0, e)."""
    if getattr(cfg, "equal_cost_chunks", 0) > 0:
        yield from equal_cost_chunks(cfg.seq_len, cfg.equal_cost_chunks)
        return
    for s0 in range(0, cfg.seq_len, cfg.prefill_chunk):
        yield s0, min(cfg.seq_len, s0 + cfg.prefill_chunk)


def equal_cost_chunks(n: int, K: int):
    """Prefill chunks of equal dense attention cost ([P2] 四, pipeline-parallel optimisation,
    DCPP, Figure 9: chunk sizes follow the attention kernel's cost so that chunks take equal
    time). READING: the cost unit is one 128 x 128 block of the dense causal mask, so query
    block b costs b + 1 and the first m blocks cost 1 + 2 + ... + m. Chunk k < K closes at
    the first block boundary where that cumulative cost reaches k/K of the whole; the last
    chunk closes at n. A boundary that repeats the previous one is dropped."""
    nb = -(-n // BLOCK)
    cum = []                       # cum[i] = cost of blocks 0..i (Python ints: exact)
    total = 0
    for b in range(nb):
        total += b + 1
        cum.append(total)
    import bisect
    cuts = []
    for k in range(1, K):
        need = -(-k * total // K)  # ceil(k T / K): cumulative cost the chunk must reach
        m = bisect.bisect_left(cum, need) + 1
        if not cuts or m > cuts[-1]:
            cuts.append(m)
    rows = [min(n, BLOCK * m) for m in cuts if m < nb] + [n]
    s0 = 0
    for e in rows:
        yield s0, e
        s0 = e


def softmax_rows(l: np.ndarray):
    """Row softmax and log-sum-exp of logits l[n, J] (entries -inf are excluded)."""
    m = np.max(l, axis=1, keepdims=True)
    p = np.exp(l - m)
    s = np.sum(p, axis=1, keepdims=True)
    return p / s, (m + np.log(s))[:, 0]


# ----------------------------------------------------------------------------------------
# Vertical-slash estimator  [P2 section 四 "稀疏注意力机制": MInference vertical-slash
# pattern, key tokens selected per prefill chunk]. READING: the last vs_last_q rows R of
# the chunk; p_ij = softmax over j in [0, i] of the DCA logits; vertical score of column
# j = sum over R of p_ij; slash score of offset o = sum over R of p_{i, i-o} (o is the
# true token distance, which keeps a slash line continuous across DCA chunks).
# Scores are stored as float32 (the form the selection consumes).
# ----------------------------------------------------------------------------------------
def estimator_rows(s0: int, e: int, cfg) -> np.ndarray:
    return np.arange(max(s0, e - cfg.vs_last_q), e)


def estimate_head(q_R: np.ndarray, R: np.ndarray, krot_g: np.ndarray, e: int, cfg):
    """Scores of one Q head for a prefill chunk ending at e, from its estimator rows R
    (raw q rows q_R[|R|, D]). Returns (vert[e] f32, slash[e] f32, lse[|R|] f64)."""
    js = np.arange(e)
    l = dca_logits(q_R, R, krot_g[:e], js, cfg)
    l = np.where(js[None, :] <= R[:, None], l, -np.inf)
    p, lse = softmax_rows(l)
    vert = np.sum(p, axis=0)
    slash = np.zeros(e, dtype=np.float64)
    for r, i in enumerate(R):
        slash[: i + 1] += p[r, i::-1]          # offset o = i - j for j = i, i-1, ..., 0
    return vert.astype(np.float32), slash.astype(np.float32), lse


# ----------------------------------------------------------------------------------------
# Selection. READING: per Q head, the vs_vertical columns with the largest vertical
# score and the vs_slash offsets with the largest slash score; offsets below
# vs_force_local are always kept (score +inf); larger score first, equal scores by the
# smaller index; a budget >= the candidate count keeps every candidate.
# ----------------------------------------------------------------------------------------
def top_budget(scores: np.ndarray, budget: int) -> np.ndarray:
    scores = np.asarray(scores, dtype=np.float64)
    if np.any(np.isnan(scores)):
        raise ValueError("NaN score")
    n = scores.shape[0]
    if budget >= n:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -scores))
    return np.sort(order[:budget]).astype(np.int64)


def select_head(vert: np.ndarray, slash: np.ndarray, cfg):
    """Return (V, S): sorted vertical columns and sorted slash offsets of one head."""
    sl = np.asarray(slash, dtype=np.float64).copy()
    sl[: cfg.vs_force_local] = np.inf
    return top_budget(vert, cfg.vs_vertical), top_budget(sl, cfg.vs_slash)


# ----------------------------------------------------------------------------------------
# Block mask. READING: 128 x 128 blocks; query block b covers rows r0 = 128 b ..
# r1 = min(128 b + 127, e - 1); key block kb is computed when some slash line i - j = o
# (o in S, o <= r1) crosses it, i.e. floor(max(0, r0 - o)/128) <= kb <= floor((r1 - o)/128);
# verticals not inside a computed block stay as single columns (the residual list).
# ----------------------------------------------------------------------------------------
def computed_blocks(S: np.ndarray, b: int, e: int, bs: int = BLOCK) -> np.ndarray:
    """Boolean[nkb] over key blocks of query block b (nkb = ceil(e / bs))."""
    nkb = (e + bs - 1) // bs
    r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
    o = np.asarray(S, dtype=np.int64)
    o = o[o <= r1]
    lo, hi = np.maximum(0, r0 - o) // bs, (r1 - o) // bs
    # mark every block lo..hi of every offset: +1 at lo, -1 after hi, running sum > 0
    cnt = np.zeros(nkb + 1, dtype=np.int64)
    np.add.at(cnt, lo, 1)
    np.add.at(cnt, hi + 1, -1)
    return np.cumsum(cnt)[:nkb] > 0


def residual_verticals(V: np.ndarray, blocks: np.ndarray, b: int, e: int,
                       bs: int = BLOCK) -> np.ndarray:
    r1 = min(b * bs + bs - 1, e - 1)
    V = np.asarray(V)
    keep = (V <= r1) & ~blocks[np.minimum(V // bs, blocks.shape[0] - 1)]
    return V[keep]


def attended_mask(i: int, blocks: np.ndarray, V: np.ndarray, bs: int = BLOCK) -> np.ndarray:
    """Boolean[i + 1]: the attended set A(i) = {j <= i in a computed block} union
    {j in V, j <= i}."""
    js = np.arange(i + 1)
    m = blocks[js // bs].copy()
    V = np.asarray(V)
    m[V[V <= i]] = True
    return m


# ----------------------------------------------------------------------------------------
# Output: out_i = sum over j in A(i) of softmax_j(l(i, .)) v_j, and lse_i.
# ----------------------------------------------------------------------------------------
@dataclass
class ChunkSelection:
    s0: int
    e: int
    vert: np.ndarray | None = None    # [Hq, e] float32
    slash: np.ndarray | None = None   # [Hq, e] float32
    est_lse: np.ndarray | None = None  # [Hq, |R|] natural-log LSE of the estimator rows
    V: list | None = None             # per head: sorted int64 columns
    S: list | None = None             # per head: sorted int64 offsets


def as_f64(t) -> np.ndarray:
    """Exact fp64 view of a CPU tensor / array (bf16 and fp32 widen exactly)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", dtype=torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


class Oracle:
    """The oracle for one layer: inputs q [N, Hq, D], k, v [N, Hkv, D] (any float dtype,
    widened exactly to fp64) and a workload ``cfg``."""

    def __init__(self, q, k, v, cfg):
        self.cfg = cfg
        self.q = q            # kept in its input dtype; rows widened on demand
        self.k = as_f64(k)
        self.v = as_f64(v)
        self._krot = {}

    def krot(self, g: int) -> np.ndarray:
        if g not in self._krot:
            self._krot[g] = rotated_keys(self.k[:, g, :], self.cfg)
        return self._krot[g]

    def q_rows(self, rows: np.ndarray, h: int) -> np.ndarray:
        rows = np.asarray(rows, dtype=np.int64)
        if isinstance(self.q, np.ndarray):
            return np.asarray(self.q[rows, h, :], dtype=np.float64)
        import torch
        return as_f64(self.q[torch.from_numpy(rows), h, :])

    # -- per prefill chunk ---------------------------------------------------------------
    def select_chunk(self, s0: int, e: int, heads=None) -> ChunkSelection:
        cfg = self.cfg
        sel = ChunkSelection(s0, e)
        if cfg.dense:
            return sel
        G = cfg.group
        heads = range(cfg.n_q_heads) if heads is None else heads
        sel.vert = np.zeros((cfg.n_q_heads, e), np.float32)
        sel.slash = np.zeros((cfg.n_q_heads, e), np.float32)
        nR = len(estimator_rows(s0, e, cfg))
        sel.est_lse = np.zeros((cfg.n_q_heads, nR))
        sel.V, sel.S = [None] * cfg.n_q_heads, [None] * cfg.n_q_heads
        R = estimator_rows(s0, e, cfg)
        for h in heads:
            vt, sl, lse = estimate_head(self.q_rows(R, h), R, self.krot(h // G), e, cfg)
            sel.vert[h], sel.slash[h], sel.est_lse[h] = vt, sl, lse
            sel.V[h], sel.S[h] = select_head(vt, sl, cfg)
        return sel

    def blocks(self, h: int, b: int, sel: ChunkSelection) -> np.ndarray:
        key = (h, b)
        cache = sel.__dict__.setdefault("_blocks", {})
        if key not in cache:
            cache[key] = computed_blocks(sel.S[h], b, sel.e)
        return cache[key]

    def attended(self, i: int, h: int, sel: ChunkSelection) -> np.ndarray:
        if self.cfg.dense:
            return np.ones(i + 1, dtype=bool)
        return attended_mask(i, self.blocks(h, i // BLOCK, sel), sel.V[h])

    def attend_rows(self, rows: np.ndarray, h: int, sel: ChunkSelection):
        """Output rows out[n, D] and lse[n] of head h for query rows (all in sel's chunk)."""
        rows = np.asarray(rows)
        imax = int(rows.max())
        js = np.arange(imax + 1)
        l = dca_logits(self.q_rows(rows, h), rows, self.krot(h // self.cfg.group)[: imax + 1],
                       js, self.cfg)
        for r, i in enumerate(rows):
            a = np.zeros(imax + 1, dtype=bool)
            a[: i + 1] = self.attended(int(i), h, sel)
            l[r, ~a] = -np.inf
        p, lse = softmax_rows(l)
        return p @ self.v[: imax + 1, h // self.cfg.group, :], lse

    def decode_row(self, pos: int, h: int):
        """Decode step of the token at `pos`: out and lse of head h over keys [0, pos] with
        the DCA logits, densely ([P2] 四 "Dual Chunk Attention"; [P2] 三: generation after the
        long context). Equals row pos of the dense prefill by definition."""
        js = np.arange(pos + 1)
        l = dca_logits(self.q_rows(np.array([pos]), h), np.array([pos]),
                       self.krot(h // self.cfg.group)[: pos + 1], js, self.cfg)
        p, lse = softmax_rows(l)
        return (p @ self.v[: pos + 1, h // self.cfg.group, :])[0], float(lse[0])

    def recall_rows(self, rows: np.ndarray, h: int, sel: ChunkSelection) -> np.ndarray:
        """Share of the dense softmax mass of each row that its attended set A(i) keeps
        ([P2] 四 稀疏注意力机制: sparsity refinement limits the accuracy loss)."""
        rows = np.asarray(rows)
        imax = int(rows.max())
        js = np.arange(imax + 1)
        l = dca_logits(self.q_rows(rows, h), rows, self.krot(h // self.cfg.group)[: imax + 1],
                       js, self.cfg)
        res = np.zeros(len(rows))
        for r, i in enumerate(rows):
            p, _ = softmax_rows(l[[r], : i + 1])
            res[r] = float(np.sum(p[0][self.attended(int(i), h, sel)]))
        return res

    # -- whole layer -----------------------------------------------------------------------
    def run(self, rows_by_head=None, batch: int = 32):
        """Run the layer. rows_by_head: None (every row of every head) or a dict
        h -> sorted array of rows. Returns (out dict h -> [n, D], lse dict h -> [n],
        list of ChunkSelection)."""
        cfg = self.cfg
        if rows_by_head is None:
            rows_by_head = {h: np.arange(cfg.seq_len) for h in range(cfg.n_q_heads)}
        out = {h: np.zeros((len(r), cfg.head_dim)) for h, r in rows_by_head.items()}
        lse = {h: np.zeros(len(r)) for h, r in rows_by_head.items()}
        sels = []
        for s0, e in prefill_chunks(cfg):
            need = {h: np.nonzero((r >= s0) & (r < e))[0] for h, r in rows_by_head.items()}
            heads = [h for h, ix in need.items() if len(ix)]
            sel = self.select_chunk(s0, e, heads)
            sels.append(sel)
            for h in heads:
                ix = need[h]
                for b0 in range(0, len(ix), batch):
                    part = ix[b0: b0 + batch]
                    o, ls = self.attend_rows(rows_by_head[h][part], h, sel)
                    out[h][part], lse[h][part] = o, ls
        return out, lse, sels


# ----------------------------------------------------------------------------------------
# Log-sum-exp merge of partial attentions over a partition of A(i):
#   lse = log sum_p exp(lse_p),  out = sum_p exp(lse_p - lse) out_p.
# ----------------------------------------------------------------------------------------
def lse_merge(outs: np.ndarray, lses: np.ndarray):
    """outs[P, n, D], lses[P, n] -> (out[n, D], lse[n])."""
    m = np.max(lses, axis=0)
    w = np.exp(lses - m[None, :])
    s = np.sum(w, axis=0)
    return np.sum(w[:, :, None] * outs, axis=0) / s[:, None], m + np.log(s)

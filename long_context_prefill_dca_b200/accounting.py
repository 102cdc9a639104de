"""Algorithmic work of the layer: the number of attended (query, key) pairs, Σ|A(i)| over
rows and heads, counted from the layer's own block masks (the attention FLOPs are 4 D per
pair: QK^T and PV, 2 D each)."""
from __future__ import annotations

import numpy as np


def pairs_from_counts(cnt, s0: int, e: int) -> float:
    """Attended pairs of one prefill chunk from its per-(head, query block) counts
    [Hq][nqb][8] (blocks per DCA pattern, residual columns per pattern, total residuals):
    every computed block but the diagonal one gives each row 128 keys, the diagonal block
    its causal part, each residual vertical column one key per row."""
    c = np.asarray(cnt, dtype=np.float64)
    nqb = c.shape[1]
    r0 = s0 + 128 * np.arange(nqb)
    rows = np.minimum(128, e - r0).astype(np.float64)
    nblk = c[:, :, 0] + c[:, :, 1] + c[:, :, 2]
    nres = c[:, :, 6]
    pairs = rows[None] * (128.0 * (nblk - 1.0) + nres) + rows[None] * (rows[None] + 1) / 2
    return float(pairs.sum())


def dense_pairs(s0: int, e: int, n_q_heads: int) -> float:
    i = np.arange(s0, e, dtype=np.float64)
    return float(np.sum(i + 1)) * n_q_heads


def attended_pairs(w, g, device):
    """(total pairs over all rows and heads, computed-block density, per-chunk pairs).
    Runs the same estimator / selection / mask kernels as the layer (not timed)."""
    import torch
    from long_context_prefill_dca_b200 import q1m
    from long_context_prefill_dca_b200.layer import Stages
    bounds = q1m.prefill_bounds(w)
    if w.dense:
        per = [dense_pairs(s0, e, w.n_q_heads) for s0, e in bounds]
        return sum(per), 1.0, per
    st = Stages(w, device=device)
    blocks, causal, per = 0.0, 0.0, []
    for s0, e in bounds:
        st.keys(g["k"], g["v"], s0, e)
        vert, slash = st.estimate(g["q"], s0, e)
        V, S = st.select(vert, slash, e)
        _, _, cnt = st.masks(V, S, s0, e)
        c = cnt.cpu().numpy()
        per.append(pairs_from_counts(c, s0, e))
        blocks += float(c[:, :, 0:3].astype(np.float64).sum())
        nqb = c.shape[1]
        causal += float(((s0 // 128 + np.arange(nqb)) + 1).sum()) * w.n_q_heads
        del vert, slash, V, S, cnt
    del st
    torch.cuda.empty_cache()
    return sum(per), blocks / causal, per

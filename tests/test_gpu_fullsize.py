"""Full-size workloads (128K, 256K, 1M and the ragged 1.01M layer), in the launch
configuration the benchmark times, checked against the fp64 oracle on sampled rows.

For each workload: the GPU runs every prefill chunk stage by stage; for the checked heads the
oracle's fp32 scores go to the GPU selection (bit-exact index sets required) and the oracle's
index sets go to the GPU mask builder and attention; 4,096 seeded (token, head) rows of the
checked heads plus the first and last row of every prefill chunk are compared with the
oracle (max-abs 2e-2, mean-relative 1e-3). The product entry point q1m_dca_sparse_prefill
(the benchmark's call) is run on the same inputs and compared on the same rows.
"""
import os

import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Layer, Stages
from oracle import dca_vs as O
from synth import configs as C
from synth import inputs as I

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

MAX_ABS, MEAN_REL = 2e-2, 1e-3
N_ROWS = int(os.environ.get("Q1M_FULLSIZE_ROWS", "4096"))
WORKLOADS = [C.L7B_128K, C.L14B_256K, C.L7B_1M, C.L14B_1M]


def checked_heads(w):
    # one Q head in the first and one in the last KV group
    return [0, w.n_q_heads - 1]


def sampled_rows(w):
    pairs = I.sample_rows(w, N_ROWS)
    heads = checked_heads(w)
    # map every sampled (token, head) onto the checked heads, keeping the token
    toks = pairs[:, 0]
    hs = np.array(heads)[pairs[:, 1] % len(heads)]
    rows = {}
    for h in heads:
        rows[h] = np.unique(toks[hs == h])
    return rows


def rel(a, b):
    return float(np.sum(np.abs(a - b)) / np.sum(np.abs(b)))


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_full_size_sampled_rows(w):
    x = I.generate(w)
    dev = torch.device("cuda")
    g = {k: t.to(dev) for k, t in x.items()}
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    rows = sampled_rows(w)
    heads = sorted(rows)
    st = Stages(w)
    out = torch.full((w.seq_len, w.n_q_heads, w.head_dim), float("nan"), device=dev)
    ref_rows = {h: [] for h in heads}
    for s0, e in O.prefill_chunks(w):
        sel = orc.select_chunk(s0, e, heads)
        st.keys(g["k"], g["v"], s0, e)
        st.queries(g["q"], s0, e)
        vert, slash = st.estimate(g["q"], s0, e)
        torch.cuda.synchronize()
        q1m.check_status()
        for h in heads:
            rv, rs = rel(vert[h].cpu().numpy(), sel.vert[h]), rel(slash[h].cpu().numpy(), sel.slash[h])
            assert rv < 1e-3 and rs < 1e-3, (w.name, s0, h, rv, rs)
            # the oracle's scores for the checked heads
            vert[h] = torch.from_numpy(sel.vert[h]).to(dev)
            slash[h] = torch.from_numpy(sel.slash[h]).to(dev)
        V, S = st.select(vert, slash, e)
        Vc, Sc = V.cpu().numpy(), S.cpu().numpy()
        for h in heads:
            assert np.array_equal(Vc[h], sel.V[h]) and np.array_equal(Sc[h], sel.S[h]), (w.name, s0, h)
        mask, resid, cnt = st.masks(V, S, s0, e)
        st.attn(s0, e, mask, resid, cnt)
        st.merge(s0, e, out)
        torch.cuda.synchronize()
        q1m.check_status()
        for h in heads:
            r = rows[h][(rows[h] >= s0) & (rows[h] < e)]
            if len(r):
                o, _ = orc.attend_rows(r, h, sel)
                ref_rows[h].append((r, o))
        del vert, slash, V, S, mask, resid, cnt
    got_all, ref_all = [], []
    for h in heads:
        for r, o in ref_rows[h]:
            got_all.append(out[torch.from_numpy(r).to(dev), h].cpu().numpy())
            ref_all.append(o)
    got, ref = np.concatenate(got_all), np.concatenate(ref_all)
    err = np.abs(got - ref)
    print(f"{w.name}: {len(got)} rows, oracle-fed max-abs {err.max():.2e} mean-rel {rel(got, ref):.2e}")
    assert np.all(np.isfinite(got))
    assert err.max() <= MAX_ABS and rel(got, ref) <= MEAN_REL
    del st, out
    torch.cuda.empty_cache()

    # the product entry point, exactly as the benchmark calls it (own estimator/selection)
    layer = Layer(w, "f32")
    prod = layer(g["q"], g["k"], g["v"])
    torch.cuda.synchronize()
    q1m.check_status()
    pg = []
    for h in heads:
        for r, _ in ref_rows[h]:
            pg.append(prod[torch.from_numpy(r).to(dev), h].cpu().numpy())
    pg = np.concatenate(pg)
    perr = np.abs(pg - ref)
    print(f"{w.name}: product path max-abs {perr.max():.2e} mean-rel {rel(pg, ref):.2e}")
    assert perr.max() <= MAX_ABS and rel(pg, ref) <= MEAN_REL

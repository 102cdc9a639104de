"""Checks that pin the fp64 oracle to facts outside itself.

Each check returns a float error (0 means exact agreement) or a bool; the pin tests
assert on them, and the mutation tests plant plausible mistakes in the oracle (on the
CPU) and assert that some check then fails. None of these re-types an oracle formula:
each compares against a library routine, an independent formulation, a closed form, an
invariant or a brute-force enumeration.
"""
from __future__ import annotations

import cmath
import math
import os

import numpy as np
import torch

from oracle import dca_vs as O
from synth.configs import Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(**kw) -> Workload:
    base = dict(name="pin", seq_len=96, n_q_heads=2, n_kv_heads=1, head_dim=8,
                in_dtype="f32", rope_base=100.0, dca_chunk=24, local_window=6, yarn_s=1.0,
                prefill_chunk=96, vs_vertical=0, vs_slash=0)
    base.update(kw)
    return Workload(**base)


def rand_qkv(cfg, seed=0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((cfg.seq_len, cfg.n_q_heads, cfg.head_dim))
    k = g.standard_normal((cfg.seq_len, cfg.n_kv_heads, cfg.head_dim))
    v = g.standard_normal((cfg.seq_len, cfg.n_kv_heads, cfg.head_dim))
    return q, k, v


def full_output(q, k, v, cfg):
    orc = O.Oracle(q, k, v, cfg)
    out, lse, sels = orc.run()
    o = np.stack([out[h] for h in range(cfg.n_q_heads)], axis=1)   # [N, Hq, D]
    l = np.stack([lse[h] for h in range(cfg.n_q_heads)], axis=0)   # [Hq, N]
    return o, l, sels


# -- YaRN -----------------------------------------------------------------------------------
def check_yarn_golden() -> float:
    err = 0.0
    for line in open(os.path.join(GOLDEN, "yarn_scale.txt")):
        if line.startswith("#") or not line.strip():
            continue
        s, r, inv_t = map(float, line.split())
        err = max(err, abs(O.yarn_inv_t(s) - inv_t), abs(math.sqrt(O.yarn_inv_t(s)) - r))
    return err


# -- RoPE -----------------------------------------------------------------------------------
def check_rope_vs_transformers() -> float:
    """Against the Qwen2 rotary embedding of the transformers library."""
    from transformers import Qwen2Config
    from transformers.models.qwen2 import modeling_qwen2 as m
    d, base = 64, 1e4
    cfg = Qwen2Config(hidden_size=d, num_attention_heads=1, num_key_value_heads=1,
                      rope_theta=base, max_position_embeddings=4096)
    emb = m.Qwen2RotaryEmbedding(cfg)
    g = np.random.default_rng(1)
    pos = np.array([0, 1, 2, 7, 100, 999, 2047])
    x = g.standard_normal((len(pos), d))
    xt = torch.from_numpy(x)[None, None]          # [1, 1, n, d]
    cos, sin = emb(xt, torch.from_numpy(pos)[None])
    ref, _ = m.apply_rotary_pos_emb(xt, xt, cos.to(torch.float64), sin.to(torch.float64))
    got = O.rope(x, pos, base)
    freq_err = float(np.max(np.abs(emb.inv_freq.double().numpy() - O.rope_theta(d, base))
                            / O.rope_theta(d, base)))
    return max(float(np.max(np.abs(ref[0, 0].numpy() - got))), freq_err)


def check_rope_complex() -> float:
    """Rotate-half RoPE is multiplication of z_f = x_f + i x_{f+D/2} by e^{i p theta_f}."""
    g = np.random.default_rng(2)
    d, base = 16, 500.0
    x = g.standard_normal(d)
    err = 0.0
    for p in (0, 1, 5, 77, 4095):
        got = O.rope(x, np.array(p), base)
        for f in range(d // 2):
            th = base ** (-2.0 * f / d)
            z = complex(x[f], x[f + d // 2]) * cmath.exp(1j * p * th)
            err = max(err, abs(got[f] - z.real), abs(got[f + d // 2] - z.imag))
    return err


def check_rope_relative() -> float:
    """<R(a) q, R(b) k> depends on b - a only."""
    g = np.random.default_rng(3)
    d, base = 32, 1e4
    q, k = g.standard_normal(d), g.standard_normal(d)
    err = 0.0
    for a, b, s in ((3, 10, 50), (0, 7, 1000), (100, 100, 9)):
        d0 = O.rope(q, np.array(a), base) @ O.rope(k, np.array(b), base)
        d1 = O.rope(q, np.array(a + s), base) @ O.rope(k, np.array(b + s), base)
        err = max(err, abs(d0 - d1))
    return err


# -- DCA ------------------------------------------------------------------------------------
def brute_relative(i: int, j: int, c: int, w: int) -> int:
    """DCA relative position by an independent characterisation: the true distance is kept
    for pairs in the same chunk and for pairs in the previous chunk whose query is among
    the first w positions of its chunk; every other pair sees the query pinned at the last
    trained position c - 1, i.e. relative position c - 1 - (key position in its chunk)."""
    L = c - w
    ci, cj = 0, 0
    while (ci + 1) * L <= i:
        ci += 1
    while (cj + 1) * L <= j:
        cj += 1
    t = i - ci * L
    if ci == cj or (cj == ci - 1 and t < w):
        return i - j
    return c - 1 - (j - cj * L)


def brute_logit(q, k, rel, base, scale) -> float:
    d = q.shape[0]
    acc = 0.0
    for f in range(d // 2):
        th = base ** (-2.0 * f / d)
        zq = complex(q[f], q[f + d // 2])
        zk = complex(k[f], k[f + d // 2])
        acc += (zq.conjugate() * zk * cmath.exp(-1j * rel * th)).real
    return acc * scale


def check_dca_brute_force(cfg=None) -> float:
    """Oracle logits against pair-by-pair complex arithmetic on relative positions."""
    cfg = cfg or tiny(yarn_s=3.0)
    q, k, _ = rand_qkv(cfg, 4)
    krot = O.rotated_keys(k[:, 0, :], cfg)
    scale = O.yarn_inv_t(cfg.yarn_s) / math.sqrt(cfg.head_dim)
    err = 0.0
    for i in range(0, cfg.seq_len, 5):
        js = np.arange(i + 1)
        got = O.dca_logits(q[[i], 0, :], np.array([i]), krot[: i + 1], js, cfg)[0]
        for j in js:
            rel = brute_relative(i, int(j), cfg.dca_chunk, cfg.local_window)
            err = max(err, abs(got[j] - brute_logit(q[i, 0], k[j, 0], rel, cfg.rope_base,
                                                     scale)))
    return err


def check_dca_invariants(cfg=None) -> bool:
    """Every remapped relative position lies in [0, c-1]; pairs closer than w keep their
    true distance."""
    cfg = cfg or tiny()
    c, w = cfg.dca_chunk, cfg.local_window
    n = cfg.seq_len
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    ok = True
    for p in (O.INTRA, O.SUCC, O.INTER):
        pat = O.dca_pattern(i, j, cfg)
        rel = O.dca_query_position(np.broadcast_to(i, pat.shape), p, cfg) - \
            O.dca_key_position(np.broadcast_to(j, pat.shape), cfg)
        sel = (pat == p) & (j <= i)
        ok &= bool(np.all((rel[sel] >= 0) & (rel[sel] <= c - 1)))
        near = sel & (i - j < w)
        ok &= bool(np.all(rel[near] == (i - j)[near]))
    return ok


def check_short_equals_causal_rope() -> float:
    """seq_len <= dca_chunk: DCA reduces to ordinary causal RoPE attention, computed here
    by transformers' Qwen2 rotation and torch's scaled_dot_product_attention (fp64)."""
    from transformers.models.qwen2 import modeling_qwen2 as m
    cfg = tiny(seq_len=48, dca_chunk=64, local_window=16, n_q_heads=4, n_kv_heads=2,
               head_dim=16, yarn_s=2.0, rope_base=1e3, prefill_chunk=48)
    q, k, v = rand_qkv(cfg, 5)
    o, lse, _ = full_output(q, k, v, cfg)
    d, n = cfg.head_dim, cfg.seq_len
    th = torch.from_numpy(O.rope_theta(d, cfg.rope_base))
    ang = torch.arange(n, dtype=torch.float64)[:, None] * th[None, :]
    emb = torch.cat([ang, ang], dim=-1)
    cos, sin = emb.cos()[None], emb.sin()[None]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]          # [1, Hq, N, D]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    qr, kr = m.apply_rotary_pos_emb(qt, kt, cos, sin)
    G = cfg.group
    kr = kr.repeat_interleave(G, dim=1)
    vt = vt.repeat_interleave(G, dim=1)
    scale = O.yarn_inv_t(cfg.yarn_s) / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, vt, is_causal=True,
                                                           scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    s = (qr @ kr.transpose(-1, -2))[0] * scale
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
    ref_lse = torch.logsumexp(s, dim=-1).numpy()
    return max(float(np.max(np.abs(o - ref))), float(np.max(np.abs(lse - ref_lse))))


# -- softmax / output -----------------------------------------------------------------------
def check_v_ones(cfg=None) -> float:
    cfg = cfg or tiny(vs_vertical=5, vs_slash=12, vs_force_local=4, prefill_chunk=40)
    q, k, _ = rand_qkv(cfg, 6)
    v = np.ones_like(k)
    o, _, _ = full_output(q, k, v, cfg)
    return float(np.max(np.abs(o - 1.0)))


def check_full_budget_is_dense() -> float:
    sp = tiny(seq_len=300, dca_chunk=80, local_window=16, vs_vertical=1, vs_slash=10**6,
              prefill_chunk=128)
    dn = sp.with_(vs_vertical=0, vs_slash=0)
    q, k, v = rand_qkv(sp, 7)
    o1, l1, _ = full_output(q, k, v, sp)
    o2, l2, _ = full_output(q, k, v, dn)
    return max(float(np.max(np.abs(o1 - o2))), float(np.max(np.abs(l1 - l2))))


def check_causal() -> float:
    """Row i does not depend on keys or values after i."""
    cfg = tiny(seq_len=200, dca_chunk=64, local_window=16, vs_vertical=4, vs_slash=30,
               vs_force_local=8, prefill_chunk=200)
    q, k, v = rand_qkv(cfg, 8)
    i = 150
    o1, _, _ = full_output(q, k, v, cfg)
    k2, v2 = k.copy(), v.copy()
    k2[i + 1:] += 10.0
    v2[i + 1:] -= 10.0
    # the estimator of this single-chunk layer reads the last rows' keys <= 199, so keep
    # the chunk's selection fixed by comparing rows through the oracle's own attended set
    orc1 = O.Oracle(q, k, v, cfg)
    orc2 = O.Oracle(q, k2, v2, cfg)
    sel = orc1.select_chunk(0, cfg.seq_len)
    a, _ = orc1.attend_rows(np.array([i]), 1, sel)
    b, _ = orc2.attend_rows(np.array([i]), 1, sel)
    return float(np.max(np.abs(a - b))) + float(np.max(np.abs(o1[i, 1] - a[0])))


def check_lse_merge() -> float:
    g = np.random.default_rng(9)
    n, J, d = 5, 40, 6
    l = g.standard_normal((n, J)) * 3
    v = g.standard_normal((J, d))
    p, lse = O.softmax_rows(l)
    full = p @ v
    part = g.integers(0, 3, size=J)
    outs, lses = [], []
    for t in range(3):
        lt = np.where(part[None, :] == t, l, -np.inf)
        pt, lst = O.softmax_rows(lt)
        outs.append(pt @ v)
        lses.append(lst)
    mo, ml = O.lse_merge(np.stack(outs), np.stack(lses))
    return max(float(np.max(np.abs(mo - full))), float(np.max(np.abs(ml - lse))))


# -- estimator ------------------------------------------------------------------------------
def check_estimator_mass() -> float:
    """Every estimator row's probabilities sum to one, so column sums and diagonal sums
    each total |R|; the estimator rows' LSE equals dense attention's LSE."""
    cfg = tiny(seq_len=220, dca_chunk=64, local_window=16, n_q_heads=2, vs_vertical=8,
               vs_slash=20, vs_last_q=16, vs_force_local=4, prefill_chunk=100, yarn_s=2.5)
    q, k, v = rand_qkv(cfg, 10)
    orc = O.Oracle(q, k, v, cfg)
    err = 0.0
    for s0, e in O.prefill_chunks(cfg):
        sel = orc.select_chunk(s0, e)
        R = O.estimator_rows(s0, e, cfg)
        for h in range(cfg.n_q_heads):
            err = max(err, abs(float(np.sum(sel.vert[h], dtype=np.float64)) - len(R)) / len(R),
                      abs(float(np.sum(sel.slash[h], dtype=np.float64)) - len(R)) / len(R))
            dense = O.Oracle(q, k, v, cfg.with_(vs_vertical=0, vs_slash=0))
            _, lse = dense.attend_rows(R, h, O.ChunkSelection(s0, e))
            err = max(err, float(np.max(np.abs(lse - sel.est_lse[h]))))
    return err


def check_estimator_brute_force() -> float:
    """Vertical and slash scores against per-pair loops over a tiny layer."""
    cfg = tiny(seq_len=60, dca_chunk=24, local_window=6, n_q_heads=1, vs_vertical=3,
               vs_slash=5, vs_last_q=7, vs_force_local=2, prefill_chunk=60, yarn_s=1.7)
    q, k, v = rand_qkv(cfg, 11)
    orc = O.Oracle(q, k, v, cfg)
    e = cfg.seq_len
    sel = orc.select_chunk(0, e)
    scale = O.yarn_inv_t(cfg.yarn_s) / math.sqrt(cfg.head_dim)
    vert = np.zeros(e)
    slash = np.zeros(e)
    for i in range(e - cfg.vs_last_q, e):
        ls = [brute_logit(q[i, 0], k[j, 0], brute_relative(i, j, cfg.dca_chunk,
                                                           cfg.local_window), cfg.rope_base,
                          scale) for j in range(i + 1)]
        m = max(ls)
        z = sum(math.exp(x - m) for x in ls)
        for j in range(i + 1):
            p = math.exp(ls[j] - m) / z
            vert[j] += p
            slash[i - j] += p
    return max(float(np.max(np.abs(vert - sel.vert[0]))),
               float(np.max(np.abs(slash - sel.slash[0]))))


# -- selection and masks --------------------------------------------------------------------
def check_topk_properties() -> bool:
    g = np.random.default_rng(12)
    ok = True
    for trial in range(200):
        n = int(g.integers(1, 60))
        k = int(g.integers(0, 70))
        sc = g.integers(0, 6, size=n).astype(np.float32)   # many ties
        sel = O.top_budget(sc, k)
        if k >= n:
            ok &= np.array_equal(sel, np.arange(n))
            continue
        ok &= len(sel) == k and len(set(sel.tolist())) == k and np.all(np.diff(sel) > 0)
        uns = np.setdiff1d(np.arange(n), sel)
        if k and len(uns):
            lo = sc[sel].min()
            ok &= sc[uns].max() <= lo
            # among the boundary value, the selected ones have the smallest indices
            tie_sel = sel[sc[sel] == lo]
            tie_uns = uns[sc[uns] == lo]
            if len(tie_uns):
                ok &= tie_sel.max() < tie_uns.min()
    return bool(ok)


def check_force_local() -> bool:
    cfg = tiny(vs_vertical=3, vs_slash=10, vs_force_local=4)
    g = np.random.default_rng(13)
    e = 50
    vert = g.random(e).astype(np.float32)
    slash = g.random(e).astype(np.float32)
    slash[:4] = 0.0
    V, S = O.select_head(vert, slash, cfg)
    return bool(set(range(4)) <= set(S.tolist()) and len(S) == 10 and len(V) == 3)


def check_mask_brute_force() -> bool:
    """Block formula against an element-wise enumeration of the slash lines."""
    g = np.random.default_rng(14)
    bs = 16
    ok = True
    for trial in range(30):
        e = int(g.integers(20, 300))
        S = np.sort(g.choice(e, size=int(g.integers(1, 12)), replace=False))
        nkb = (e + bs - 1) // bs
        for b in range(nkb):
            got = O.computed_blocks(S, b, e, bs)
            r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
            sset = set(S.tolist())
            want = np.zeros(nkb, dtype=bool)
            for kb in range(nkb):
                for i in range(r0, r1 + 1):
                    for j in range(kb * bs, min(kb * bs + bs, e)):
                        if (i - j) in sset:
                            want[kb] = True
            ok &= np.array_equal(got, want)
    return bool(ok)


def check_attended_set() -> bool:
    """A(i) by enumeration: j <= i, and (its block is crossed by a slash line for some row
    of i's block, or j is a selected vertical)."""
    g = np.random.default_rng(15)
    bs = O.BLOCK
    e = 700
    S = np.sort(np.concatenate([np.arange(8), g.choice(np.arange(8, e), 6, replace=False)]))
    V = np.sort(g.choice(e, 30, replace=False))
    ok = True
    sset, vset = set(S.tolist()), set(V.tolist())
    for i in (0, 5, 127, 128, 300, 511, 699):
        b = i // bs
        m = O.attended_mask(i, O.computed_blocks(S, b, e), V)
        r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
        # offsets realised by some (row of block b, key of block kb) pair
        crossed = [bool(sset & set(range(r0 - min(kb * bs + bs, e) + 1, r1 - kb * bs + 1)))
                   for kb in range(b + 1)]
        for j in range(i + 1):
            ok &= bool(m[j]) == (crossed[j // bs] or j in vset)
    return bool(ok)


def check_residual_verticals() -> bool:
    """The residual vertical columns of a query block, together with its computed blocks,
    give exactly the attended set of every row of the block (no selected column lost or
    counted twice); they lie outside the computed blocks, ascend, and never pass the block's
    last row."""
    rng = np.random.default_rng(21)
    bs = O.BLOCK
    ok = True
    for t in range(40):
        e = int(rng.integers(1, 700))
        b = int(rng.integers(0, (e - 1) // bs + 1))
        r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
        V = rng.choice(e, size=min(e, int(rng.integers(0, 40))), replace=False)
        if t % 2:          # the block's own first and last rows among the columns
            V = np.concatenate([V, [r0, r1]])
        V = np.unique(V)
        lo_o = bs if t % 4 >= 2 and e > bs else 0     # no short offsets: diagonal block may be skipped
        S = np.sort(rng.choice(np.arange(lo_o, e), size=min(e - lo_o, int(rng.integers(1, 30))),
                               replace=False))
        blocks = O.computed_blocks(S, b, e)
        res = np.asarray(O.residual_verticals(V, blocks, b, e))
        ok &= bool(np.all(np.diff(res) > 0)) and bool(np.all(res <= r1))
        ok &= not bool(np.any(blocks[res // bs])) if len(res) else True
        for i in range(r0, r1 + 1):
            parts = blocks[np.arange(i + 1) // bs].copy()
            parts[res[res <= i]] = True
            ok &= bool(np.array_equal(O.attended_mask(i, blocks, V), parts))
    return bool(ok)


def check_recall() -> float:
    """Recall is 1 for a full budget and equals exp(lse_sparse - lse_dense) otherwise, on a
    layer whose selection covers every block and on a sparser one where rows keep only part
    of the dense mass (the check fails if that second case does not reach recall < 0.9)."""
    err, low = 0.0, 1.0
    for n, ns, rows in ((260, 12, [3, 70, 129, 200, 259]), (1400, 4, [3, 129, 700, 1100, 1399])):
        cfg = tiny(seq_len=n, dca_chunk=80, local_window=16, vs_vertical=4, vs_slash=ns,
                   vs_force_local=2, prefill_chunk=n)
        rows = np.array(rows)
        q, k, v = rand_qkv(cfg, 16)
        orc = O.Oracle(q, k, v, cfg)
        sel = orc.select_chunk(0, cfg.seq_len)
        rec = orc.recall_rows(rows, 1, sel)
        _, lse_s = orc.attend_rows(rows, 1, sel)
        dense = O.Oracle(q, k, v, cfg.with_(vs_vertical=0, vs_slash=0))
        _, lse_d = dense.attend_rows(rows, 1, O.ChunkSelection(0, cfg.seq_len))
        full = cfg.with_(vs_vertical=10**6, vs_slash=10**6)
        of = O.Oracle(q, k, v, full)
        sf = of.select_chunk(0, cfg.seq_len)
        err = max(err, float(np.max(np.abs(rec - np.exp(lse_s - lse_d)))),
                  float(np.max(np.abs(of.recall_rows(rows, 1, sf) - 1.0))),
                  float(max(0.0, np.max(rec) - 1.0)))
        low = min(low, float(np.min(rec)))
    return err if low < 0.9 else float("inf")


def check_fixed_chunks() -> bool:
    """Fixed-size chunked prefill (the pages' --max-num-batched-tokens): hand-worked chunk
    lists, and the layer's selections follow them (each selection's [s0, e) is a chunk and
    its estimator rows are that chunk's last rows)."""
    cases = {(300, 128): [(0, 128), (128, 256), (256, 300)], (256, 128): [(0, 128), (128, 256)],
             (5, 128): [(0, 5)], (129, 128): [(0, 128), (128, 129)]}
    ok = True
    for (n, P), want in cases.items():
        ok &= list(O.prefill_chunks(tiny(seq_len=n, prefill_chunk=P))) == want
    cfg = tiny(seq_len=300, dca_chunk=80, local_window=16, vs_vertical=4, vs_slash=10,
               vs_force_local=2, prefill_chunk=128)
    q, k, v = rand_qkv(cfg, 31)
    sels = O.Oracle(q, k, v, cfg).run()[2]
    ok &= [(s.s0, s.e) for s in sels] == cases[(300, 128)]
    for s in sels:
        ok &= s.est_lse.shape[1] == min(cfg.vs_last_q, s.e - s.s0)
    return bool(ok)


def check_equal_cost_chunks() -> int:
    """The equal-cost chunking against the hand-worked fixture and its invariants: chunks
    tile [0, n) in 128-row blocks, there are at most K, and each chunk's dense cost is within
    one block row's cost (the largest block's b + 1) of T / K, except that dropped empty
    chunks merge their share into a neighbour. Returns the number of cases checked."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "equal_cost_chunks.txt")
    cases = 0
    for line in open(path):
        if not line.strip() or line.startswith("#"):
            continue
        n, K, *ends = (int(x) for x in line.split())
        got = [e for _, e in O.equal_cost_chunks(n, K)]
        assert got == ends, (n, K, got, ends)
        cases += 1
    rng = np.random.default_rng(7)
    for _ in range(200):
        n = int(rng.integers(1, 40000)); K = int(rng.integers(1, 40))
        ch = list(O.equal_cost_chunks(n, K))
        nb = -(-n // 128)
        assert ch[0][0] == 0 and ch[-1][1] == n and len(ch) <= K
        assert all(a[1] == b[0] for a, b in zip(ch, ch[1:]))
        assert all(e % 128 == 0 for _, e in ch[:-1]) and all(e > s for s, e in ch)
        T = nb * (nb + 1) // 2
        costs = [sum(b + 1 for b in range(s // 128, -(-e // 128))) for s, e in ch]
        assert sum(costs) == T
        if len(ch) == K:   # nothing dropped: every chunk is within one block of T / K
            assert max(abs(c - T / K) for c in costs) <= nb + 1, (n, K, costs)
        cases += 1
    return cases


def check_decode_row() -> float:
    """The decode step against pair-by-pair brute force (independently worded relative
    positions, complex-arithmetic RoPE) over every key j <= pos, for positions on both sides
    of DCA chunk boundaries, and V = 1 giving out = 1."""
    cfg = tiny(yarn_s=3.0, n_q_heads=3, n_kv_heads=1)
    q, k, v = rand_qkv(cfg, 9)
    orc = O.Oracle(q, k, v, cfg)
    scale = O.yarn_inv_t(cfg.yarn_s) / math.sqrt(cfg.head_dim)
    L = O.dca_len(cfg)
    err = 0.0
    for pos in (0, 1, L - 1, L, 2 * L - 1, 2 * L, 2 * L + 5, cfg.seq_len - 1):
        for h in range(cfg.n_q_heads):
            got, lse = orc.decode_row(pos, h)
            lg = np.array([brute_logit(q[pos, h], k[j, 0], brute_relative(pos, j, cfg.dca_chunk,
                                                                          cfg.local_window),
                                       cfg.rope_base, scale) for j in range(pos + 1)])
            mx = lg.max()
            w = np.exp(lg - mx)
            ref = (w[:, None] * v[: pos + 1, 0, :]).sum(0) / w.sum()
            err = max(err, float(np.max(np.abs(got - ref))), abs(lse - (mx + math.log(w.sum()))))
    ones = O.Oracle(q, k, np.ones_like(v), cfg)
    err = max(err, float(np.max(np.abs(ones.decode_row(cfg.seq_len - 1, 1)[0] - 1.0))))
    # the decode step of the token at pos is row pos of the dense prefill (reading C12)
    for pos in (0, L, 2 * L + 5, cfg.seq_len - 1):
        o, l = orc.attend_rows(np.array([pos]), 2, O.ChunkSelection(0, cfg.seq_len))
        d, dl = orc.decode_row(pos, 2)
        err = max(err, float(np.max(np.abs(o[0] - d))), abs(float(l[0]) - dl))
    return err


def check_key_order_invariance() -> float:
    """The output does not depend on the order in which the attended keys are summed: the
    oracle's rows against the same softmax taken over a random permutation of the (logit,
    value) pairs of each row."""
    cfg = tiny(yarn_s=2.0, vs_vertical=6, vs_slash=10, vs_force_local=4)
    q, k, v = rand_qkv(cfg, 12)
    orc = O.Oracle(q, k, v, cfg)
    sel = orc.select_chunk(0, cfg.seq_len)
    rows = np.array([5, 30, 61, 95])
    got, _ = orc.attend_rows(rows, 0, sel)
    rng = np.random.default_rng(3)
    err = 0.0
    for r, i in enumerate(rows):
        js = np.nonzero(orc.attended(int(i), 0, sel))[0]
        perm = rng.permutation(len(js))
        jp = js[perm]
        l = O.dca_logits(q[[i], 0, :], np.array([i]), orc.krot(0)[jp], jp, cfg)[0]
        w = np.exp(l - l.max())
        ref = (w[:, None] * v[jp, 0, :]).sum(0) / w.sum()
        err = max(err, float(np.max(np.abs(got[r] - ref))))
    return err

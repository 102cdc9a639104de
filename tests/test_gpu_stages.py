"""Parity of every stage of the CUDA path with the fp64 oracle, on small seeded workloads
that span several 128-row tiles, DCA chunks and prefill chunks, with ragged tails.

Protocol: the oracle never takes CUDA results as input. The GPU selection is fed the
oracle's fp32 scores and must return the oracle's index sets bit for bit; the GPU mask
builder is fed the oracle's index sets and must return the oracle's block masks and residual
lists bit for bit; the GPU attention runs on those masks and must match the oracle's output
within max-abs 2e-2 and mean-relative 1e-3 (fp32 accumulation, fp32 output).
"""
import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Layer, Stages
from oracle import dca_vs as O
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_REL = 2e-2, 1e-3
CASES = [C.TINY_2K, C.SMALL_SPARSE, C.SMALL_DENSE_D128, C.SMALL_SPARSE_D64]
SPARSE = [w for w in CASES if not w.dense]

_cache = {}


def case(w):
    """Inputs (CPU and GPU) and the oracle's full result for workload w."""
    if w.name not in _cache:
        x = I.generate(w)
        g = {k: t.cuda() for k, t in x.items()}
        orc = O.Oracle(x["q"], x["k"], x["v"], w)
        out, lse, sels = orc.run()
        o = np.stack([out[h] for h in range(w.n_q_heads)], axis=1)
        l = np.stack([lse[h] for h in range(w.n_q_heads)], axis=0)
        _cache[w.name] = dict(x=x, g=g, orc=orc, out=o, lse=l, sels=sels)
    return _cache[w.name]


def mean_rel(a, b):
    return float(np.sum(np.abs(a - b)) / np.sum(np.abs(b)))


def f16(t):
    return t.view(torch.float16).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_rope_table(w):
    st = Stages(w)
    tab = st.table.view(w.dca_chunk, w.head_dim // 2, 2).cpu().numpy().astype(np.float64)
    ang = np.arange(w.dca_chunk)[:, None] * O.rope_theta(w.head_dim, w.rope_base)[None, :]
    assert np.max(np.abs(tab[..., 0] - np.cos(ang))) < 2e-7
    assert np.max(np.abs(tab[..., 1] - np.sin(ang))) < 2e-7


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_rope_dca_keys_and_query_views(w):
    c = case(w)
    st = Stages(w)
    n = w.seq_len
    s0, e = 0, min(n, w.prefill_chunk)
    st.keys(c["g"]["k"], c["g"]["v"], 0, n)
    st.queries(c["g"]["q"], s0, e)
    torch.cuda.synchronize()
    q1m.check_status()
    for g in range(w.n_kv_heads):
        ref = O.rotated_keys(O.as_f64(c["x"]["k"][:, g]), w)
        got = f16(st.k_rot[g, :n])
        assert np.all(np.abs(got - ref) <= 6e-4 * np.abs(ref) + 1e-6)
        vref = O.as_f64(c["x"]["v"][:, g])
        assert np.all(np.abs(f16(st.v16[g, :n]) - vref) <= 6e-4 * np.abs(vref) + 1e-7)
    scale = O.logit_scale(w) * np.log2(np.e)
    rows = np.arange(s0, e)
    for x, pat in ((0, O.INTRA), (1, O.SUCC), (2, O.INTER)):
        for h in range(w.n_q_heads):
            ref = O.rope(O.as_f64(c["x"]["q"][s0:e, h]), O.dca_query_position(rows, pat, w),
                         w.rope_base) * scale
            got = f16(st.qv[x, h, : e - s0])
            assert np.all(np.abs(got - ref) <= 6e-4 * np.abs(ref) + 1e-6), (x, h)
    assert np.all(f16(st.qv[:, :, e - s0:]) == 0)


def run_chunk_scores(w, st, c, s0, e):
    st.keys(c["g"]["k"], c["g"]["v"], s0, e)
    return st.estimate(c["g"]["q"], s0, e)


@pytest.mark.parametrize("w", SPARSE, ids=lambda w: w.name)
def test_estimator_scores(w):
    c = case(w)
    st = Stages(w)
    for sel in c["sels"]:
        vert, slash = run_chunk_scores(w, st, c, sel.s0, sel.e)
        torch.cuda.synchronize()
        q1m.check_status()
        gv, gs = vert.cpu().numpy(), slash.cpu().numpy()
        rv, rs = mean_rel(gv, sel.vert), mean_rel(gs, sel.slash)
        print(f"{w.name} chunk [{sel.s0},{sel.e}) vert rel-L1 {rv:.2e} slash rel-L1 {rs:.2e}")
        assert rv < 1e-3 and rs < 1e-3
        # every estimator row's probabilities sum to one
        nR = len(O.estimator_rows(sel.s0, sel.e, w))
        assert np.allclose(gv.sum(1), nR, rtol=2e-3) and np.allclose(gs.sum(1), nR, rtol=2e-3)


# every head-pair layout of the estimator's second pass: one head (a lone pair), four heads
# (one accumulator), six and seven heads (two accumulators, the last pair full or alone); a
# last prefill chunk of 40 rows (fewer estimator rows than 64)
GROUPS = [
    C.SMALL_SPARSE.with_(name=f"est-g{G}-d{D}", n_q_heads=2 * G, n_kv_heads=2, head_dim=D,
                         seq_len=1064, prefill_chunk=512, vs_vertical=40, vs_slash=80,
                         seed=C.SEED_BASE + 60 + G)
    for G, D in ((1, 128), (4, 64), (6, 128), (7, 128))
]


@pytest.mark.parametrize("w", GROUPS, ids=lambda w: w.name)
def test_estimator_scores_every_group_size(w):
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    st = Stages(w)
    for s0, e in O.prefill_chunks(w):
        sel = orc.select_chunk(s0, e)
        st.keys(g["k"], g["v"], s0, e)
        vert, slash = st.estimate(g["q"], s0, e)
        torch.cuda.synchronize()
        q1m.check_status()
        gv, gs = vert.cpu().numpy(), slash.cpu().numpy()
        nR = len(O.estimator_rows(s0, e, w))
        for h in range(w.n_q_heads):
            rv, rs = mean_rel(gv[h], sel.vert[h]), mean_rel(gs[h], sel.slash[h])
            assert rv < 1e-3 and rs < 1e-3, (w.name, s0, h, rv, rs)
            assert abs(gv[h].sum() - nR) < 2e-3 * nR and abs(gs[h].sum() - nR) < 2e-3 * nR


# the 7B head shape (7 Q heads per KV head) on 12,288 tokens: the last prefill chunk's 96 key
# tiles fall into 18 splits of 6 tiles in the estimator's first pass
DOMINANT = C.SMALL_SPARSE.with_(name="est-dominant-key", seq_len=12288, n_q_heads=28, n_kv_heads=4,
                                head_dim=128, rope_base=1e6, dca_chunk=4096, local_window=512,
                                yarn_s=4.0, prefill_chunk=4096, vs_vertical=200, vs_slash=400,
                                sinks=0, bands=0, seed=C.SEED_BASE + 70)


def test_estimator_scores_with_a_dominant_late_key():
    """One key per KV head whose logit lies 35 to 180 log2 units (depending on the row) above
    every other key of the estimator rows. At the last prefill chunk it is in the fifth key tile
    of its split (tile 40; splits of 6 tiles). Against the reference that a split's first tile
    set, the rows with the larger gaps sum past 2^64 or overflow there and redo the tile against
    its own maximum; the others keep the reference with sums up to 2^64. At the middle chunk the
    key falls in the first tile of its split. The scores must still match the oracle and sum to
    one per row. The planted direction is the lowest-frequency rotary pair (dimensions 63 and
    127), which the rotations barely turn at these distances."""
    w = DOMINANT
    x = I.generate(w)
    D, G = w.head_dim, w.group
    u = np.zeros(D, np.float32)
    u[D // 2 - 1] = u[D - 1] = np.float32(1 / np.sqrt(2))
    pos = 40 * 128 + 37
    q, k = x["q"].float(), x["k"].float()
    for g in range(w.n_kv_heads):
        q[:, g * G:(g + 1) * G, :] += 4.0 * torch.from_numpy(u)
        k[pos, g, :] += 175.0 * torch.from_numpy(u)
    x["q"], x["k"] = q.to(x["q"].dtype), k.to(x["k"].dtype)
    g = {n: t.cuda() for n, t in x.items()}
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    st = Stages(w)
    for s0, e in O.prefill_chunks(w):
        sel = orc.select_chunk(s0, e)
        st.keys(g["k"], g["v"], s0, e)
        vert, slash = st.estimate(g["q"], s0, e)
        torch.cuda.synchronize()
        q1m.check_status()
        gv, gs = vert.cpu().numpy(), slash.cpu().numpy()
        nR = len(O.estimator_rows(s0, e, w))
        if e > pos + 1:
            # the planted key takes nearly all of every estimator row's probability
            assert np.all(sel.vert[:, pos] > 0.99 * nR)
        for h in range(w.n_q_heads):
            rv, rs = mean_rel(gv[h], sel.vert[h]), mean_rel(gs[h], sel.slash[h])
            assert rv < 1e-3 and rs < 1e-3, (s0, h, rv, rs)
            assert abs(gv[h].sum() - nR) < 2e-3 * nR and abs(gs[h].sum() - nR) < 2e-3 * nR


def _gpu_select(w, st, vert, slash, e):
    V, S = st.select(torch.from_numpy(np.ascontiguousarray(vert)).cuda(),
                     torch.from_numpy(np.ascontiguousarray(slash)).cuda(), e)
    torch.cuda.synchronize()
    q1m.check_status()
    return V.cpu().numpy(), S.cpu().numpy()


@pytest.mark.parametrize("w", SPARSE, ids=lambda w: w.name)
def test_selection_bit_exact_on_oracle_scores(w):
    c = case(w)
    st = Stages(w)
    for sel in c["sels"]:
        V, S = _gpu_select(w, st, sel.vert, sel.slash, sel.e)
        for h in range(w.n_q_heads):
            assert np.array_equal(V[h], sel.V[h]), (sel.s0, h)
            assert np.array_equal(S[h], sel.S[h]), (sel.s0, h)


def test_selection_ties_and_budgets():
    """Quantised scores (many ties), zero scores, budgets at and above the candidate count."""
    g = np.random.default_rng(21)
    for e, nv, ns, fl in ((777, 50, 90, 64), (300, 300, 299, 5), (1000, 2000, 40, 64),
                          (5000, 1, 64, 64), (129, 17, 1, 1)):
        w = C.SMALL_SPARSE.with_(vs_vertical=nv, vs_slash=ns, vs_force_local=fl)
        st = Stages(w)
        vert = (np.round(g.random((w.n_q_heads, e)) * 7) / 7).astype(np.float32)
        slash = (np.round(g.random((w.n_q_heads, e)) * 3) / 3).astype(np.float32)
        vert[0, :] = 0.0
        V, S = _gpu_select(w, st, vert, slash, e)
        for h in range(w.n_q_heads):
            rv, rs = O.select_head(vert[h], slash[h], w)
            assert np.array_equal(V[h], rv) and np.array_equal(S[h], rs), (e, nv, ns, h)


def _unpack(mask_words, nkb):
    m = mask_words.astype(np.uint32)
    bits = (m[..., None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(*m.shape[:-1], -1)[..., :nkb].astype(bool)


def _seg_counts(blocks, b, w):
    Lb = O.dca_len(w) // 128
    cb = b // Lb
    kb = np.arange(len(blocks))
    seg = np.where(kb // Lb == cb, 0, np.where(kb // Lb == cb - 1, 1, 2))
    return [int(np.sum(blocks[: b + 1] & (seg[: b + 1] == x))) for x in range(3)]


@pytest.mark.parametrize("w", SPARSE, ids=lambda w: w.name)
def test_block_masks_bit_exact_on_oracle_selection(w):
    c = case(w)
    st = Stages(w)
    orc = c["orc"]
    for sel in c["sels"]:
        s0, e = sel.s0, sel.e
        V = torch.from_numpy(np.stack(sel.V).astype(np.int32)).cuda()
        S = torch.from_numpy(np.stack(sel.S).astype(np.int32)).cuda()
        mask, resid, cnt = st.masks(V, S, s0, e)
        torch.cuda.synchronize()
        q1m.check_status()
        nkb = (e + 127) // 128
        bits = _unpack(mask.cpu().numpy(), nkb)
        resid, cnt = resid.cpu().numpy(), cnt.cpu().numpy()
        L = O.dca_len(w)
        for h in range(w.n_q_heads):
            for qb in range((e - s0 + 127) // 128):
                b = s0 // 128 + qb
                ref = orc.blocks(h, b, sel)
                assert np.array_equal(bits[h, qb], ref), (s0, h, qb)
                rv = O.residual_verticals(sel.V[h], ref, b, e)
                assert cnt[h, qb, 6] == len(rv)
                assert np.array_equal(resid[h, qb, : len(rv)], rv), (s0, h, qb)
                assert list(cnt[h, qb, :3]) == _seg_counts(ref, b, w), (s0, h, qb)
                cb = b * 128 // L
                segs = [int(np.sum(rv // L == cb)), int(np.sum(rv // L == cb - 1)),
                        int(np.sum(rv // L <= cb - 2))]
                assert list(cnt[h, qb, 3:6]) == segs


def run_oracle_fed(w, c, out_dtype="f32"):
    """Stage pipeline with the oracle's selections fed to the GPU mask builder."""
    st = Stages(w, out_dtype)
    dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = torch.full((w.seq_len, w.n_q_heads, w.head_dim), float("nan"), dtype=dt, device="cuda")
    lse = torch.full((w.n_q_heads, w.seq_len), float("nan"), device="cuda")
    for sel in c["sels"]:
        s0, e = sel.s0, sel.e
        st.keys(c["g"]["k"], c["g"]["v"], s0, e)
        st.queries(c["g"]["q"], s0, e)
        if w.dense:
            st.attn(s0, e)
        else:
            V = torch.from_numpy(np.stack(sel.V).astype(np.int32)).cuda()
            S = torch.from_numpy(np.stack(sel.S).astype(np.int32)).cuda()
            mask, resid, cnt = st.masks(V, S, s0, e)
            st.attn(s0, e, mask, resid, cnt)
        st.merge(s0, e, out, lse)
    torch.cuda.synchronize()
    q1m.check_status()
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_matches_oracle_on_oracle_selection(w):
    c = case(w)
    out, lse = run_oracle_fed(w, c)
    ref = c["out"]
    assert np.all(np.isfinite(out))
    err = np.abs(out - ref)
    print(f"{w.name}: max-abs {err.max():.2e} mean-rel {mean_rel(out, ref):.2e} "
          f"lse max-abs {np.abs(lse - c['lse']).max():.2e}")
    if err.max() > MAX_ABS:
        per = err.reshape(-1, 128, w.n_q_heads, w.head_dim) if w.seq_len % 128 == 0 else None
        if per is not None:
            print("per (block, head) max error:", np.round(per.max(axis=(1, 3)), 4).tolist())
    assert err.max() <= MAX_ABS
    assert mean_rel(out, ref) <= MEAN_REL
    assert np.abs(lse - c["lse"]).max() <= 2e-3


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_layer_end_to_end(w):
    """The product entry point (own estimator and selection) against the oracle."""
    c = case(w)
    layer = Layer(w)
    lse = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    out = layer(c["g"]["q"], c["g"]["k"], c["g"]["v"], lse=lse)
    torch.cuda.synchronize()
    q1m.check_status()
    out = out.cpu().numpy()
    ref = c["out"]
    err = np.abs(out - ref)
    print(f"{w.name}: end-to-end max-abs {err.max():.2e} mean-rel {mean_rel(out, ref):.2e}")
    assert err.max() <= MAX_ABS
    assert mean_rel(out, ref) <= MEAN_REL


@pytest.mark.parametrize("w", [C.SMALL_SPARSE, C.TINY_2K], ids=lambda w: w.name)
def test_bf16_output(w):
    c = case(w)
    out, _ = run_oracle_fed(w, c, "bf16")
    ref = torch.from_numpy(c["out"]).to(torch.bfloat16).float().numpy()
    assert np.abs(out - ref).max() <= MAX_ABS
    assert mean_rel(out, ref) <= MEAN_REL


def test_lse_merge_identity():
    g = np.random.default_rng(5)
    hq, rows, d = 3, 200, 128
    ld = 256
    outs = g.standard_normal((3, hq, ld, d)).astype(np.float32)
    lses = (g.standard_normal((3, hq, ld)) * 4).astype(np.float32)
    lses[1, :, 7] = -np.inf
    w = C.SMALL_SPARSE
    o = torch.empty(rows, hq, d, device="cuda")
    l = torch.empty(hq, rows, device="cuda")
    q1m.lse_merge(torch.from_numpy(outs).cuda(), torch.from_numpy(lses).cuda(), 3, ld, 0, rows,
                  rows, hq, d, q1m.F32, None, o, l)
    torch.cuda.synchronize()
    for h in range(hq):
        ro, rl = O.lse_merge(outs[:, h, :rows].astype(np.float64),
                             lses[:, h, :rows].astype(np.float64) * np.log(2.0))
        assert np.abs(o[:, h].cpu().numpy() - ro).max() < 1e-5
        assert np.abs(l[h].cpu().numpy() - rl).max() < 1e-5


def test_bounded_wait_returns_timeout_and_library_recovers():
    st = q1m.selftest_wait_timeout(2_000_000)
    assert st == -5
    assert q1m.status_poll() == 0
    # the context is still usable
    w = C.TINY_2K
    c = case(w)
    out = Layer(w)(c["g"]["q"], c["g"]["k"], c["g"]["v"])
    torch.cuda.synchronize()
    q1m.check_status()
    assert np.abs(out.cpu().numpy() - c["out"]).max() <= MAX_ABS


def test_fma_pipe_exp2_error_bound():
    """The kernel's polynomial 2^x against CUDA's exp2f and fp64, over the range the
    softmax feeds it (x - max <= 8 by the lazy rescale; very negative values underflow)."""
    xs = np.concatenate([np.linspace(-130.0, 8.0, 1_000_003), np.arange(-127, 9, dtype=np.float64),
                         np.arange(-127, 9) + 0.5, [-np.inf]]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    yp, ym, yr = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    q1m.selftest_exp2(x, yp, ym, yr)
    torch.cuda.synchronize()
    yp, yr = yp.cpu().numpy().astype(np.float64), yr.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    normal = xs >= -126.0
    rel = np.abs(yp[normal] - ref[normal]) / ref[normal]
    assert rel.max() < 4e-6, rel.max()
    assert np.abs(yr[normal] - ref[normal]).max() / ref[normal].max() < 1e-6
    # below -126 the result is tiny (no wrap-around), as is 2^-inf
    assert np.all(yp[~normal] >= 0) and np.all(yp[~normal] < 1.2e-38)


@pytest.mark.parametrize("w", SPARSE, ids=lambda w: w.name)
def test_attention_recall_matches_oracle(w):
    """recall_i = exp(lse_sparse - lse_dense) from the GPU against the oracle's share of the
    dense softmax mass kept by A(i), on the oracle's selection."""
    c = case(w)
    _, lse_s = run_oracle_fed(w, c)
    wd = w.with_(vs_vertical=0, vs_slash=0)
    lse_d = torch.empty(w.n_q_heads, w.seq_len, device="cuda")
    Layer(wd)(c["g"]["q"], c["g"]["k"], c["g"]["v"], lse=lse_d)
    r = torch.empty_like(lse_d)
    q1m.attention_recall(torch.from_numpy(lse_s).cuda(), lse_d, r)
    torch.cuda.synchronize()
    q1m.check_status()
    r = r.cpu().numpy()
    g = np.random.default_rng(3)
    orc = c["orc"]
    for sel in c["sels"]:
        for h in range(w.n_q_heads):
            rows = np.sort(g.choice(np.arange(sel.s0, sel.e), size=16, replace=False))
            ref = orc.recall_rows(rows, h, sel)
            assert np.abs(r[h, rows] - ref).max() < 5e-3, (sel.s0, h)
    assert np.all((r > 0) & (r <= 1.0))

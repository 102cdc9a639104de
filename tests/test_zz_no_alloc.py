"""The allocation-free attention entry point (q1m_block_sparse_attn_noalloc).

Some callers cannot allocate device memory on this path: a memory planner or pool owns every
allocation, or the calling thread must never wait on the allocator. For them the library
keeps the attention stage's only scratch, its work-unit list, in a static device array. This
test calls that entry point through the C ABI twice in a row and checks each result against
the entry point that takes caller-provided scratch, within the tolerance the other parity
tests use, on a sparse workload (gathered residual columns, several chunks) and a dense one.
It lives in its own file that pytest collects last and works alone or after the other tests.
"""
import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Stages
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_REL = 2e-2, 1e-3


def _chunk_inputs(w, st, g, s0, e):
    st.keys(g["k"], g["v"], s0, e)
    st.queries(g["q"], s0, e)
    if w.dense:
        return None, None, None
    vert, slash = st.estimate(g["q"], s0, e)
    V, S = st.select(vert, slash, e)
    return st.masks(V, S, s0, e)


@pytest.mark.parametrize("w", [C.SMALL_SPARSE, C.TINY_2K], ids=lambda w: w.name)
def test_noalloc_matches_scratch_entry_point_on_two_calls(w):
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    st = Stages(w)
    for s0 in range(0, w.seq_len, w.prefill_chunk):
        e = min(w.seq_len, s0 + w.prefill_chunk)
        mask, resid, cnt = _chunk_inputs(w, st, g, s0, e)
        # the kernels write only the partials of patterns a row has keys in: start from NaN
        st.o_part.fill_(float("nan"))
        st.lse_part.fill_(float("nan"))
        st.attn(s0, e, mask, resid, cnt)
        torch.cuda.synchronize()
        q1m.check_status()
        rows = e - s0
        ref_o = st.o_part[:, :, :rows].clone()
        ref_l = st.lse_part[:, :, :rows].clone()
        if resid is not None and resid.shape[-1] == 0:
            resid = torch.empty(w.n_q_heads, mask.shape[1], 1, dtype=torch.int32, device="cuda")
        for call in range(2):
            o_part = torch.full_like(st.o_part, float("nan"))
            lse_part = torch.full_like(st.lse_part, float("nan"))
            q1m.block_sparse_attn_noalloc(st.qv, st.ld_rows, st.k_rot, st.v16, st.ld_tokens, mask,
                                          resid.contiguous() if resid is not None else None, cnt,
                                          s0, e, w.n_q_heads, w.n_kv_heads, w.head_dim, st.p,
                                          o_part, lse_part)
            torch.cuda.synchronize()
            q1m.check_status()
            got_l = lse_part[:, :, :rows]
            # the same partials written, the same empty (-inf) ones
            assert torch.equal(torch.isnan(got_l), torch.isnan(ref_l)), (s0, call)
            finite = torch.isfinite(ref_l)
            assert torch.equal(torch.isfinite(got_l), finite), (s0, call)
            assert finite.any()
            assert (got_l[finite] - ref_l[finite]).abs().max().item() <= 2e-3
            vo = finite[..., None].expand_as(ref_o)
            a = o_part[:, :, :rows][vo].cpu().numpy()
            b = ref_o[vo].cpu().numpy()
            assert np.abs(a - b).max() <= MAX_ABS, (s0, call)
            assert np.abs(a - b).sum() <= MEAN_REL * np.abs(b).sum(), (s0, call)


# One Q head and one KV head, D = 64, dense: the smallest layer whose prefill chunk reaches
# the static list's limit (about 2 GB of device buffers).
LIMIT = C.Workload(
    name="noalloc-limit", seq_len=128 * 10916, n_q_heads=1, n_kv_heads=1, head_dim=64,
    in_dtype="bf16", rope_base=1e7, dca_chunk=262144, local_window=4096, yarn_s=4.0,
    prefill_chunk=128 * 10916, vs_vertical=0, vs_slash=0, seed=C.SEED_BASE + 40)


@pytest.mark.parametrize("nqb", [8193, 10916], ids=["8193-blocks", "limit-blocks"])
def test_noalloc_at_its_largest_chunks(nqb):
    """A chunk past 8,192 query blocks (its work-unit sort then needs more than the default
    48 KB of shared memory) and a chunk of exactly the largest size the static list holds:
    the allocation-free call, twice, against the scratch entry point, and a few rows of the
    merged result against the fp64 oracle."""
    from oracle import dca_vs as O
    w = LIMIT
    e = 128 * nqb
    assert nqb <= q1m.NOALLOC_MAX_QUERY_BLOCKS
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    st = Stages(w)
    st.keys(g["k"], g["v"], 0, e)
    st.queries(g["q"], 0, e)
    st.o_part.fill_(float("nan"))
    st.lse_part.fill_(float("nan"))
    st.attn(0, e)
    torch.cuda.synchronize()
    q1m.check_status()
    ref_o, ref_l = st.o_part[:, :, :e].clone(), st.lse_part[:, :, :e].clone()
    finite = torch.isfinite(ref_l)
    assert finite[0].all()       # every row has intra keys
    vo = finite[..., None].expand_as(ref_o)
    b = ref_o[vo]
    for call in range(2):
        st.o_part.fill_(float("nan"))
        st.lse_part.fill_(float("nan"))
        q1m.block_sparse_attn_noalloc(st.qv, st.ld_rows, st.k_rot, st.v16, st.ld_tokens, None,
                                      None, None, 0, e, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                      st.p, st.o_part, st.lse_part)
        torch.cuda.synchronize()
        q1m.check_status()
        got_l = st.lse_part[:, :, :e]
        assert torch.equal(torch.isfinite(got_l), finite), call
        assert (got_l[finite] - ref_l[finite]).abs().max().item() <= 2e-3, call
        a = st.o_part[:, :, :e][vo]
        assert (a - b).abs().max().item() <= MAX_ABS, call
        assert (a - b).abs().sum().item() <= MEAN_REL * b.abs().sum().item(), call
    del ref_o, ref_l, vo, b, a
    out = torch.full((w.seq_len, 1, w.head_dim), float("nan"), device="cuda")
    st.merge(0, e, out)
    torch.cuda.synchronize()
    q1m.check_status()
    rows = np.unique(np.concatenate([[0, 127, 128, e - 129, e - 1],
                                     np.random.default_rng(nqb).integers(0, e, 5)]))
    orc = O.Oracle(x["q"][:e], x["k"][:e], x["v"][:e], w)
    ref, _ = orc.attend_rows(rows, 0, orc.select_chunk(0, e))
    got = out[torch.from_numpy(rows).cuda(), 0].cpu().numpy()
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS and err.sum() <= MEAN_REL * np.abs(ref).sum(), err.max()


def test_noalloc_rejects_chunks_beyond_its_static_list():
    """One query block more than the static list holds: refused by the size check, which
    comes before every other check. Every pointer is NULL, so no call of this test can reach
    a launch even if that order changed (the NULL check would refuse it instead)."""
    import ctypes
    w = C.SMALL_DENSE_D128
    e = 128 * (q1m.NOALLOC_MAX_QUERY_BLOCKS + 1)
    p = q1m.params(w.with_(prefill_chunk=e))
    lib = q1m.library()
    st = lib.q1m_block_sparse_attn_noalloc(None, e, None, None, e, None, None, None, 0, e,
                                           w.n_q_heads, w.n_kv_heads, w.head_dim,
                                           ctypes.byref(p), None, None, None)
    assert st == -2, lib.q1m_last_error()
    assert b"exceeds" in lib.q1m_last_error()

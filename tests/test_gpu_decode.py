"""DCA decode attention (q1m_dca_decode) against the fp64 oracle's decode row: runs of
decode steps from an empty cache and after a prefill of the cache, across 32-key tile and
DCA chunk boundaries, for G = 1, 2, 5, 8 query heads per KV head and D = 64 / 128; the
appended cache rows against the prefill's key rotation, bit for bit; the range check; and
the 7B-shape token at position 1,048,575 on sampled heads."""
import numpy as np
import pytest
import torch

from long_context_prefill_dca_b200 import q1m
from long_context_prefill_dca_b200.layer import Stages
from oracle import dca_vs as O
from synth import configs as C
from synth import inputs as I

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_REL = 2e-2, 1e-3

BASE = C.Workload(name="dec", seq_len=1300, n_q_heads=4, n_kv_heads=2, head_dim=128,
                  in_dtype="bf16", rope_base=1e4, dca_chunk=512, local_window=128, yarn_s=2.0,
                  prefill_chunk=1408, vs_vertical=0, vs_slash=0, sinks=4, bands=2,
                  band_hi=300, seed=0x5EED0200)
CASES = [
    (BASE, 1100, 1200),                                                     # crosses 3L = 1152
    (BASE.with_(name="dec-g1-d64", n_q_heads=3, n_kv_heads=3, head_dim=64, in_dtype="f32"), 370, 420),
    (BASE.with_(name="dec-g8", n_q_heads=8, n_kv_heads=1, seq_len=900), 760, 800),   # crosses 2L
    (BASE.with_(name="dec-g5", n_q_heads=10, n_kv_heads=2, seq_len=700), 0, 40),       # from empty
]


def rel(a, b):
    return float(np.sum(np.abs(a - b)) / max(np.sum(np.abs(b)), 1e-30))


def decode_run(w, x, g, p0, p1, st=None):
    st = st or Stages(w)
    if p0 > 0:
        st.keys(g["k"], g["v"], 0, p0)
    outs, lses = [], []
    for pos in range(p0, p1):
        out = torch.empty(w.n_q_heads, w.head_dim, device="cuda")
        lse = torch.empty(w.n_q_heads, device="cuda")
        st.decode(g["q"][pos], g["k"][pos], g["v"][pos], pos, out, lse)
        outs.append(out)
        lses.append(lse)
    torch.cuda.synchronize()
    q1m.check_status()
    return st, torch.stack(outs).cpu().numpy(), torch.stack(lses).cpu().numpy()


@pytest.mark.parametrize("w,p0,p1", CASES, ids=[c[0].name + f"-{c[1]}-{c[2]}" for c in CASES])
def test_decode_steps_match_oracle(w, p0, p1):
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    _, got, got_lse = decode_run(w, x, g, p0, p1)
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    ref = np.zeros_like(got)
    ref_lse = np.zeros_like(got_lse)
    for r, pos in enumerate(range(p0, p1)):
        for h in range(w.n_q_heads):
            ref[r, h], ref_lse[r, h] = orc.decode_row(pos, h)
    err = np.abs(got - ref)
    print(f"{w.name}: {p1 - p0} steps, max-abs {err.max():.2e} mean-rel {rel(got, ref):.2e}")
    assert np.all(np.isfinite(got))
    assert err.max() <= MAX_ABS and rel(got, ref) <= MEAN_REL
    assert np.abs(got_lse - ref_lse).max() <= 2e-3


def test_decode_appends_the_prefill_rotation():
    """Rows written by decode steps equal the prefill's key rotation of the same tokens."""
    w = BASE
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    st, _, _ = decode_run(w, x, g, 1000, 1070)
    ref = Stages(w)
    ref.keys(g["k"], g["v"], 0, 1070)
    torch.cuda.synchronize()
    assert torch.equal(st.k_rot[:, :1070], ref.k_rot[:, :1070])
    assert torch.equal(st.v16[:, :1070], ref.v16[:, :1070])
    # the rest of the last token's 32-key tile is zeroed
    assert int(st.k_rot[:, 1070:1088].abs().sum()) == 0 and int(st.v16[:, 1070:1088].abs().sum()) == 0


def test_decode_range_check():
    w = BASE.with_(in_dtype="f32")
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    st = Stages(w)
    st.keys(g["k"], g["v"], 0, 50)
    kk = g["k"][50].clone()
    kk[1, 3] = 1e30
    out = torch.empty(w.n_q_heads, w.head_dim, device="cuda")
    st.decode(g["q"][50], kk, g["v"][50], 50, out)
    assert q1m.status_poll() == -6
    assert q1m.status_poll() == 0


@pytest.mark.slow
def test_decode_full_size_last_token():
    """The 7B shape: the token at position 1,048,575 after the 1,048,575-token cache."""
    w = C.L7B_1M.with_(vs_vertical=0, vs_slash=0)
    x = I.generate(w)
    g = {k: t.cuda() for k, t in x.items()}
    n = w.seq_len
    st = Stages(w)
    st.keys(g["k"], g["v"], 0, n - 1)
    out = torch.empty(w.n_q_heads, w.head_dim, device="cuda")
    lse = torch.empty(w.n_q_heads, device="cuda")
    st.decode(g["q"][n - 1], g["k"][n - 1], g["v"][n - 1], n - 1, out, lse)
    torch.cuda.synchronize()
    q1m.check_status()
    orc = O.Oracle(x["q"], x["k"], x["v"], w)
    got, gl = out.cpu().numpy(), lse.cpu().numpy()
    for h in (0, w.n_q_heads - 1):
        ref, rl = orc.decode_row(n - 1, h)
        err = np.abs(got[h] - ref)
        print(f"7b-1m decode head {h}: max-abs {err.max():.2e} rel {rel(got[h], ref):.2e}")
        assert err.max() <= MAX_ABS and rel(got[h], ref) <= MEAN_REL and abs(gl[h] - rl) <= 2e-3

"""Plant plausible mistakes in the oracle (CPU only) and require that a pin catches each.

This shows the pins in test_oracle_pins.py are sensitive: a dropped term, a wrong sign,
an off-by-one in the DCA remap, the mask or the selection each fails at least one check.
"""
import math

import numpy as np
import pytest

from oracle import dca_vs as O
from tests import oracle_checks as C


def _all_checks():
    """name -> True when the check passes."""
    res = {}
    res["yarn"] = C.check_yarn_golden() < 1e-12
    res["rope_tf"] = C.check_rope_vs_transformers() < 2e-4
    res["rope_cplx"] = C.check_rope_complex() < 1e-12
    res["dca_brute"] = C.check_dca_brute_force() < 1e-10
    res["dca_inv"] = C.check_dca_invariants()
    res["short"] = C.check_short_equals_causal_rope() < 1e-10
    res["v_ones"] = C.check_v_ones() < 1e-12
    res["full_budget"] = C.check_full_budget_is_dense() < 1e-12
    res["est_mass"] = C.check_estimator_mass() < 1e-5
    res["est_brute"] = C.check_estimator_brute_force() < 1e-6
    res["topk"] = C.check_topk_properties()
    res["force"] = C.check_force_local()
    res["mask"] = C.check_mask_brute_force()
    res["attended"] = C.check_attended_set()
    res["chunks"] = _passes(C.check_equal_cost_chunks)
    res["decode"] = C.check_decode_row() < 1e-10
    res["rope_rel"] = C.check_rope_relative() < 1e-10
    res["causal"] = C.check_causal() < 1e-12
    res["lse_merge"] = C.check_lse_merge() < 1e-12
    res["recall"] = C.check_recall() < 1e-12
    res["key_order"] = C.check_key_order_invariance() < 1e-12
    res["residual"] = C.check_residual_verticals()
    res["fixed_chunks"] = C.check_fixed_chunks()
    return res


def _passes(check) -> bool:
    try:
        check()
        return True
    except AssertionError:
        return False


def _chunks_variant(cost_of_block, ceil_target=True, drop_repeats=True):
    def chunks(n, K):
        nb = -(-n // O.BLOCK)
        cum, total = [], 0
        for b in range(nb):
            total += cost_of_block(b)
            cum.append(total)
        import bisect
        cuts = []
        for k in range(1, K):
            need = -(-k * total // K) if ceil_target else k * total // K
            m = bisect.bisect_left(cum, need) + 1
            if not drop_repeats or not cuts or m > cuts[-1]:
                cuts.append(m)
        rows = [min(n, O.BLOCK * m) for m in cuts if m < nb] + [n]
        s0 = 0
        for e in rows:
            yield s0, e
            s0 = e
    return chunks


def _rope_sign(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * O.rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _rope_interleaved(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * O.rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _theta_wrong(d, base):
    f = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -f / d)


def _len_is_c(cfg):
    return cfg.dca_chunk


def _succ_clamp_c(i, pattern, cfg):
    L, c = O.dca_len(cfg), cfg.dca_chunk
    t = np.asarray(i) % L
    if pattern == O.INTRA:
        return t
    if pattern == O.SUCC:
        return np.minimum(t + L, c)
    return np.full_like(t, c - 1)


def _inter_at_c(i, pattern, cfg):
    L, c = O.dca_len(cfg), cfg.dca_chunk
    t = np.asarray(i) % L
    if pattern == O.INTRA:
        return t
    if pattern == O.SUCC:
        return np.minimum(t + L, c - 1)
    return np.full_like(t, c)


def _yarn_unsquared(s):
    return 1.0 if s <= 1.0 else 0.1 * math.log(s) + 1.0


def _scale_no_sqrt_d(cfg):
    return O.yarn_inv_t(cfg.yarn_s)


def _estimate_slash_unreversed(q_R, R, krot_g, e, cfg):
    js = np.arange(e)
    l = O.dca_logits(q_R, R, krot_g[:e], js, cfg)
    l = np.where(js[None, :] <= R[:, None], l, -np.inf)
    p, lse = O.softmax_rows(l)
    slash = np.zeros(e)
    for r, i in enumerate(R):
        slash[: i + 1] += p[r, : i + 1]
    return np.sum(p, 0).astype(np.float32), slash.astype(np.float32), lse


def _estimator_rows_off(s0, e, cfg):
    return np.arange(max(s0, e - cfg.vs_last_q - 1), e - 1)


def _blocks_off_by_one(S, b, e, bs=O.BLOCK):
    nkb = (e + bs - 1) // bs
    r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
    o = np.asarray(S, dtype=np.int64)
    o = o[o <= r1]
    lo, hi = np.maximum(0, r0 - o) // bs, (r1 - o) // bs
    m = np.zeros(nkb, dtype=bool)
    for a, z in zip(lo, hi):
        m[a: z] = True          # drops the last block of each range
    return m


def _top_ties_reversed(scores, budget):
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    if budget >= n:
        return np.arange(n)
    order = np.lexsort((-np.arange(n), -scores))
    return np.sort(order[:budget])


def _select_no_force(vert, slash, cfg):
    return O.top_budget(vert, cfg.vs_vertical), O.top_budget(slash, cfg.vs_slash)


def _attended_without_verticals(i, blocks, V, bs=O.BLOCK):
    js = np.arange(i + 1)
    return blocks[js // bs].copy()


def _key_at_j(j, cfg):
    return np.asarray(j)


def _softmax_unnormalised(l):
    m = np.max(l, axis=1, keepdims=True)
    p = np.exp(l - m)
    return p, (m + np.log(np.sum(p, axis=1, keepdims=True)))[:, 0]


def _merge_unnormalised(outs, lses):
    m = np.max(lses, axis=0)
    w = np.exp(lses - m[None, :])
    return np.sum(w[:, :, None] * outs, axis=0), m + np.log(np.sum(w, axis=0))


def _estimate_not_causal(q_R, R, krot_g, e, cfg):
    js = np.arange(e)
    p, lse = O.softmax_rows(O.dca_logits(q_R, R, krot_g[:e], js, cfg))
    slash = np.zeros(e, dtype=np.float64)
    for r, i in enumerate(R):
        slash[: i + 1] += p[r, i::-1]
    return np.sum(p, axis=0).astype(np.float32), slash.astype(np.float32), lse


def _residual_inside_blocks(V, blocks, b, e, bs=O.BLOCK):
    V = np.asarray(V)
    return V[V <= min(b * bs + bs - 1, e - 1)]


def _residual_cut_early(V, blocks, b, e, bs=O.BLOCK):
    r1 = min(b * bs + bs - 1, e - 1)
    V = np.asarray(V)
    return V[(V < r1) & ~blocks[np.minimum(V // bs, blocks.shape[0] - 1)]]


def _decode_without_own_key(self, pos, h):
    js = np.arange(max(pos, 1))
    l = O.dca_logits(self.q_rows(np.array([pos]), h), np.array([pos]),
                     self.krot(h // self.cfg.group)[: len(js)], js, self.cfg)
    p, lse = O.softmax_rows(l)
    return (p @ self.v[: len(js), h // self.cfg.group, :])[0], float(lse[0])


def _recall_squared(self, rows, h, sel):
    rows = np.asarray(rows)
    imax = int(rows.max())
    js = np.arange(imax + 1)
    l = O.dca_logits(self.q_rows(rows, h), rows, self.krot(h // self.cfg.group)[: imax + 1],
                     js, self.cfg)
    res = np.zeros(len(rows))
    for r, i in enumerate(rows):
        p, _ = O.softmax_rows(l[[r], : i + 1])
        res[r] = float(np.sum(p[0][self.attended(int(i), h, sel)])) ** 2
    return res


def _pattern_wrong_neighbour(i, j, cfg):
    L = O.dca_len(cfg)
    ci, cj = np.asarray(i) // L, np.asarray(j) // L
    return np.where(ci == cj, O.INTRA, np.where(cj == ci - 2, O.SUCC, O.INTER))


def _blocks_no_clamp(S, b, e, bs=O.BLOCK):
    nkb = (e + bs - 1) // bs
    r0, r1 = b * bs, min(b * bs + bs - 1, e - 1)
    o = np.asarray(S, dtype=np.int64)
    o = o[o <= r1]
    lo, hi = (r0 - o) // bs, (r1 - o) // bs
    cnt = np.zeros(nkb + 1, dtype=np.int64)
    np.add.at(cnt, lo, 1)            # a negative start wraps to the end of the array
    np.add.at(cnt, hi + 1, -1)
    return np.cumsum(cnt)[:nkb] > 0


def _top_unsorted(scores, budget):
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    if budget >= n:
        return np.arange(n, dtype=np.int64)
    return np.lexsort((np.arange(n), -scores))[:budget].astype(np.int64)


def _softmax_lse_base2(l):
    m = np.max(l, axis=1, keepdims=True)
    p = np.exp(l - m)
    s = np.sum(p, axis=1, keepdims=True)
    return p / s, (m + np.log2(s))[:, 0]


def _estimator_single_row(s0, e, cfg):
    return np.arange(e - 1, e)


def _forced_on_top_of_budget(vert, slash, cfg):
    S = O.top_budget(slash, cfg.vs_slash)
    return (O.top_budget(vert, cfg.vs_vertical),
            np.union1d(S, np.arange(min(cfg.vs_force_local, len(slash)))).astype(np.int64))


def _intra_query_unwrapped(i, pattern, cfg):
    if pattern == O.INTRA:
        return np.asarray(i)
    L, c = O.dca_len(cfg), cfg.dca_chunk
    t = np.asarray(i) % L
    return np.minimum(t + L, c - 1) if pattern == O.SUCC else np.full_like(t, c - 1)


def _fixed_chunks_one_row_longer(cfg):
    if getattr(cfg, "equal_cost_chunks", 0) > 0:
        yield from O.equal_cost_chunks(cfg.seq_len, cfg.equal_cost_chunks)
        return
    for s0 in range(0, cfg.seq_len, cfg.prefill_chunk + 1):
        yield s0, min(cfg.seq_len, s0 + cfg.prefill_chunk + 1)


MUTATIONS = [
    ("rope sign flipped", "rope", _rope_sign),
    ("rope pairs interleaved", "rope", _rope_interleaved),
    ("rope frequency exponent halved", "rope_theta", _theta_wrong),
    ("DCA chunk length c instead of c - w", "dca_len", _len_is_c),
    ("successive query clamped at c", "dca_query_position", _succ_clamp_c),
    ("inter query at c", "dca_query_position", _inter_at_c),
    ("YaRN factor not squared", "yarn_inv_t", _yarn_unsquared),
    ("logit scale without 1/sqrt(D)", "logit_scale", _scale_no_sqrt_d),
    ("slash offsets not reversed", "estimate_head", _estimate_slash_unreversed),
    ("estimator rows shifted by one", "estimator_rows", _estimator_rows_off),
    ("mask drops the last block of a slash range", "computed_blocks", _blocks_off_by_one),
    ("top-k ties broken towards larger index", "top_budget", _top_ties_reversed),
    ("forced local diagonals dropped", "select_head", _select_no_force),
    ("vertical columns left out of the attended set", "attended_mask",
     _attended_without_verticals),
    ("chunk cost of block b taken as b", "equal_cost_chunks", _chunks_variant(lambda b: b)),
    ("chunk cost of block b taken as 1", "equal_cost_chunks", _chunks_variant(lambda b: 1)),
    ("chunk target rounded down", "equal_cost_chunks", _chunks_variant(lambda b: b + 1, ceil_target=False)),
    ("repeated chunk boundaries kept", "equal_cost_chunks",
     _chunks_variant(lambda b: b + 1, drop_repeats=False)),
    ("keys rotated at j instead of j mod L", "dca_key_position", _key_at_j),
    ("softmax weights not normalised", "softmax_rows", _softmax_unnormalised),
    ("LSE merge weights not normalised", "lse_merge", _merge_unnormalised),
    ("estimator softmax not causal", "estimate_head", _estimate_not_causal),
    ("residual verticals keep columns inside computed blocks", "residual_verticals",
     _residual_inside_blocks),
    ("residual verticals stop one row early", "residual_verticals", _residual_cut_early),
    ("decode step leaves out the token's own key", "Oracle.decode_row", _decode_without_own_key),
    ("recall squared", "Oracle.recall_rows", _recall_squared),
    ("successive pattern taken two chunks back", "dca_pattern", _pattern_wrong_neighbour),
    ("slash block range not clamped at key block 0", "computed_blocks", _blocks_no_clamp),
    ("selected indices not in ascending order", "top_budget", _top_unsorted),
    ("log-sum-exp in base 2", "softmax_rows", _softmax_lse_base2),
    ("estimator reads only the last row", "estimator_rows", _estimator_single_row),
    ("forced diagonals added on top of the slash budget", "select_head", _forced_on_top_of_budget),
    ("intra query at i instead of i mod L", "dca_query_position", _intra_query_unwrapped),
    ("fixed prefill chunks one row longer", "prefill_chunks", _fixed_chunks_one_row_longer),
]


@pytest.mark.parametrize("name,attr,fn", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(monkeypatch, name, attr, fn):
    owner = O
    for part in attr.split(".")[:-1]:
        owner = getattr(owner, part)
    monkeypatch.setattr(owner, attr.split(".")[-1], fn)
    res = _all_checks()
    failed = [k for k, ok in res.items() if not ok]
    assert failed, f"no pin caught the planted mistake: {name}"

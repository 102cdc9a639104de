"""The attended-pair count behind the benchmark's effective TFLOP/s, computed from the mask
kernel's per-(head, query block) counts, equals Σ|A(i)| over the oracle's attended sets
(CPU only)."""
import numpy as np
import pytest

from long_context_prefill_dca_b200 import accounting as A
from oracle import dca_vs as O


def _counts_and_truth(rng, s0, e, hq, force):
    """cnt [hq][nqb][8] laid out as the mask stage writes it (blocks per DCA pattern, residual
    columns per pattern, total residuals, 0) from random selections, and the oracle's
    Σ|A(i)| over rows [s0, e) of every head."""
    bs = O.BLOCK
    nqb = -(-(e - s0) // bs)
    cnt = np.zeros((hq, nqb, 8), dtype=np.int32)
    truth = 0
    for h in range(hq):
        V = np.sort(rng.choice(e, size=min(e, int(rng.integers(0, 30))), replace=False))
        S = np.union1d(np.arange(min(force, e)),
                       rng.choice(e, size=min(e, int(rng.integers(0, 20))), replace=False))
        for qb in range(nqb):
            b = s0 // bs + qb
            blocks = O.computed_blocks(S, b, e)
            res = O.residual_verticals(V, blocks, b, e)
            nblk = int(blocks.sum())
            # split the blocks over the three patterns arbitrarily: only their sum counts
            cnt[h, qb, 0], cnt[h, qb, 1] = nblk // 2, nblk - nblk // 2
            cnt[h, qb, 3], cnt[h, qb, 5] = len(res) // 3, len(res) - len(res) // 3
            cnt[h, qb, 6] = len(res)
            for i in range(b * bs, min(b * bs + bs, e)):
                truth += int(O.attended_mask(i, blocks, V).sum())
    return cnt, truth


@pytest.mark.parametrize("s0,e", [(0, 1), (0, 5), (0, 128), (0, 700), (256, 700), (384, 1111),
                                  (128, 129)])
def test_pairs_from_counts_equals_the_oracle_attended_sets(s0, e):
    rng = np.random.default_rng(1000 * s0 + e)
    cnt, truth = _counts_and_truth(rng, s0, e, hq=3, force=1 + int(rng.integers(0, 8)))
    assert A.pairs_from_counts(cnt, s0, e) == truth


def test_dense_pairs_is_the_causal_count():
    for s0, e, hq in [(0, 1, 1), (0, 1000, 4), (512, 1500, 7)]:
        assert A.dense_pairs(s0, e, hq) == hq * sum(i + 1 for i in range(s0, e))


def test_full_selection_counts_every_causal_pair():
    """With every offset selected each row attends all j <= i: the count is dense."""
    s0, e, hq = 256, 900, 2
    bs = O.BLOCK
    nqb = -(-(e - s0) // bs)
    cnt = np.zeros((hq, nqb, 8), dtype=np.int32)
    for qb in range(nqb):
        cnt[:, qb, 0] = s0 // bs + qb + 1
    assert A.pairs_from_counts(cnt, s0, e) == A.dense_pairs(s0, e, hq)

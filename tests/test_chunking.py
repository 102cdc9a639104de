"""Chunked-prefill boundaries: the library's q1m_prefill_bounds (host code, no GPU needed)
against the oracle's own implementation, bit for bit, in both the fixed-size and the
equal-cost mode."""
import numpy as np
import pytest

from long_context_prefill_dca_b200 import q1m
from oracle import dca_vs as O
from synth import configs as C


def test_bounds_match_oracle_fixed_and_equal_cost():
    rng = np.random.default_rng(11)
    base = C.SMALL_SPARSE
    for _ in range(300):
        n = int(rng.integers(1, 3_000_000))
        if rng.random() < 0.5:
            w = base.with_(seq_len=n, prefill_chunk=128 * int(rng.integers(1, 2048)))
        else:
            w = base.with_(seq_len=n, equal_cost_chunks=int(rng.integers(1, 64)))
        assert q1m.prefill_bounds(w) == list(O.prefill_chunks(w)), (n, w.prefill_chunk, w.equal_cost_chunks)


def test_bounds_at_the_benchmark_size():
    w = C.L7B_1M.with_(equal_cost_chunks=8)
    b = q1m.prefill_bounds(w)
    assert b == list(O.prefill_chunks(w)) and len(b) == 8 and b[-1][1] == w.seq_len


def test_bounds_reject_bad_params():
    with pytest.raises(q1m.Q1MError):
        q1m.prefill_bounds(C.SMALL_SPARSE.with_(equal_cost_chunks=-1))
    with pytest.raises(q1m.Q1MError):
        q1m.prefill_bounds(C.SMALL_SPARSE.with_(prefill_chunk=100))


@pytest.mark.parametrize("n,K", [((1 << 28) - 1, 7), ((1 << 27) + 77, 1000), (1 << 26, 1),
                                 (5000, 4096), (129, 3)])
def test_equal_cost_bounds_at_extreme_sizes(n, K):
    """Near the library's largest sequence (2^28 rows: 128-bit cost arithmetic on the C side,
    Python integers in the oracle) and with more chunks than blocks (dropped boundaries)."""
    w = C.SMALL_SPARSE.with_(seq_len=n, equal_cost_chunks=K)
    got = q1m.prefill_bounds(w)
    assert got == list(O.prefill_chunks(w))
    assert got[-1][1] == n and len(got) <= min(K, -(-n // 128))

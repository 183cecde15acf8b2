"""The fp64 oracle against what the pages and the mathematics fix (no GPU)."""
import pytest

import oracle
from tests import pin_suite


@pytest.mark.parametrize("name", sorted(pin_suite.PINS))
def test_oracle_pin(name):
    pin_suite.PINS[name](oracle.attention)


def test_oracle_thread_count_invariance():
    """Rows are computed by one thread each, so any thread count gives the same bits."""
    import numpy as np
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((2, 3, 37, 8)) for _ in range(3))
    a = oracle.attention(q, k, v, scale=0.3, causal=True, nthreads=1)
    b = oracle.attention(q, k, v, scale=0.3, causal=True, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_oracle_rejects_bad_arguments():
    import numpy as np
    q = np.zeros((1, 3, 4, 2))
    k = np.zeros((1, 2, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention(q, k, k, scale=1.0)  # 3 query heads over 2 kv heads
    with pytest.raises(ValueError):
        oracle.attention(np.zeros((1, 2, 4, 2)), k, k, scale=1.0, rows=[8])  # row out of range


def test_flop_conventions():
    """The pair count and the closed FLOP conventions agree (exactly for full and
    causal-without-window up to the diagonal's half, within 0.03% on the workloads)."""
    import workloads
    for n in (3, 4, 5):
        w = workloads.BY_NUMBER[n]
        exact = oracle.flops(w.B, w.Hq, w.N, w.d, w.causal, w.window)
        closed = oracle.flops(w.B, w.Hq, w.N, w.d, w.causal, w.window, convention="closed")
        assert abs(exact / closed - 1.0) < 3e-4
    for N, causal, window in [(1, True, 0), (7, True, 0), (9, True, 3), (9, False, 0), (5, True, 9)]:
        assert oracle.valid_pairs(N, causal, window) == oracle.valid_pairs_closed(N, causal, window)

"""Pins for the fp64 softmax / top-K oracle (oracle/softmax.py).

Each pin takes a module-like object with ``softmax(x)`` and ``softmax_topk(x, k)`` and
raises AssertionError when it disagrees with
  * a library softmax and log-sum-exp (torch, float64, CPU),
  * closed forms (equal inputs give 1/V; one input far above the rest takes almost all
    the mass; the log-sum-exp of equal inputs is x + ln V),
  * invariants (rows sum to one, adding a constant changes nothing but the LSE),
  * the online normalizer recurrence of "Online normalizer calculation for softmax",
    restated here from its description (one pass keeping a running maximum and a
    normalizer rescaled whenever the maximum grows), element by element and by blocks,
  * top-K by brute force (every element outside the list is below or tied with the
    last one kept, ties resolved to the lower index, probabilities = softmax entries).
tests/test_oracle_softmax_pins.py plants mistakes in copies of the oracle and checks that
each fails a pin.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _x(rows, V, seed, scale=3.0):
    return np.random.default_rng(seed).standard_normal((rows, V)) * scale


def online_normalizer(row, block=1):
    """Running maximum m and normalizer d over a row, one block at a time: the block's
    maximum raises m, the old d is scaled by exp(m_old - m_new), and the block's
    exp(x - m_new) are added."""
    m, d = -math.inf, 0.0
    for s in range(0, len(row), block):
        blk = row[s:s + block]
        mn = max(m, float(np.max(blk)))
        d = (d * math.exp(m - mn) if m != -math.inf else 0.0) + float(np.sum(np.exp(blk - mn)))
        m = mn
    return m, d


def pin_library(mod):
    for n, (rows, V) in enumerate([(3, 1), (4, 7), (5, 1000), (2, 4099)]):
        x = _x(rows, V, 10 + n)
        y, lse = mod.softmax(x)
        ty = torch.softmax(torch.from_numpy(x), dim=1).numpy()
        tl = torch.logsumexp(torch.from_numpy(x), dim=1).numpy()
        assert np.max(np.abs(y - ty)) < 1e-15 and np.max(np.abs(lse - tl)) < 1e-12


def pin_closed_forms(mod):
    V = 37
    x = np.full((2, V), 2.5)
    y, lse = mod.softmax(x)
    assert np.max(np.abs(y - 1.0 / V)) < 1e-15 and np.max(np.abs(lse - (2.5 + math.log(V)))) < 1e-12
    x = np.zeros((1, V))
    x[0, 11] = 60.0
    y, _ = mod.softmax(x)
    assert abs(y[0, 11] - 1.0 / (1.0 + (V - 1) * math.exp(-60.0))) < 1e-15
    assert np.argmax(y[0]) == 11
    # a range wider than exp's: only the maximum as reference keeps every term finite
    y, lse = mod.softmax(np.array([[-500.0, 0.0, 500.0]]))
    assert np.all(np.isfinite(y)) and abs(y[0, 2] - 1.0) < 1e-15 and abs(y[0, 1] - math.exp(-500.0)) < 1e-230
    assert abs(lse[0] - 500.0) < 1e-12
    y, lse = mod.softmax(np.array([[0.0, math.log(3.0)]]))  # weights 1 : 3
    assert abs(y[0, 0] - 0.25) < 1e-15 and abs(y[0, 1] - 0.75) < 1e-15 and abs(lse[0] - math.log(4.0)) < 1e-15


def pin_invariants(mod):
    x = _x(6, 513, 21, scale=8.0)
    y, lse = mod.softmax(x)
    assert np.all(y > 0) and np.max(np.abs(y.sum(axis=1) - 1.0)) < 1e-13
    y2, lse2 = mod.softmax(x + 700.0)  # would overflow exp without the maximum
    assert np.all(np.isfinite(y2)) and np.max(np.abs(y2 - y)) < 1e-13
    assert np.max(np.abs(lse2 - (lse + 700.0))) < 1e-10
    # order is kept: a larger input has a larger probability
    o = np.argsort(x[0])
    assert np.all(np.diff(y[0][o]) >= 0)


def pin_online_normalizer(mod):
    x = _x(3, 777, 31, scale=5.0)
    _, lse = mod.softmax(x)
    for r in range(3):
        for block in (1, 4, 64, 777):
            m, d = online_normalizer(x[r], block)
            assert abs(m + math.log(d) - lse[r]) < 1e-12, (r, block)


def pin_topk(mod):
    x = _x(5, 300, 41)
    x[1, 7] = x[1, 200] = x[1, 250] = 50.0  # a three-way tie at the top
    x[2, :] = 1.0                            # all equal: the first k indices
    y, lse_full = mod.softmax(x)
    for k in (1, 3, 8, 300):
        probs, idx, lse = mod.softmax_topk(x, k)
        assert idx.shape == (5, k) and probs.shape == (5, k)
        assert np.max(np.abs(lse - lse_full)) < 1e-15
        for r in range(5):
            assert len(set(idx[r].tolist())) == k
            vals = x[r, idx[r]]
            assert np.all(np.diff(vals) <= 0)                       # descending
            rest = np.setdiff1d(np.arange(300), idx[r])
            if rest.size:
                assert np.max(x[r, rest]) <= vals[-1]                # nothing left out is larger
            for a in range(k - 1):                                   # ties: lower index first
                if vals[a] == vals[a + 1]:
                    assert idx[r, a] < idx[r, a + 1]
            if rest.size:
                tied_out = rest[x[r, rest] == vals[-1]]
                assert np.all(tied_out > idx[r, -1]) if tied_out.size else True
            assert np.max(np.abs(probs[r] - y[r, idx[r]])) < 1e-15
    probs, idx, _ = mod.softmax_topk(x, 3)
    assert idx[1].tolist() == [7, 200, 250] and idx[2].tolist() == [0, 1, 2]


PINS = {name[4:]: fn for name, fn in sorted(globals().items()) if name.startswith("pin_") and callable(fn)}


def failures(mod):
    bad = []
    for name, fn in PINS.items():
        try:
            fn(mod)
        except Exception:  # noqa: BLE001
            bad.append(name)
    return bad

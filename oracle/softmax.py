"""fp64 oracle for the stand-alone softmax and the fused softmax + top-K.

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it, and it
shares no code with the CUDA library.

Source: "Online normalizer calculation for softmax" (Milakov and Gimelshein): the
classical softmax of a vector, computed with fewer memory accesses, and softmax fused
with top-K.  The method reaches the classical result up to rounding, so the oracle is
the classical definition written out in fp64, row by row:

  m = max_i x_i,   d = sum_i exp(x_i - m),   y_i = exp(x_i - m) / d,   lse = m + ln d

Top-K of a row: the K largest inputs in descending order, ties broken towards the lower
index (the reading this library takes; the page does not say), each returned with its
index and its softmax probability exp(x_k - m) / d.

Parity of every function here is pinned by tests/test_oracle_softmax_pins.py.
"""
from __future__ import annotations

import numpy as np


def _rows(x) -> np.ndarray:
    a = np.asarray(x.float().numpy() if hasattr(x, "numpy") and hasattr(x, "float") else x, dtype=np.float64)
    if a.ndim != 2:
        raise ValueError("softmax oracle: expected a 2-D [rows, V] array")
    return a


def softmax(x):
    """Classical softmax of every row of ``x`` [rows, V] in fp64.  Returns (y, lse)."""
    a = _rows(x)
    if a.shape[1] == 0:
        return np.zeros_like(a), np.full(a.shape[0], -np.inf)
    m = a.max(axis=1, keepdims=True)
    e = np.exp(a - m)
    d = e.sum(axis=1, keepdims=True)
    return e / d, (m + np.log(d))[:, 0]


def softmax_topk(x, k: int):
    """Top-``k`` of every row with their softmax probabilities.

    Returns (probs [rows, k] fp64, idx [rows, k] int64, lse [rows] fp64); entries are in
    descending order of x, ties towards the lower index."""
    a = _rows(x)
    rows, V = a.shape
    if not 1 <= k <= V:
        raise ValueError("softmax oracle: need 1 <= k <= V")
    y, lse = softmax(a)
    idx = np.empty((rows, k), dtype=np.int64)
    cols = np.arange(V)
    for r in range(rows):
        order = np.lexsort((cols, -a[r]))  # primary: value descending; then index ascending
        idx[r] = order[:k]
    probs = np.take_along_axis(y, idx, axis=1)
    return probs, idx, lse


__all__ = ["softmax", "softmax_topk"]

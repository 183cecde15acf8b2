"""Test-side restatements of the streaming (online-softmax) recurrences on the pages.

These exist only to pin the dense fp64 oracle: the pages state that the streaming
recurrence reaches exactly the dense result, so running both on the same score row in
fp64 must agree to rounding.  They are written from the pages' descriptions, not from
their listings, and are never used by the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np


def score_rows(q, k, scale, causal=False, window=0, softcap=0.0):
    """Masked, soft-capped scores of one head in fp64: q [N, d], k [N, d] -> [N, N]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = scale * (q @ k.T)
    if softcap > 0:
        s = softcap * np.tanh(s / softcap)
    n = s.shape[0]
    i = np.arange(n)[:, None]
    j = np.arange(s.shape[1])[None, :]
    if causal:
        s = np.where(j > i, -np.inf, s)
    if window > 0:
        s = np.where(i - j >= window, -np.inf, s)
    return s


def stream_row(s, v, tile):
    """Tiled online softmax over one score row (numerator form).

    Per tile: new maximum = max(running maximum, tile maximum); the running sum and the
    running weighted sum of values are multiplied by exp(old - new) and the tile's
    exp(score - new) terms are added ("Online Softmax Without the Attention Matrix",
    the streaming function).  A running maximum still at -inf contributes a factor 0
    instead of exp(-inf - -inf) (the guard in oxios FlashAttention::attention).
    Returns (output, log-sum-exp)."""
    s = np.asarray(s, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    m = -math.inf
    den = 0.0
    num = np.zeros(v.shape[1])
    for start in range(0, s.shape[0], tile):
        ts = s[start:start + tile]
        tv = v[start:start + tile]
        new_m = max(m, float(ts.max()))
        if new_m == -math.inf:
            continue  # every score so far is masked
        corr = 0.0 if m == -math.inf else math.exp(m - new_m)
        w = np.exp(ts - new_m)
        den = den * corr + w.sum()
        num = num * corr + w @ tv
        m = new_m
    if den == 0.0:
        return np.zeros(v.shape[1]), -math.inf
    return num / den, m + math.log(den)


def stream_row_seeded(s, v):
    """Per-key streaming with the state seeded from key 0 (nx_flashattn_scale.nx, the
    FLASHATTENTION streaming loop): m = s0, l = 1, acc = v0, then for each later key
    the running state is rescaled by exp(m - m_new) and the key's exp(s - m_new) added.
    Requires s[0] finite."""
    s = np.asarray(s, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    m = float(s[0])
    l = 1.0
    acc = v[0].copy()
    for j in range(1, s.shape[0]):
        mnew = max(m, float(s[j]))
        corr = math.exp(m - mnew)
        p = math.exp(float(s[j]) - mnew)
        l = l * corr + p
        acc = acc * corr + p * v[j]
        m = mnew
    return acc / l, m + math.log(l)


def unstabilised_row(s, v, tile):
    """The same running ratio with no maximum subtracted (Module 16, section 16.2,
    second 'Measured' note): exact for small scores, overflows for large ones."""
    s = np.asarray(s, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    den = 0.0
    num = np.zeros(v.shape[1])
    with np.errstate(over="ignore", invalid="ignore"):
        for start in range(0, s.shape[0], tile):
            w = np.exp(s[start:start + tile])
            den = den + w.sum()
            num = num + w @ v[start:start + tile]
        return num / den

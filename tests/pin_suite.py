"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each pin takes an ``attn`` callable with the signature of ``oracle.attention`` and
raises ``AssertionError`` when the callable disagrees with

  * values the pages print for a worked example (tests/golden/worked_examples.json),
  * closed forms and special cases,
  * invariants (rows sum to one, causal row = prefix attention, block merge),
  * a library softmax (torch, float64, CPU) on tiny inputs,
  * brute-force streaming restatements of the pages' recurrences.

They are chosen so that a plausible mistake anywhere in the oracle (a dropped term, a
wrong sign or index, an off-by-one mask, a transposed operand, a wrong head mapping)
fails at least one of them; tests/test_oracle_mutants.py plants such mistakes in copies
of the oracle and checks that.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
from tests import streaming_ref as sr

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(shape, seed, mult=1.0):
    return _rng(seed).standard_normal(shape) * mult


def _torch_ref(q, k, v, scale, causal=False, window=0, softcap=0.0):
    """Library reduction: torch.softmax / torch.logsumexp in float64 on the CPU, with
    K and V repeated per query-head group."""
    q = torch.as_tensor(np.asarray(q, dtype=np.float64))
    k = torch.as_tensor(np.asarray(k, dtype=np.float64))
    v = torch.as_tensor(np.asarray(v, dtype=np.float64))
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    s = torch.matmul(q, k.transpose(-1, -2)) * scale
    if softcap > 0:
        s = softcap * torch.tanh(s / softcap)
    nq, nk = s.shape[-2], s.shape[-1]
    pos = torch.arange(nq)[:, None] + (nk - nq)
    j = torch.arange(nk)[None, :]
    mask = torch.zeros(nq, nk, dtype=torch.bool)
    if causal:
        mask |= j > pos
    if window > 0:
        mask |= (pos - j) >= window
    s = s.masked_fill(mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    o = torch.matmul(torch.softmax(s, dim=-1), v)
    return o.numpy(), lse.numpy()


# --------------------------------------------------------------------------- pins

def pin_worked_example(attn):
    """Notebook worked example: scores 1000 + ln i (i = 1..4), values 10, 20, 30, 40.
    Dense and streaming (tiles 1, 2, 4) both give 30 within 1e-10; the log-sum-exp has
    the closed form 1000 + ln(1 + 2 + 3 + 4)."""
    ex = GOLD["notebook_worked_example"]
    scores = np.array([1000.0 + math.log(i) for i in range(1, 5)])
    values = np.array(ex["values"])
    q = np.ones((1, 1, 4, 1))
    k = scores.reshape(1, 1, 4, 1)
    v = values.reshape(1, 1, 4, 1)
    o, lse = attn(q, k, v, scale=1.0)
    assert np.all(np.abs(o - ex["expected_output"]) < ex["tolerance"]), o.ravel()
    assert np.all(np.abs(lse - (1000.0 + math.log(10.0))) < 1e-9), lse.ravel()
    for t in ex["tile_sizes"]:
        out, _ = sr.stream_row(scores, values[:, None], t)
        assert abs(out[0] - ex["expected_output"]) < ex["tolerance"]
    # the same example with the one-query row causal over all four keys (query is last)
    o1, lse1 = attn(q[:, :, :1], k, v, scale=1.0, causal=True)
    assert abs(o1.ravel()[0] - 30.0) < 1e-10 and abs(lse1.ravel()[0] - (1000 + math.log(10))) < 1e-9


def pin_merge_identities(attn):
    """Module 16, 16.2: l = e^(m1-m) l1 + e^(m2-m) l2 and the share-weighted output
    merge; the exercise value l = 1.6494; and oracle(first keys) merged with
    oracle(last keys) equals oracle(all keys)."""
    ex = GOLD["merge_exercise"]
    _, l, _ = oracle.merge(np.array(ex["m1"]), np.array(ex["l1"]), np.zeros((1,)),
                           np.array(ex["m2"]), np.array(ex["l2"]), np.zeros((1,)))
    assert abs(float(l) - ex["expected_l"]) < ex["tolerance"], l
    B, Hq, Hkv, N, d = 1, 4, 2, 23, 6
    q, k, v = _rand((B, Hq, N, d), 11), _rand((B, Hkv, N, d), 12), _rand((B, Hkv, N, d), 13)
    scale = 0.4
    o_full, lse_full = attn(q, k, v, scale=scale)
    for a in (1, 9, 22):
        o1, lse1 = attn(q, k[:, :, :a], v[:, :, :a], scale=scale)
        o2, lse2 = attn(q, k[:, :, a:], v[:, :, a:], scale=scale)
        g = Hq // Hkv
        kk = np.repeat(k, g, axis=1)
        s_all = np.einsum("bhid,bhjd->bhij", q, kk) * scale
        m1 = s_all[..., :a].max(-1)
        m2 = s_all[..., a:].max(-1)
        l1 = np.exp(lse1 - m1)
        l2 = np.exp(lse2 - m2)
        m, l, o = oracle.merge(m1, l1, o1, m2, l2, o2)
        assert np.max(np.abs(o - o_full)) < 1e-12
        assert np.max(np.abs(m + np.log(l) - lse_full)) < 1e-12


def pin_rows_sum_to_one(attn):
    """With V = I the output row is the softmax row itself: non-negative, zero on masked
    keys, summing to one (Module 16, 16.2: normalised attention weights)."""
    N = 17
    q, k = _rand((1, 1, N, 4), 21), _rand((1, 1, N, 4), 22)
    v = np.eye(N).reshape(1, 1, N, N)
    q_pad = np.concatenate([q, np.zeros((1, 1, N, N - 4))], axis=-1)
    k_pad = np.concatenate([k, np.zeros((1, 1, N, N - 4))], axis=-1)
    for causal, window, cap in [(False, 0, 0.0), (True, 0, 0.0), (True, 5, 0.0), (True, 3, 2.0)]:
        p, lse = attn(q_pad, k_pad, v, scale=0.7, causal=causal, window=window, softcap=cap)
        p = p[0, 0]
        assert np.all(p >= 0)
        assert np.max(np.abs(p.sum(-1) - 1.0)) < 1e-12
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        masked = np.zeros((N, N), bool)
        if causal:
            masked |= j > i
        if window:
            masked |= i - j >= window
        assert np.all(p[masked] == 0.0)
        assert np.all(p[~masked] > 0.0)


def pin_streaming_brute_force(attn):
    """Brute force on tiny inputs: for every tile size 1..N the tiled online-softmax
    recurrence (notebook streaming function, with the oxios -inf guard) equals the
    oracle to 1e-12, with every mask / soft-cap combination (Module 16, 16.2
    'Measured': exact for every block size; the causal mask uses global positions)."""
    for N, d in [(1, 1), (2, 3), (7, 2), (16, 5), (33, 8)]:
        q, k, v = _rand((1, 1, N, d), 31 + N), _rand((1, 1, N, d), 32 + N), _rand((1, 1, N, d), 33 + N)
        for causal, window, cap in [(False, 0, 0.0), (True, 0, 0.0), (True, 4, 0.0), (False, 0, 1.5), (True, 2, 3.0)]:
            o, lse = attn(q, k, v, scale=0.9, causal=causal, window=window, softcap=cap)
            s = sr.score_rows(q[0, 0], k[0, 0], 0.9, causal, window, cap)
            for i in range(N):
                for t in range(1, N + 1):
                    so, slse = sr.stream_row(s[i], v[0, 0], t)
                    assert np.max(np.abs(so - o[0, 0, i])) < 1e-12, (N, d, causal, window, cap, i, t)
                    assert abs(slse - lse[0, 0, i]) < 1e-12


def pin_library_softmax(attn):
    """Tiny shapes against torch.softmax / torch.logsumexp in float64 (the textbook
    definition through a library routine), MHA and GQA, every mask, soft-cap on/off,
    and cross-attention shapes (fewer queries than keys)."""
    cases = [
        (2, 4, 4, 9, 9, 5, False, 0, 0.0),
        (1, 6, 2, 13, 13, 8, True, 0, 0.0),
        (2, 4, 1, 10, 10, 3, True, 3, 0.0),
        (1, 2, 2, 12, 12, 4, True, 5, 2.5),
        (1, 3, 3, 11, 11, 7, False, 0, 4.0),
        (1, 4, 2, 3, 8, 5, True, 0, 0.0),
        (1, 2, 1, 1, 6, 4, True, 2, 0.0),
    ]
    for n, (B, Hq, Hkv, Nq, Nk, d, causal, window, cap) in enumerate(cases):
        q = _rand((B, Hq, Nq, d), 40 + n)
        k = _rand((B, Hkv, Nk, d), 50 + n)
        v = _rand((B, Hkv, Nk, d), 60 + n)
        scale = 1.0 / math.sqrt(d) * (1.0 + 0.1 * n)
        o, lse = attn(q, k, v, scale=scale, causal=causal, window=window, softcap=cap)
        ro, rlse = _torch_ref(q, k, v, scale, causal, window, cap)
        assert np.max(np.abs(o - ro)) < 1e-12, (n, np.max(np.abs(o - ro)))
        assert np.max(np.abs(lse - rlse)) < 1e-12, (n, np.max(np.abs(lse - rlse)))


def pin_row_subset(attn):
    """Asking for a subset of rows returns exactly those rows of the full result."""
    B, Hq, Hkv, N, d = 2, 4, 2, 19, 6
    q, k, v = _rand((B, Hq, N, d), 71), _rand((B, Hkv, N, d), 72), _rand((B, Hkv, N, d), 73)
    o, lse = attn(q, k, v, scale=0.5, causal=True, window=7)
    rows = np.array([0, 5, 18, 19 + 3, 3 * 19 + 17, B * Hq * N - 1])
    so, slse = attn(q, k, v, scale=0.5, causal=True, window=7, rows=rows)
    assert np.array_equal(so, o.reshape(-1, d)[rows])
    assert np.array_equal(slse, lse.reshape(-1)[rows])


def pin_closed_forms(attn):
    """Special cases with closed forms."""
    N, d = 12, 5
    q, k, v = _rand((1, 2, N, d), 81), _rand((1, 2, N, d), 82), _rand((1, 2, N, d), 83)
    # constant values -> output is that constant
    vc = np.full((1, 2, N, d), 3.25)
    o, _ = attn(q, k, vc, scale=0.8, causal=True, window=4, softcap=2.0)
    assert np.max(np.abs(o - 3.25)) < 1e-12
    # zero queries -> uniform weights: O = mean of V over the valid keys, LSE = ln(#valid)
    qz = np.zeros_like(q)
    for causal, window in [(False, 0), (True, 0), (True, 4)]:
        o, lse = attn(qz, k, v, scale=0.8, causal=causal, window=window, softcap=1.5)
        for i in range(N):
            lo = max(0, i - window + 1) if window else 0
            hi = i if causal else N - 1
            cnt = hi - lo + 1
            assert np.max(np.abs(o[0, :, i] - v[0, :, lo:hi + 1].mean(axis=1))) < 1e-12
            assert np.max(np.abs(lse[0, :, i] - math.log(cnt))) < 1e-12
    # one key -> O = v0, LSE = s00
    o, lse = attn(q[:, :, :1], k[:, :, :1], v[:, :, :1], scale=0.8)
    s00 = 0.8 * np.sum(q[0, :, 0] * k[0, :, 0], axis=-1)
    assert np.max(np.abs(o[0, :, 0] - v[0, :, 0])) < 1e-12
    assert np.max(np.abs(lse[0, :, 0] - s00)) < 1e-12
    # causal row 0 sees only key 0; a window of 1 sees only the diagonal
    o, lse = attn(q, k, v, scale=0.8, causal=True)
    assert np.max(np.abs(o[0, :, 0] - v[0, :, 0])) < 1e-12
    o, lse = attn(q, k, v, scale=0.8, causal=True, window=1)
    sii = 0.8 * np.sum(q[0] * k[0], axis=-1)
    assert np.max(np.abs(o[0] - v[0])) < 1e-12
    assert np.max(np.abs(lse[0] - sii)) < 1e-12
    # a window of at least N keys is plain causal attention
    oa, la = attn(q, k, v, scale=0.8, causal=True, window=N)
    ob, lb = attn(q, k, v, scale=0.8, causal=True)
    assert np.max(np.abs(oa - ob)) == 0.0 and np.max(np.abs(la - lb)) == 0.0
    # a huge cap is no cap
    oa, la = attn(q, k, v, scale=0.8, softcap=1e30)
    ob, lb = attn(q, k, v, scale=0.8)
    assert np.max(np.abs(oa - ob)) < 1e-12 and np.max(np.abs(la - lb)) < 1e-12
    # the scale multiplies the scores: scale s on q equals scale 1 on s*q
    oa, la = attn(q, k, v, scale=0.37)
    ob, lb = attn(q * 0.37, k, v, scale=1.0)
    assert np.max(np.abs(oa - ob)) < 1e-12 and np.max(np.abs(la - lb)) < 1e-12


def pin_softcap_values(attn):
    """Section 16.5 printed values with kappa = 30: with one key the log-sum-exp is the
    capped score itself (30 -> 22.85, 5 -> 4.95, 100 -> 29.9, 300 -> ~30)."""
    ex = GOLD["softcap_values"]
    for c in ex["cases"]:
        q = np.ones((1, 1, 1, 1))
        k = np.full((1, 1, 1, 1), c["z"])
        v = np.ones((1, 1, 1, 1))
        _, lse = attn(q, k, v, scale=1.0, softcap=ex["kappa"])
        assert abs(lse.ravel()[0] - c["expected"]) < c["tolerance"], (c, lse)
        assert abs(lse.ravel()[0] - float(oracle.softcap(c["z"], ex["kappa"]))) < 1e-12
    # the cap keeps the order of scores, and maps 0 to 0
    zs = np.linspace(-200, 200, 41)
    caps = oracle.softcap(zs, 50.0)
    assert np.all(np.diff(caps) > 0) and abs(float(oracle.softcap(0.0, 50.0))) == 0.0
    assert np.all(np.abs(caps) < 50.0)


def pin_stability(attn):
    """Scores x40 (Module 16, 16.2 second 'Measured' note): the max-subtracted oracle
    stays finite and equals the library softmax; the same ratio without the maximum
    overflows.  Also Q x 8 as in the grouped-query workload."""
    N, d = 16, 8
    q, k, v = _rand((1, 1, N, d), 91), _rand((1, 1, N, d), 92), _rand((1, 1, N, d), 93)
    for mult in (40.0, 8.0 * math.sqrt(d)):
        o, lse = attn(q * mult, k, v, scale=1.0)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
        ro, rlse = _torch_ref(q * mult, k, v, 1.0)
        assert np.max(np.abs(o - ro)) < 1e-12
        assert np.max(np.abs(lse - rlse)) < 1e-10 * max(1.0, float(np.max(np.abs(rlse))))
    s = sr.score_rows(q[0, 0] * 40.0 * 40.0, k[0, 0], 1.0)
    bad = sr.unstabilised_row(s[0], v[0, 0], 4)
    assert not np.all(np.isfinite(bad))
    small = sr.score_rows(q[0, 0] * 0.1, k[0, 0], 1.0)
    o_small, _ = attn(q * 0.1, k, v, scale=1.0)
    assert np.max(np.abs(sr.unstabilised_row(small[3], v[0, 0], 4) - o_small[0, 0, 3])) < 1e-12


def pin_causal_prefix(attn):
    """The causal row i is non-causal attention of query i over keys 0..i (positions in
    the full sequence, Module 16, 16.2 'Measured')."""
    N, d = 14, 6
    q, k, v = _rand((1, 2, N, d), 101), _rand((1, 2, N, d), 102), _rand((1, 2, N, d), 103)
    o, lse = attn(q, k, v, scale=0.6, causal=True)
    for i in range(N):
        oi, li = attn(q[:, :, i:i + 1], k[:, :, :i + 1], v[:, :, :i + 1], scale=0.6)
        assert np.max(np.abs(oi[0, :, 0] - o[0, :, i])) < 1e-12
        assert np.max(np.abs(li[0, :, 0] - lse[0, :, i])) < 1e-12


def pin_gqa_grouping(attn):
    """Query head hq reads key/value head hq // (Hq / Hkv): GQA equals MHA with K and V
    repeated per group, and query heads in one group share keys."""
    B, Hq, Hkv, N, d = 1, 6, 2, 9, 4
    q, k, v = _rand((B, Hq, N, d), 111), _rand((B, Hkv, N, d), 112), _rand((B, Hkv, N, d), 113)
    o, lse = attn(q, k, v, scale=0.5, causal=True)
    o2, lse2 = attn(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), scale=0.5, causal=True)
    assert np.max(np.abs(o - o2)) < 1e-15 and np.max(np.abs(lse - lse2)) < 1e-15
    for hq in range(Hq):
        oh, lh = attn(q[:, hq:hq + 1], k[:, hq // 3:hq // 3 + 1], v[:, hq // 3:hq // 3 + 1], scale=0.5, causal=True)
        assert np.max(np.abs(oh[0, 0] - o[0, hq])) < 1e-15


def pin_nx_modular(attn):
    """nx_flashattn_scale.nx workload (n=64, d=32, modular inputs, scale 1/sqrt(32)):
    the direct result equals the key-0-seeded per-key streaming recurrence, with zero
    elements off by 1e-3 or more (the program's own check) and agreement to 1e-12 in
    fp64."""
    import workloads
    w = workloads.WORKLOADS["modular_n64_d32"]
    q, k, v = workloads.make_inputs(w)
    o, lse = attn(q, k, v, scale=w.scale)
    s = sr.score_rows(q[0, 0].double().numpy(), k[0, 0].double().numpy(), w.scale)
    vv = v[0, 0].double().numpy()
    worst = 0.0
    fails = 0
    for i in range(w.N):
        so, sl = sr.stream_row_seeded(s[i], vv)
        fails += int(np.sum(np.abs(so - o[0, 0, i]) >= GOLD["nx_direct_vs_streaming"]["tolerance"]))
        worst = max(worst, float(np.max(np.abs(so - o[0, 0, i]))), abs(sl - lse[0, 0, i]))
    assert fails == GOLD["nx_direct_vs_streaming"]["expected_fails"]
    assert worst < 1e-12, worst
    ro, rlse = _torch_ref(q.double().numpy(), k.double().numpy(), v.double().numpy(), w.scale)
    assert np.max(np.abs(o - ro)) < 1e-12 and np.max(np.abs(lse - rlse)) < 1e-12


def _kept_keys(pos, nk, causal, window, n_sink):
    """The keys a query at position ``pos`` sees, built as sets from the section's words:
    with a window, the ``window`` most recent tokens up to the query itself, together with
    the first ``n_sink`` tokens (Module 16, 16.6), never a token after the query when
    causal (16.2)."""
    visible = set(range(nk)) if not causal else set(range(max(0, min(pos + 1, nk))))
    if window <= 0:
        return sorted(visible)
    recent = set(range(max(0, pos - window + 1), pos + 1))
    sinks = set(range(n_sink))
    return sorted(visible & (recent | sinks))


def pin_attention_sinks(attn):
    """Attention sinks (Module 16, 16.6: the first tokens kept alongside the sliding
    window).  (a) Against a library softmax over the key set built explicitly per row,
    self- and cross-attention shapes, sinks fewer and more than the window, rows before
    the sinks end; (b) no sinks is the plain window and sinks covering every key are
    plain causal attention, bit for bit; (c) zero queries give LSE = ln(#kept keys) in
    closed form; (d) a row whose sinks and window are disjoint is the block merge
    (16.2) of attention over the sinks alone and over the window alone."""
    cases = [  # Nq, Nk, d, window, n_sink, cap
        (21, 21, 5, 4, 3, 0.0),
        (21, 21, 4, 1, 4, 0.0),
        (16, 16, 3, 6, 9, 2.0),
        (7, 19, 6, 5, 2, 0.0),
        (19, 19, 4, 3, 1, 0.0),
    ]
    for n, (nq, nk, d, window, n_sink, cap) in enumerate(cases):
        q, k, v = _rand((1, 2, nq, d), 401 + n), _rand((1, 1, nk, d), 411 + n), _rand((1, 1, nk, d), 421 + n)
        scale = 0.7
        o, lse = attn(q, k, v, scale=scale, causal=True, window=window, n_sink=n_sink, softcap=cap)
        for h in range(2):
            for i in range(nq):
                keep = _kept_keys(i + nk - nq, nk, True, window, n_sink)
                s = torch.as_tensor(scale * (q[0, h, i] @ k[0, 0, keep].T))
                if cap > 0:
                    s = cap * torch.tanh(s / cap)
                w = torch.softmax(s, dim=-1).numpy()
                assert np.max(np.abs(o[0, h, i] - w @ v[0, 0, keep])) < 1e-12, (n, h, i)
                assert abs(lse[0, h, i] - float(torch.logsumexp(s, dim=-1))) < 1e-12, (n, h, i)
    # (b) limits
    N, d = 18, 4
    q, k, v = _rand((1, 2, N, d), 431), _rand((1, 2, N, d), 432), _rand((1, 2, N, d), 433)
    oa, la = attn(q, k, v, scale=0.6, causal=True, window=5, n_sink=0)
    ob, lb = attn(q, k, v, scale=0.6, causal=True, window=5)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)
    oa, la = attn(q, k, v, scale=0.6, causal=True, window=5, n_sink=N)
    ob, lb = attn(q, k, v, scale=0.6, causal=True)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)
    # (c) uniform weights
    for window, n_sink in [(4, 4), (1, 2), (6, 1)]:
        o, lse = attn(np.zeros_like(q), k, v, scale=0.6, causal=True, window=window, n_sink=n_sink)
        for i in range(N):
            cnt = min(i + 1, window) + min(n_sink, max(0, i - window + 1))
            assert abs(lse[0, 0, i] - math.log(cnt)) < 1e-12, (window, n_sink, i)
    # (d) block merge of the sinks and the window
    W, S = 4, 3
    o, lse = attn(q, k, v, scale=0.6, causal=True, window=W, n_sink=S)
    for i in range(S + W, N):
        o1, l1 = attn(q[:, :, i:i + 1], k[:, :, :S], v[:, :, :S], scale=0.6)
        o2, l2 = attn(q[:, :, i:i + 1], k[:, :, i - W + 1:i + 1], v[:, :, i - W + 1:i + 1], scale=0.6)
        s = 0.6 * np.einsum("hd,hjd->hj", q[0, :, i], k[0])
        m1, m2 = s[:, :S].max(-1), s[:, i - W + 1:i + 1].max(-1)
        m, l, om = oracle.merge(m1, np.exp(l1[0, :, 0] - m1), o1[0, :, 0], m2, np.exp(l2[0, :, 0] - m2), o2[0, :, 0])
        assert np.max(np.abs(om - o[0, :, i])) < 1e-12
        assert np.max(np.abs(m + np.log(l) - lse[0, :, i])) < 1e-12


def pin_cross_attention(attn):
    """Fewer (or more) queries than keys: the queries are the last Nq positions of the
    key sequence.  Non-causal cross-attention of one query row equals self-attention's
    row over the same keys; causal rows equal the prefix attention at their global
    position; with more queries than keys the rows before the first key see nothing
    (O = 0, LSE = -inf, as the oxios routine leaves a row whose sum stays zero)."""
    nk, d = 13, 4
    k, v = _rand((1, 1, nk, d), 441), _rand((1, 1, nk, d), 442)
    qs = _rand((1, 1, nk, d), 443)
    o_self, l_self = attn(qs, k, v, scale=0.5, causal=True)
    for nq in (1, 4, nk):
        o, lse = attn(qs[:, :, nk - nq:], k, v, scale=0.5, causal=True)
        assert np.array_equal(o[0, 0], o_self[0, 0, nk - nq:]) and np.array_equal(lse[0, 0], l_self[0, 0, nk - nq:])
    o_full, l_full = attn(qs, k, v, scale=0.5)
    o, lse = attn(qs[:, :, 5:6], k, v, scale=0.5)
    assert np.array_equal(o[0, 0, 0], o_full[0, 0, 5]) and lse[0, 0, 0] == l_full[0, 0, 5]
    qm = _rand((1, 1, nk + 3, d), 444)
    o, lse = attn(qm, k, v, scale=0.5, causal=True)
    assert np.all(o[0, 0, :3] == 0.0) and np.all(lse[0, 0, :3] == -np.inf)
    ref, rl = attn(qm[:, :, 3:], k, v, scale=0.5, causal=True)
    assert np.array_equal(o[0, 0, 3:], ref[0, 0]) and np.array_equal(lse[0, 0, 3:], rl[0, 0])


def _bf16_from_bits(bits):
    """bf16 torch tensor whose elements have exactly the given 16-bit patterns."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16)


def pin_bf16_inputs(attn):
    """bf16 inputs are read as the exact values they store: the oracle on bf16 tensors
    equals, bit for bit, the oracle on the same tensors widened to float64 by torch
    (an independent library conversion).  The values cover both signs, bf16
    subnormals (a query row of subnormals against keys of 2^120 makes them decide the
    scores) and magnitudes up to 2^120 (a one-hot softmax copies such a V row into O),
    so a wrong shift, a byte swap or a lost sign changes the output.  MHA, GQA and
    cross shapes, with the masks and the soft-cap."""
    rng = _rng(97)

    def rand_bits(shape):
        x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
        return x.view(torch.int16).numpy().view(np.uint16).copy()

    cases = [  # B, Hq, Hkv, Nq, Nk, d, causal, window, cap
        (1, 2, 2, 7, 7, 5, False, 0, 0.0),
        (2, 4, 2, 9, 9, 6, True, 0, 0.0),
        (1, 2, 1, 3, 8, 4, True, 3, 0.0),
        (1, 2, 2, 6, 6, 4, True, 0, 2.5),
    ]
    for B, Hq, Hkv, Nq, Nk, d, causal, window, cap in cases:
        qb, kb, vb = rand_bits((B, Hq, Nq, d)), rand_bits((B, Hkv, Nk, d)), rand_bits((B, Hkv, Nk, d))
        # query row 0 of head 0: bf16 subnormals (exponent field 0) of both signs;
        # key row 0: +-2^120 (0x7b80 / 0xfb80), so q.k of that pair is of order 2^-10
        qb[0, 0, 0, :] = np.array([0x0001, 0x8003, 0x007F, 0x0040, 0x8011, 0x0002][:d], dtype=np.uint16)
        kb[0, 0, 0, :] = np.array([0x7B80, 0xFB80, 0x7B80, 0x7B80, 0xFB80, 0x7B80][:d], dtype=np.uint16)
        # value rows with 2^100 (0x7180), -1.25 * 2^110 (0xf6a0), subnormals, small
        # negatives and the largest finite bf16 of both signs (0x7f7f / 0xff7f)
        vb[0, 0, 1, :] = np.array([0x7180, 0xF6A0, 0x0005, 0x8005, 0xBF40, 0x3F81][:d], dtype=np.uint16)
        vb[0, -1, -1, :] = np.array([0x8001, 0x0080, 0xC2F7, 0x42F7, 0x7F7F, 0xFF7F][:d], dtype=np.uint16)
        q, k, v = _bf16_from_bits(qb), _bf16_from_bits(kb), _bf16_from_bits(vb)
        o_b, l_b = attn(q, k, v, scale=0.37, causal=causal, window=window, softcap=cap)
        o_d, l_d = attn(q.to(torch.float64), k.to(torch.float64), v.to(torch.float64), scale=0.37, causal=causal,
                        window=window, softcap=cap)
        assert np.array_equal(o_b, o_d, equal_nan=True) and np.array_equal(l_b, l_d, equal_nan=True)
        assert np.all(np.isfinite(l_b)) or causal


def pin_empty(attn):
    """No queries (or a zero batch) gives empty outputs and no error (oxios returns an
    empty result for empty input)."""
    o, lse = attn(np.zeros((0, 2, 5, 3)), np.zeros((0, 2, 5, 3)), np.zeros((0, 2, 5, 3)), scale=1.0)
    assert o.shape == (0, 2, 5, 3) and lse.shape == (0, 2, 5)
    o, lse = attn(np.zeros((1, 2, 0, 3)), np.zeros((1, 2, 0, 3)), np.zeros((1, 2, 0, 3)), scale=1.0)
    assert o.size == 0 and lse.size == 0


PINS = {name[4:]: fn for name, fn in sorted(globals().items()) if name.startswith("pin_") and callable(fn)}


def failures(attn):
    """Names of the pins that ``attn`` fails (an exception counts as a failure)."""
    bad = []
    for name, fn in PINS.items():
        try:
            fn(attn)
        except Exception:  # noqa: BLE001 - any error is a failed pin
            bad.append(name)
    return bad

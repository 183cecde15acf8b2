"""GPU parity of fa_fwd_ext: cross-attention (Nq != Nk), attention sinks, and both with
split-KV, against the fp64 oracle element by element (bf16 tolerances O 2e-2,
LSE 1e-3).

Readings under test: query row i sits at key position i + (Nk - Nq) (the queries are
the last Nq positions, as when decoding against a key/value cache); the first n_sink
keys are exempt from the window ("Module 16: Efficient and Long Attention", section
16.6) but not from the causal mask; a row with no valid key gives O = 0, LSE = -inf.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.test_parity_gpu import TOL, guarded, guards_intact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import online_softmax_11_b200 as fa_mod
    from online_softmax_11_b200 import build
    build.build()
    fa_mod.load()
    return fa_mod


def compare_rows(o, lse, ro, rlse):
    """Max-abs comparison; rows the oracle leaves empty (LSE = -inf) must be exactly
    O = 0 and LSE = -inf on the GPU too."""
    tol_o, tol_l = TOL["bfloat16"]
    empty = np.isneginf(rlse)
    assert np.array_equal(np.isneginf(lse), empty), "rows without keys differ"
    assert np.all(o[empty] == 0.0)
    full = ~empty
    assert np.all(np.isfinite(o[full])) and np.all(np.isfinite(lse[full]))
    eo = float(np.max(np.abs(o[full] - ro[full]))) if full.any() else 0.0
    el = float(np.max(np.abs(lse[full] - rlse[full]))) if full.any() else 0.0
    assert eo <= tol_o, f"O max-abs error {eo:.3e} > {tol_o}"
    assert el <= tol_l, f"LSE max-abs error {el:.3e} > {tol_l}"


def run_ext(fa, q, k, v, *, causal, window, n_sink, softcap, num_splits, scale):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, Hq, Nq, d = q.shape
    obuf, o = guarded((B, Hq, Nq, d), q.dtype, dev)
    lbuf, lse = guarded((B, Hq, Nq), torch.float32, dev)
    fa.forward_ext(qd, kd, vd, scale=scale, causal=causal, window=window, n_sink=n_sink, softcap=softcap,
                   num_splits=num_splits, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert guards_intact(obuf) and guards_intact(lbuf), "kernel wrote outside its outputs"
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, n_sink, softcap, num_splits
    (1, 2, 2, 1, 700, 128, True, 0, 0, 0.0, 0),        # one decode step
    (2, 4, 2, 1, 1500, 64, True, 0, 0, 0.0, 4),        # decode, split-KV
    (1, 2, 1, 300, 1000, 128, True, 0, 0, 0.0, 0),     # chunk of new queries over a cache
    (1, 2, 2, 77, 513, 128, False, 0, 0, 0.0, 0),      # plain cross-attention
    (1, 2, 2, 600, 257, 64, False, 0, 0, 0.0, 2),
    (1, 2, 2, 1000, 300, 128, True, 0, 0, 0.0, 0),     # more queries than keys: empty rows
    (1, 2, 2, 700, 130, 64, True, 0, 0, 0.0, 3),
    (1, 2, 2, 200, 2000, 128, True, 256, 0, 0.0, 0),   # window over a cache
    (1, 2, 2, 1000, 1000, 128, True, 128, 4, 0.0, 0),  # sinks beside a window
    (2, 4, 2, 900, 900, 64, True, 200, 4, 0.0, 0),
    (1, 2, 2, 1000, 1000, 128, True, 1, 4, 0.0, 0),    # window of one token + sinks
    (1, 2, 2, 800, 800, 128, True, 150, 130, 0.0, 0),  # sinks span two key tiles
    (1, 2, 2, 700, 700, 128, True, 100, 300, 0.0, 0),  # more sinks than the window
    (1, 2, 2, 1000, 1000, 128, True, 256, 4, 30.0, 0),  # sinks with the soft-cap
    (1, 2, 2, 1100, 1100, 128, True, 128, 4, 0.0, 3),  # sinks with split-KV
    (1, 2, 1, 600, 2500, 128, True, 300, 4, 0.0, 2),   # all of it at once
    (1, 2, 2, 300, 300, 128, False, 0, 4, 0.0, 0),     # sinks without a window: no effect
    # few query rows per key/value head (group x Nq <= 16): the decode kernel
    (2, 32, 8, 1, 4099, 128, True, 0, 0, 0.0, 0),     # one decoding step, GQA 4
    (2, 32, 8, 4, 1000, 128, True, 0, 0, 0.0, 0),     # 16 rows: 4 heads x 4 queries
    (1, 16, 2, 2, 777, 64, True, 0, 0, 0.0, 3),       # 16 rows, d = 64, split-KV
    (1, 8, 8, 3, 20, 128, True, 0, 0, 0.0, 0),        # fewer keys than one tile
    (1, 8, 8, 5, 3, 128, True, 0, 0, 0.0, 0),         # more queries than keys: empty rows
    (1, 4, 1, 4, 3000, 128, True, 512, 4, 0.0, 2),    # window + sinks
    (1, 4, 2, 2, 2000, 128, True, 300, 0, 30.0, 0),   # window + soft-cap
    (1, 4, 4, 1, 1500, 64, False, 0, 0, 0.0, 0),      # non-causal cross-attention
    (1, 2, 1, 7, 40000, 128, True, 0, 0, 0.0, 5),     # long cache, split-KV
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,window,n_sink,softcap,splits", CASES)
def test_ext_matches_oracle(fa, B, Hq, Hkv, Nq, Nk, d, causal, window, n_sink, softcap, splits):
    q, k, v = workloads.random_cross_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nq + 7 * Nk + n_sink)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    o, lse = run_ext(fa, q, k, v, causal=causal, window=window, n_sink=n_sink, softcap=softcap,
                     num_splits=splits, scale=scale)
    ro, rlse = oracle.attention(q, k, v, scale=scale, causal=causal, window=window, n_sink=n_sink, softcap=softcap)
    compare_rows(o, lse, ro, rlse)


def test_ext_self_attention_is_fa_fwd(fa):
    """Nq == Nk, no sinks, no split: the same kernel as fa_fwd, bit for bit."""
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in workloads.random_inputs(1, 4, 2, 777, 128, seed=31))
    o1, l1 = fa.forward(q, k, v, causal=True, window=300)
    o2, l2 = fa.forward_ext(q, k, v, causal=True, window=300)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_ext_no_keys(fa):
    """Nk == 0: every row is empty (O = 0, LSE = -inf); k and v may be NULL."""
    dev = torch.device("cuda:0")
    q = torch.randn(1, 2, 70, 64, device=dev).to(torch.bfloat16)
    o = torch.full_like(q, float("nan"))
    lse = torch.zeros(1, 2, 70, device=dev)
    lib = fa.load()
    rc = lib.fa_fwd_ext(ctypes.c_void_p(q.data_ptr()), None, None, ctypes.c_void_p(o.data_ptr()),
                        ctypes.c_void_p(lse.data_ptr()), 1, 2, 2, 70, 0, 64, 0.125, 1, 0, 0, 0.0, 0, None, 0,
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert bool((o == 0).all()) and bool(torch.isneginf(lse).all())


def test_ext_sinks_full_size_local_workload(fa):
    """The local soft-capped workload (B=2, H=16, N=32768, window 4096, cap 50) with 4
    attention sinks, at full size, compared on the standard row sample of four heads."""
    w = workloads.WORKLOADS["local_b2_h16_n32k_d128_w4k_cap50"]
    q, k, v = workloads.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = fa.forward_ext(qd, kd, vd, scale=w.scale, causal=True, window=w.window, n_sink=4, softcap=w.softcap)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    rows = workloads.sample_rows(w, workloads.standard_row_sample(w.N), heads=[0, 9, 20, 31])
    ro, rlse = oracle.attention(q, k, v, scale=w.scale, causal=True, window=w.window, n_sink=4, softcap=w.softcap,
                                rows=rows)
    rt = torch.from_numpy(rows).to(dev)
    compare_rows(o.reshape(-1, w.d)[rt].double().cpu().numpy(), lse.reshape(-1)[rt].double().cpu().numpy(), ro, rlse)


def test_decode_full_size_workload(fa):
    """One decoding step at full size (B=32, Hq=32, Hkv=8, Nk=16384), plain and with 4
    chunks, on a row sample of eight heads."""
    w = workloads.EXTRA_WORKLOADS["decode_b32_h32kv8_q1_k16k_d128"]
    q, k, v = workloads.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rows = workloads.sample_rows(w, [0], heads=[0, 1, 5, 100, 513, 777, 1000, 1023])
    ro, rlse = oracle.attention(q, k, v, scale=w.scale, causal=True, rows=rows)
    rt = torch.from_numpy(rows).to(dev)
    for splits in (0, 4):
        o, lse = fa.forward_ext(qd, kd, vd, scale=w.scale, causal=True, num_splits=splits)
        torch.cuda.synchronize()
        assert fa.check_status() == 0
        compare_rows(o.reshape(-1, w.d)[rt].double().cpu().numpy(), lse.reshape(-1)[rt].double().cpu().numpy(),
                     ro, rlse)


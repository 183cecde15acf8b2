"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by
element, on the same seeded inputs.

Tolerances (max-abs over every compared element):
  fp32 path (fa_fwd_f32): O 1e-5, LSE 1e-5
  bf16 path (fa_fwd):     O 2e-2, LSE 1e-3  (bf16 operands, fp32 accumulation)
Small shapes are compared in full; they span several 128-row / 128-key tiles and ragged
tails.  The five workloads run at full size in the same launch configuration the
benchmark times, and are compared on a deterministic sample of rows that the oracle
computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = {"float32": (1e-5, 1e-5), "bfloat16": (2e-2, 1e-3)}
GUARD = 4096  # guard-band elements before and after every output buffer


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import online_softmax_11_b200 as fa_mod
    from online_softmax_11_b200 import build
    build.build()
    fa_mod.load()
    return fa_mod


def guarded(shape, dtype, device):
    """A tensor of `shape` inside a larger buffer whose guard bands hold a NaN pattern."""
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device=device)
    buf.fill_(float("nan"))
    return buf, buf[GUARD:GUARD + n].view(shape)


def guards_intact(buf):
    n = buf.numel()
    head = buf[:GUARD]
    tail = buf[n - GUARD:]
    return bool(torch.isnan(head).all()) and bool(torch.isnan(tail).all())


def run_gpu(fa, q, k, v, *, scale, causal, window, softcap):
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, Hq, N, d = q.shape
    obuf, o = guarded((B, Hq, N, d), q.dtype, dev)
    lbuf, lse = guarded((B, Hq, N), torch.float32, dev)
    fa.forward(qd, kd, vd, scale=scale, causal=causal, window=window, softcap=softcap, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert guards_intact(obuf) and guards_intact(lbuf), "kernel wrote outside its outputs"
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def compare(o, lse, ro, rlse, dtype):
    tol_o, tol_l = TOL[dtype]
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    eo = float(np.max(np.abs(o - ro))) if o.size else 0.0
    el = float(np.max(np.abs(lse - rlse))) if lse.size else 0.0
    assert eo <= tol_o, f"O max-abs error {eo:.3e} > {tol_o}"
    assert el <= tol_l, f"LSE max-abs error {el:.3e} > {tol_l}"
    return eo, el


def check_full(fa, B, Hq, Hkv, N, d, dtype, causal=False, window=0, softcap=0.0, seed=0, q_mult=1.0, scale=None):
    q, k, v = workloads.random_inputs(B, Hq, Hkv, N, d, dtype=dtype, seed=seed, q_mult=q_mult)
    if scale is None:
        scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    o, lse = run_gpu(fa, q, k, v, scale=scale, causal=causal, window=window, softcap=softcap)
    ro, rlse = oracle.attention(q, k, v, scale=scale, causal=causal, window=window, softcap=softcap)
    return compare(o, lse, ro, rlse, dtype)


# ----------------------------------------------------------------------------- fp32 path

def test_modular_workload_fp32(fa):
    """n = 64, d = 32 modular inputs of nx_flashattn_scale.nx, fp32, full compare."""
    w = workloads.WORKLOADS["modular_n64_d32"]
    q, k, v = workloads.make_inputs(w)
    o, lse = run_gpu(fa, q, k, v, scale=w.scale, causal=False, window=0, softcap=0.0)
    ro, rlse = oracle.attention(q, k, v, scale=w.scale)
    compare(o, lse, ro, rlse, "float32")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,window,softcap", [
    (1, 1, 1, 1, 32, False, 0, 0.0),
    (1, 2, 2, 63, 32, True, 0, 0.0),
    (2, 2, 1, 65, 17, True, 0, 0.0),
    (1, 4, 2, 129, 64, True, 20, 0.0),
    (1, 2, 2, 200, 128, False, 0, 5.0),
    (1, 3, 3, 97, 1, True, 1, 0.0),
    (2, 4, 1, 150, 48, True, 33, 30.0),
])
def test_fp32_features(fa, B, Hq, Hkv, N, d, causal, window, softcap):
    check_full(fa, B, Hq, Hkv, N, d, "float32", causal, window, softcap, seed=N * 7 + d)


# ----------------------------------------------------------------------------- bf16 path

BF16_CASES = [
    # B, Hq, Hkv, N, d, causal, window, softcap, q_mult
    (1, 1, 1, 1, 64, False, 0, 0.0, 1.0),
    (1, 2, 2, 2, 128, True, 0, 0.0, 1.0),
    (1, 2, 2, 63, 64, False, 0, 0.0, 1.0),
    (1, 2, 2, 64, 128, True, 0, 0.0, 1.0),
    (2, 2, 2, 65, 64, True, 0, 0.0, 1.0),
    (1, 2, 2, 127, 128, False, 0, 0.0, 1.0),
    (1, 2, 2, 128, 128, True, 0, 0.0, 1.0),
    (1, 2, 2, 129, 128, True, 0, 0.0, 1.0),
    (1, 2, 2, 255, 64, True, 0, 0.0, 1.0),
    (1, 2, 2, 256, 128, False, 0, 0.0, 1.0),
    (1, 2, 2, 257, 128, True, 0, 0.0, 1.0),
    (2, 4, 1, 300, 128, True, 0, 0.0, 1.0),      # GQA, group 4
    (1, 4, 2, 513, 64, False, 0, 0.0, 1.0),      # GQA, group 2
    (1, 2, 2, 1000, 128, True, 0, 0.0, 1.0),
    (1, 2, 2, 700, 128, True, 1, 0.0, 1.0),      # window of one key: O = V
    (1, 2, 2, 700, 128, True, 5, 0.0, 1.0),
    (1, 2, 2, 900, 64, True, 200, 0.0, 1.0),
    (1, 2, 1, 1100, 128, True, 256, 50.0, 1.0),  # window + soft-cap
    (1, 2, 2, 333, 128, False, 0, 5.0, 1.0),     # tight soft-cap: general tanh path
    (1, 2, 2, 520, 128, True, 0, 20.0, 1.5),     # |s scale / cap| in (0.12, 0.3): long series
    (1, 2, 2, 520, 64, False, 0, 50.0, 1.0),     # |s scale / cap| < 0.12: short series
    (1, 2, 2, 600, 128, True, 0, 0.0, 8.0),      # large logits: running max moves a lot
    (1, 2, 2, 600, 64, False, 0, 0.0, 8.0),
    (1, 2, 2, 700, 128, True, 0, 50.0, 8.0),     # soft-cap with a moving maximum: O rescaled
    (1, 2, 1, 650, 64, True, 300, 30.0, 8.0),    # ... with a window, GQA and d = 64
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,window,softcap,q_mult", BF16_CASES)
def test_bf16_features(fa, B, Hq, Hkv, N, d, causal, window, softcap, q_mult):
    check_full(fa, B, Hq, Hkv, N, d, "bfloat16", causal, window, softcap, seed=N * 3 + d, q_mult=q_mult)


def test_bf16_temperature_scale(fa):
    """A temperature folds into the scale as 1/(T sqrt(d)) (oxios): T = 0.5 and T = 2."""
    for t in (0.5, 2.0):
        scale = float(np.float32(1.0 / (t * math.sqrt(128))))
        check_full(fa, 1, 2, 2, 260, 128, "bfloat16", True, 0, 0.0, seed=77, scale=scale)


# ----------------------------------------------------------------------------- full workloads

SAMPLE_HEADS = 8


def sampled_rows(w):
    nbh = w.B * w.Hq
    heads = sorted(set(np.linspace(0, nbh - 1, min(SAMPLE_HEADS, nbh)).round().astype(int).tolist()))
    rows = workloads.standard_row_sample(w.N)
    return workloads.sample_rows(w, rows, heads)


@pytest.mark.parametrize("name", [n for n in workloads.WORKLOADS if n != "modular_n64_d32"])
def test_workload_full_size(fa, name):
    """Full-size workload through the same call the benchmark times; O and LSE compared
    with the oracle on a deterministic row sample (8 heads spread over B*Hq; rows
    0..255, the last 256 and every 61st)."""
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.make_inputs(w)
    dev = torch.device("cuda:0")
    o = torch.empty(q.shape, dtype=q.dtype, device=dev)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    fa.forward(q.to(dev), k.to(dev), v.to(dev), scale=w.scale, causal=w.causal, window=w.window,
               softcap=w.softcap, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert bool(torch.isfinite(lse).all()) and bool(torch.isfinite(o.float()).all())
    rows = sampled_rows(w)
    ro, rlse = oracle.attention(q, k, v, scale=w.scale, causal=w.causal, window=w.window, softcap=w.softcap,
                                rows=rows)
    rows_t = torch.from_numpy(rows)
    og = o.reshape(-1, w.d)[rows_t.to(dev)].double().cpu().numpy()
    lg = lse.reshape(-1)[rows_t.to(dev)].double().cpu().numpy()
    compare(og, lg, ro, rlse, w.dtype)
    del o, lse
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- behaviour

def test_deterministic(fa):
    q, k, v = workloads.random_inputs(2, 4, 2, 777, 128, seed=5)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, l1 = fa.forward(qd, kd, vd, causal=True)
    o2, l2 = fa.forward(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_side_stream_and_no_lse(fa):
    q, k, v = workloads.random_inputs(1, 2, 2, 300, 64, seed=9)
    dev = torch.device("cuda:0")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        o = fa.forward(qd, kd, vd, causal=True, return_lse=False)
    s.synchronize()
    ro, _ = oracle.attention(q, k, v, scale=float(np.float32(1) / np.sqrt(np.float32(64))), causal=True)
    assert float(np.max(np.abs(o.double().cpu().numpy() - ro))) <= TOL["bfloat16"][0]


def test_empty_problem(fa):
    dev = torch.device("cuda:0")
    z = torch.empty((2, 2, 0, 128), dtype=torch.bfloat16, device=dev)
    o, lse = fa.forward(z, z, z)
    assert o.shape == z.shape and lse.shape == (2, 2, 0)


def test_bounded_wait_reports_timeout_and_device_stays_usable(fa):
    """Failure detection without a fault: a wait on a barrier nothing arrives at gives up
    after 20 ms, the kernel exits, FA_ERR_TIMEOUT is reported, and the next attention
    call on the same context is correct."""
    assert fa.selftest_wait_timeout(20000) == -7
    assert fa.check_status() == 0  # the status word was cleared
    check_full(fa, 1, 2, 2, 200, 128, "bfloat16", True, seed=3)

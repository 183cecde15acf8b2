"""GPU parity of the stand-alone softmax (fa_softmax) and the fused softmax + top-K
(fa_softmax_topk) against the fp64 oracle of "Online normalizer calculation for
softmax" (oracle/softmax.py), through the C ABI.

Tolerances, from the arithmetic: every output is exp2((x - m) log2 e) (approximate exp2,
relative error about 2^-22) divided by an fp32 normaliser summed over V terms in a tree
(relative error a few 1e-7 at V = 10^5).  x - m is exact near the maximum and rounded
relative to |x - m| elsewhere; with the product's rounding the exponent is off by at most
about |x - m| 2^-23, a relative output error below 1e-5 while exp(x - m) is above the
fp32 normal range (|x - m| < 87; smaller outputs flush to zero, hence the absolute slack
of 1e-38).  Bound used: relative 1e-5 on every probability, 1e-5 absolute on the LSE
(1e-4 for LSE near 1000, one fp32 ulp there being 6e-5).
Top-K indices are compared exactly where the K-th and (K+1)-th inputs differ (with
continuous random inputs they always do); ties are checked for validity.
"""
import numpy as np
import pytest
import torch

from oracle import softmax as osm

pytestmark = pytest.mark.gpu

REL, LSE_ABS = 1e-5, 1e-5


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import online_softmax_11_b200 as fa_mod
    from online_softmax_11_b200 import build
    build.build()
    fa_mod.load()
    return fa_mod


def logits(rows, V, seed, scale=4.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((rows, V), generator=g, dtype=torch.float32) * scale


# long rows (up to a million floats: the second read of a row then comes from HBM)
SHAPES = [(1, 1), (3, 5), (4, 127), (2, 1000), (5, 4099), (3, 16384), (2, 32000), (2, 50257), (2, 65536),
          (2, 70001), (3, 100003), (1, 262144), (2, 1000000)]


@pytest.mark.parametrize("rows,V", SHAPES)
def test_softmax_matches_oracle(fa, rows, V):
    x = logits(rows, V, 1000 + V)
    y, lse = fa.softmax(x.cuda(), return_lse=True)
    torch.cuda.synchronize()
    ry, rl = osm.softmax(x)
    yd = y.double().cpu().numpy()
    assert np.all(np.abs(yd - ry) <= REL * ry + 1e-38)
    assert np.max(np.abs(lse.double().cpu().numpy() - rl)) <= LSE_ABS


def test_softmax_unaligned_rows_and_large_range(fa):
    """V not a multiple of 4 (rows start off the 16-byte boundary: scalar head and tail)
    and inputs shifted by 1000 (exp would overflow without the maximum)."""
    x = logits(7, 1023, 5) + 1000.0
    y, lse = fa.softmax(x.cuda(), return_lse=True)
    torch.cuda.synchronize()
    ry, rl = osm.softmax(x)
    assert np.all(np.isfinite(y.cpu().numpy()))
    assert np.all(np.abs(y.double().cpu().numpy() - ry) <= REL * ry + 1e-38)
    assert np.max(np.abs(lse.double().cpu().numpy() - rl)) <= 1e-4  # |lse| ~ 1000: fp32 ulp is 6e-5


def test_softmax_empty_rows(fa):
    lse = torch.zeros(3, device="cuda")
    rc = fa.load().fa_softmax(None, None, lse.data_ptr(), 3, 0, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and bool(torch.isneginf(lse).all())


@pytest.mark.parametrize("rows,V,k", [(3, 5, 5), (4, 127, 1), (2, 1000, 4), (5, 4099, 5), (3, 32000, 8),
                                      (2, 50257, 16), (2, 32000, 32), (1, 262144, 10)])
def test_topk_matches_oracle(fa, rows, V, k):
    x = logits(rows, V, 2000 + V + k)
    probs, idx, lse = fa.softmax_topk(x.cuda(), k)
    torch.cuda.synchronize()
    rp, ri, rl = osm.softmax_topk(x, k)
    assert np.array_equal(idx.cpu().numpy().astype(np.int64), ri)
    assert np.all(np.abs(probs.double().cpu().numpy() - rp) <= REL * rp + 1e-38)
    assert np.max(np.abs(lse.double().cpu().numpy() - rl)) <= LSE_ABS


def test_topk_ties_go_to_lower_index(fa):
    """Equal inputs: the lower index comes first (the library's rule), checked on rows of
    constant value and on a planted tie at the top."""
    x = logits(3, 4096, 77)
    x[0, :] = 2.0
    x[1, [100, 7, 3000]] = 50.0
    x[2, 4095] = 60.0
    x[2, 0] = 60.0
    probs, idx, _ = fa.softmax_topk(x.cuda(), 4)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    assert idx[0].tolist() == [0, 1, 2, 3]
    assert idx[1, :3].tolist() == [7, 100, 3000]
    assert idx[2, :2].tolist() == [0, 4095]
    rp, ri, _ = osm.softmax_topk(x, 4)
    assert np.array_equal(idx.astype(np.int64), ri)
    assert np.all(np.abs(probs.double().cpu().numpy() - rp) <= REL * rp)


def test_topk_with_masked_inputs(fa):
    """-inf inputs (masked logits) take part like any value and never beat a finite one."""
    x = logits(2, 300, 9)
    x[0, 10:] = float("-inf")
    probs, idx, lse = fa.softmax_topk(x.cuda(), 12)
    torch.cuda.synchronize()
    rp, ri, rl = osm.softmax_topk(x, 12)
    assert np.array_equal(idx.cpu().numpy().astype(np.int64), ri)
    assert np.all(np.abs(probs.double().cpu().numpy() - rp) <= REL * rp)
    assert np.max(np.abs(lse.double().cpu().numpy() - rl)) <= LSE_ABS

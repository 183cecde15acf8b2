"""GPU parity of split-KV (fa_fwd_splitkv): every chunk count gives the oracle's result.

The keys of each query row are cut into chunks whose partial (O_s, LSE_s) are merged
with the two-block merge identities of "Module 16: Efficient and Long Attention",
section 16.2; the result must match the fp64 oracle within the bf16 tolerances
(O 2e-2, LSE 1e-3) and agree with the unsplit kernel."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.test_parity_gpu import TOL, compare

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


CASES = [
    # B, Hq, Hkv, N, d, causal, window, softcap, splits
    (1, 2, 2, 1, 128, False, 0, 0.0, 1),
    (2, 4, 2, 1000, 64, True, 0, 0.0, 1),     # one chunk over several query-tile pairs
    (1, 2, 2, 700, 128, False, 0, 0.0, 1),
    (1, 2, 2, 300, 128, False, 0, 0.0, 2),
    (2, 4, 2, 513, 64, False, 0, 0.0, 3),
    (1, 2, 2, 1000, 128, True, 0, 0.0, 4),
    (1, 2, 1, 700, 128, True, 200, 0.0, 3),
    (1, 2, 2, 640, 128, True, 0, 30.0, 2),
    (1, 2, 2, 257, 64, True, 0, 0.0, 7),      # more chunks than key tiles: empty chunks
    (1, 1, 1, 1100, 128, False, 0, 0.0, 64),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,window,softcap,splits", CASES)
def test_splitkv_matches_oracle(fa, B, Hq, Hkv, N, d, causal, window, softcap, splits):
    q, k, v = workloads.random_inputs(B, Hq, Hkv, N, d, seed=N + splits, q_mult=1.0)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = fa.forward_splitkv(qd, kd, vd, num_splits=splits, scale=scale, causal=causal, window=window,
                                softcap=softcap)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    ro, rlse = oracle.attention(q, k, v, scale=scale, causal=causal, window=window, softcap=softcap)
    compare(o.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rlse, "bfloat16")
    # and against the unsplit kernel (both are within the tolerance of the oracle; here the
    # difference is only the rounding of the per-chunk normalisation)
    o1, lse1 = fa.forward(qd, kd, vd, scale=scale, causal=causal, window=window, softcap=softcap)
    torch.cuda.synchronize()
    assert float((o1.float() - o.float()).abs().max()) <= TOL["bfloat16"][0]
    assert float((lse1 - lse).abs().max()) <= TOL["bfloat16"][1]


def test_splitkv_full_size_d64_workload(fa):
    """B=4 H=16 N=1024 d=64 with 1, 2 and 4 chunks, compared on the standard row sample."""
    w = workloads.WORKLOADS["mha_b4_h16_n1k_d64"]
    q, k, v = workloads.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    rows = workloads.sample_rows(w, workloads.standard_row_sample(w.N), heads=[0, 17, 40, 63])
    ro, rlse = oracle.attention(q, k, v, scale=w.scale, rows=rows)
    for splits in (1, 2, 4):
        o, lse = fa.forward_splitkv(qd, kd, vd, num_splits=splits, scale=w.scale)
        torch.cuda.synchronize()
        assert fa.check_status() == 0
        rt = torch.from_numpy(rows).to(dev)
        compare(o.reshape(-1, w.d)[rt].double().cpu().numpy(), lse.reshape(-1)[rt].double().cpu().numpy(), ro, rlse,
                "bfloat16")


def test_splitkv_rejects_small_workspace(fa):
    q, k, v = workloads.random_inputs(1, 2, 2, 256, 64, seed=1)
    dev = torch.device("cuda:0")
    ws = torch.empty(64, dtype=torch.uint8, device=dev)
    with pytest.raises(fa.FAError) as e:
        fa.forward_splitkv(q.to(dev), k.to(dev), v.to(dev), num_splits=2, workspace=ws)
    assert e.value.code == -8

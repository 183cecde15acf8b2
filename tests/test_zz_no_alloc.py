"""fa_fwd_splitkv_static: split-KV attention for callers that cannot allocate device memory.

Some callers (programs under a fixed device-memory plan that may not call cudaMalloc once
running, plug-ins inside a framework that owns all device memory) cannot hand the
library a workspace.  fa_fwd_splitkv_static takes none: its scratch is a fixed 32 MiB
array inside the library.  These checks call it through the C ABI and compare it with
fa_fwd_splitkv (caller workspace) on two calls in a row, with the tolerances of the
other bf16 parity tests (O 2e-2, LSE 1e-3), and check that a problem too large for the
array is refused.  The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import online_softmax_11_b200 as fa_mod
    from online_softmax_11_b200 import build
    build.build()
    fa_mod.load()
    return fa_mod


def _static_call(fa, q, k, v, o, lse, *, causal, window, softcap, num_splits):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    scale = float(np.float32(1.0) / np.sqrt(np.float32(d)))
    return fa.load().fa_fwd_splitkv_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, N, d, scale, int(causal),
        int(window), float(softcap), int(num_splits), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_workspace_entry_point_twice(fa):
    dev = torch.device("cuda:0")
    cases = [
        # B, Hq, Hkv, N, d, causal, window, softcap, num_splits, seed
        (2, 4, 2, 700, 128, True, 0, 0.0, 3, 101),
        (1, 2, 2, 333, 64, False, 0, 30.0, 2, 202),   # a smaller second call: old contents remain
    ]
    for B, Hq, Hkv, N, d, causal, window, softcap, splits, seed in cases:
        q, k, v = (t.to(dev) for t in workloads.random_inputs(B, Hq, Hkv, N, d, seed=seed))
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        rc = _static_call(fa, q, k, v, o, lse, causal=causal, window=window, softcap=softcap, num_splits=splits)
        assert rc == 0, fa.load().fa_strerror(rc)
        ro, rlse = fa.forward_splitkv(q, k, v, num_splits=splits, causal=causal, window=window, softcap=softcap)
        torch.cuda.synchronize()
        assert fa.check_status() == 0
        assert float((o.float() - ro.float()).abs().max()) <= TOL_O
        assert float((lse - rlse).abs().max()) <= TOL_LSE


def test_static_scratch_refuses_too_large_problems(fa):
    # 2 x 32 x 4096 rows x 129 floats x 4 chunks is far above the 32 MiB array
    lib = fa.load()
    need = lib.fa_fwd_splitkv_workspace(2, 32, 4096, 128, 4)
    assert need > fa.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    rc = lib.fa_fwd_splitkv_static(fake, fake, fake, fake, fake, 2, 32, 32, 4096, 128, 0.088, 1, 0, 0.0, 4, None)
    assert rc == -9

"""fa_fwd_splitkv_static: split-KV attention for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: programs that run under a fixed
device-memory plan and may not call cudaMalloc once they are running (cudaMalloc and
cudaFree can also synchronise the device), and plug-ins inside a framework that owns
all device memory and offers no scratch.  fa_fwd_splitkv_static takes no workspace; its
scratch is a fixed 32 MiB array inside the library, shared by every call.

These checks call it through the C ABI and compare it with fa_fwd_splitkv (caller
workspace) on the same inputs and chunk count: both run the same kernels, so O and LSE
must be identical bit for bit.  Each result is also compared with the fp64 oracle
element by element (O 2e-2, LSE 1e-3, the bf16 tolerances of the other parity tests).
NaN guard bands around O and LSE catch writes outside the outputs.  The cases run in a
row on the shared array, the largest first, so later calls find stale partial results
from earlier ones there; they cover the tensor-core kernel and the decode kernel (few
query rows per key/value head), one chunk and several, and the size limit exactly:
the largest problem that fits is accepted, one more query row is refused.  The file is
named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL_O, TOL_LSE = 2e-2, 1e-3
GUARD = 4096


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import online_softmax_11_b200 as fa_mod
    from online_softmax_11_b200 import build
    build.build()
    fa_mod.load()
    return fa_mod


def _guarded(shape, dtype, dev):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device=dev)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _intact(buf):
    return bool(torch.isnan(buf[:GUARD]).all()) and bool(torch.isnan(buf[-GUARD:]).all())


def _scale(d):
    return float(np.float32(1.0) / np.sqrt(np.float32(d)))


def _static_call(fa, q, k, v, o, lse, *, causal, window, softcap, num_splits):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    return fa.load().fa_fwd_splitkv_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, Hq, Hkv, N, d, _scale(d), int(causal),
        int(window), float(softcap), int(num_splits), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _largest_fitting_n(fa, d, splits):
    """The largest single-head N whose split-KV scratch fits the static array."""
    lib = fa.load()
    per_row = lib.fa_fwd_splitkv_workspace(1, 1, 1, d, splits)
    n = int(fa.STATIC_SCRATCH_BYTES // per_row)
    assert lib.fa_fwd_splitkv_workspace(1, 1, n, d, splits) <= fa.STATIC_SCRATCH_BYTES
    assert lib.fa_fwd_splitkv_workspace(1, 1, n + 1, d, splits) > fa.STATIC_SCRATCH_BYTES
    return n


def _check_case(fa, B, Hq, Hkv, N, d, causal, window, softcap, splits, seed, oracle_rows=None):
    dev = torch.device("cuda:0")
    qh, kh, vh = workloads.random_inputs(B, Hq, Hkv, N, d, seed=seed)
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    obuf, o = _guarded((B, Hq, N, d), torch.bfloat16, dev)
    lbuf, lse = _guarded((B, Hq, N), torch.float32, dev)
    rc = _static_call(fa, q, k, v, o, lse, causal=causal, window=window, softcap=softcap, num_splits=splits)
    assert rc == 0, fa.load().fa_strerror(rc)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert _intact(obuf) and _intact(lbuf), "fa_fwd_splitkv_static wrote outside O / LSE"
    # the caller-workspace entry point on the same inputs and chunk count: the same bits
    ro, rl = fa.forward_splitkv(q, k, v, num_splits=splits, scale=_scale(d), causal=causal, window=window,
                                softcap=softcap)
    torch.cuda.synchronize()
    assert fa.check_status() == 0
    assert torch.equal(o, ro) and torch.equal(lse, rl), "static scratch and caller workspace disagree"
    # and the fp64 oracle, element by element (all rows, or a sample for the large case)
    if oracle_rows is None:
        xo, xl = oracle.attention(qh, kh, vh, scale=_scale(d), causal=causal, window=window, softcap=softcap)
        go, gl = o.double().cpu().numpy(), lse.double().cpu().numpy()
    else:
        xo, xl = oracle.attention(qh, kh, vh, scale=_scale(d), causal=causal, window=window, softcap=softcap,
                                  rows=oracle_rows)
        go = o.reshape(-1, d)[torch.as_tensor(oracle_rows, device=dev)].double().cpu().numpy()
        gl = lse.reshape(-1)[torch.as_tensor(oracle_rows, device=dev)].double().cpu().numpy()
    assert np.all(np.isfinite(go)) and np.all(np.isfinite(gl))
    assert float(np.max(np.abs(go - xo))) <= TOL_O
    assert float(np.max(np.abs(gl - xl))) <= TOL_LSE


def test_static_scratch_matches_workspace_entry_point_and_oracle(fa):
    n_max = _largest_fitting_n(fa, 128, 2)
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(n_max - 64, n_max),
                                     np.arange(0, n_max, 997)])).astype(np.int64)
    # the largest problem the array holds (it fills the array; later calls find its
    # partial results there)
    _check_case(fa, 1, 1, 1, n_max, 128, True, 0, 0.0, 2, seed=301, oracle_rows=rows)
    cases = [
        # B, Hq, Hkv, N, d, causal, window, softcap, num_splits, seed
        (2, 4, 2, 700, 128, True, 0, 0.0, 3, 101),
        (1, 2, 2, 333, 64, False, 0, 30.0, 2, 202),
        (1, 2, 2, 260, 128, True, 100, 0.0, 1, 303),    # one chunk
        (2, 4, 4, 3, 128, True, 0, 0.0, 4, 404),        # 3 rows per key/value head: decode kernel
        (1, 8, 2, 4, 64, False, 0, 0.0, 3, 505),        # GQA group of 4 x 4 rows = 16: decode kernel
    ]
    for B, Hq, Hkv, N, d, causal, window, softcap, splits, seed in cases:
        _check_case(fa, B, Hq, Hkv, N, d, causal, window, softcap, splits, seed)


def test_static_scratch_size_limit_is_exact(fa):
    """One query row more than the largest accepted problem is refused with
    FA_ERR_SCRATCH_LIMIT, before any device work."""
    lib = fa.load()
    n_max = _largest_fitting_n(fa, 128, 2)
    dev = torch.device("cuda:0")
    q = torch.zeros((1, 1, n_max + 1, 128), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, n_max + 1), dtype=torch.float32, device=dev)
    rc = _static_call(fa, q, q, q, o, lse, causal=True, window=0, softcap=0.0, num_splits=2)
    assert rc == -9
    # far above the limit, too
    need = lib.fa_fwd_splitkv_workspace(2, 32, 4096, 128, 4)
    assert need > fa.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    rc = lib.fa_fwd_splitkv_static(fake, fake, fake, fake, fake, 2, 32, 32, 4096, 128, 0.088, 1, 0, 0.0, 4, None)
    assert rc == -9

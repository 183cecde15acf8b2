"""C-ABI library checks that need no GPU: it builds, loads, exports every symbol the
header declares, and rejects bad arguments before touching any device."""
import ctypes
import os
import re

import pytest

import online_softmax_11_b200 as fa
from online_softmax_11_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    fabuild.build()
    return fa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_the_binding_knows():
    assert declared_functions() == sorted(fa.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_has_no_oracle_dependency():
    """The product library and binding never reference the CPU oracle."""
    for root, _, files in os.walk(os.path.join(ROOT, "online_softmax_11_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, f)).read()
                assert "import oracle" not in src and "from oracle" not in src and "attn_fp64" not in src, f


def test_strerror_and_version(lib):
    assert lib.fa_version() >= 100
    for code in range(0, -8, -1):
        assert lib.fa_strerror(code)
    assert b"unknown" in lib.fa_strerror(-99)


FAKE = 0x10000  # a 16-byte aligned non-NULL address; never dereferenced by these calls


def call(lib, fn="fa_fwd", q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=8, d=64, scale=0.125,
         causal=0, window=0, softcap=0.0):
    return getattr(lib, fn)(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window, softcap, None)


@pytest.mark.parametrize("fn", ["fa_fwd", "fa_fwd_f32"])
def test_argument_errors(lib, fn):
    assert call(lib, fn, B=-1) == -2
    assert call(lib, fn, N=-3) == -2
    assert call(lib, fn, Hkv=0) == -2
    assert call(lib, fn, Hq=3, Hkv=2) == -2
    assert call(lib, fn, B=1 << 20, Hq=1 << 10, N=1 << 10) == -2  # rows overflow int32
    assert call(lib, fn, scale=0.0) == -5
    assert call(lib, fn, scale=-1.0) == -5
    assert call(lib, fn, scale=float("inf")) == -5
    assert call(lib, fn, scale=float("nan")) == -5
    assert call(lib, fn, softcap=float("nan")) == -5
    assert call(lib, fn, window=16, causal=0) == -3
    assert call(lib, fn, q=None) == -1
    assert call(lib, fn, o=None) == -1
    assert call(lib, fn, d=0) == -3
    assert call(lib, fn, d=129) == -3


def test_bf16_specific_errors(lib):
    assert call(lib, d=32) == -3
    assert call(lib, d=96) == -3
    assert call(lib, q=FAKE + 8) == -4
    assert call(lib, o=FAKE + 2) == -4
    assert call(lib, lse=FAKE + 2) == -4


def test_f32_alignment(lib):
    assert call(lib, "fa_fwd_f32", d=32, v=FAKE + 2) == -4


@pytest.mark.parametrize("fn", ["fa_fwd", "fa_fwd_f32"])
def test_empty_problems_are_noops(lib, fn):
    """B == 0, Hq == 0 or N == 0 return OK without touching memory (NULL pointers are
    accepted for an empty problem), like oxios' empty-input case."""
    assert call(lib, fn, q=None, k=None, v=None, o=None, lse=None, B=0) == 0
    assert call(lib, fn, q=None, k=None, v=None, o=None, lse=None, N=0) == 0
    assert call(lib, fn, q=None, k=None, v=None, o=None, lse=None, Hq=0, Hkv=1) == 0


def test_selftest_rejects_bad_limits(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == -5
    assert lib.fa_selftest_wait_timeout(2_000_000, None) == -5


def test_build_command_targets_sm100a_only():
    cmd = fabuild.command()
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert not any("sm_90" in c or "sm_80" in c for c in cmd)


def call_split(lib, num_splits=2, ws=FAKE, ws_bytes=1 << 30, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=8, d=64, scale=0.125, causal=0,
             window=0, softcap=0.0)
    a.update(kw)
    return lib.fa_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                              a["scale"], a["causal"], a["window"], a["softcap"], num_splits, ws, ws_bytes, None)


def test_splitkv_workspace_size(lib):
    # num_splits x rows x (d + 1) floats
    assert lib.fa_fwd_splitkv_workspace(2, 3, 5, 64, 4) == 4 * 2 * 3 * 5 * 65 * 4
    assert lib.fa_fwd_splitkv_workspace(0, 3, 5, 64, 4) == 0
    assert lib.fa_fwd_splitkv_workspace(1, 1, 1, 128, 0) == 0


def test_splitkv_argument_errors(lib):
    assert call_split(lib, num_splits=0) == -5
    assert call_split(lib, num_splits=fa.MAX_SPLITS + 1) == -5
    assert call_split(lib, ws=None) == -8
    assert call_split(lib, ws=FAKE + 4) == -8
    assert call_split(lib, ws_bytes=16) == -8
    assert call_split(lib, d=32) == -3
    assert call_split(lib, Hq=3) == -2
    assert call_split(lib, q=None, k=None, v=None, o=None, lse=None, ws=None, N=0) == 0  # empty problem


def call_ext(lib, num_splits=0, ws=None, ws_bytes=0, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, Nq=8, Nk=8, d=64, scale=0.125, causal=1,
             window=0, n_sink=0, softcap=0.0)
    a.update(kw)
    return lib.fa_fwd_ext(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                          a["d"], a["scale"], a["causal"], a["window"], a["n_sink"], a["softcap"], num_splits, ws,
                          ws_bytes, None)


def test_ext_argument_errors(lib):
    assert call_ext(lib, Nq=-1) == -2
    assert call_ext(lib, Nk=-1) == -2
    assert call_ext(lib, n_sink=-1) == -5
    assert call_ext(lib, num_splits=-1) == -5
    assert call_ext(lib, num_splits=fa.MAX_SPLITS + 1) == -5
    assert call_ext(lib, num_splits=2) == -8                      # split-KV needs a workspace
    assert call_ext(lib, num_splits=2, ws=FAKE, ws_bytes=16) == -8
    assert call_ext(lib, window=4, causal=0) == -3
    assert call_ext(lib, d=96) == -3
    assert call_ext(lib, q=None) == -1
    assert call_ext(lib, k=None) == -1                            # keys present, pointer missing
    assert call_ext(lib, B=1 << 16, Hkv=2, Nk=1 << 16) == -2      # key rows overflow int32
    assert call_ext(lib, q=None, k=None, v=None, o=None, lse=None, Nq=0) == 0   # no queries: empty
    assert call_ext(lib, q=None, k=None, v=None, o=None, lse=None, B=0) == 0


def test_softmax_argument_errors(lib):
    assert lib.fa_softmax(FAKE, FAKE, None, -1, 8, None) == -2
    assert lib.fa_softmax(FAKE, FAKE, None, 2, -8, None) == -2
    assert lib.fa_softmax(None, FAKE, None, 2, 8, None) == -1
    assert lib.fa_softmax(FAKE + 4, FAKE, None, 2, 8, None) == -4
    assert lib.fa_softmax(FAKE, FAKE + 8, None, 2, 8, None) == -4
    assert lib.fa_softmax(None, None, None, 0, 8, None) == 0      # no rows
    assert lib.fa_softmax_topk(FAKE, FAKE, FAKE, None, 2, 8, 0, None) == -5
    assert lib.fa_softmax_topk(FAKE, FAKE, FAKE, None, 2, 8, 9, None) == -5     # K > V
    assert lib.fa_softmax_topk(FAKE, FAKE, FAKE, None, 2, 100, 33, None) == -5  # K > 32
    assert lib.fa_softmax_topk(FAKE, None, FAKE, None, 2, 100, 4, None) == -1
    assert lib.fa_softmax_topk(FAKE + 4, FAKE, FAKE, None, 2, 100, 4, None) == -4
    assert lib.fa_softmax_topk(None, None, None, None, 0, 100, 4, None) == 0


"""fp64 CPU oracle for the FlashAttention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this package.
It shares no code with ``online_softmax_11_b200`` and never imports it; the product
path must never route through here.

Contents
--------
``attention(q, k, v, ...)``
    The dense definition of attention in fp64 (``attn_fp64.c``): per query row the
    whole score row is built, soft-capped, masked, max-subtracted, exponentiated,
    normalised and multiplied by V.  Sources: the dense line of the worked example in
    "Online Softmax Without the Attention Matrix"; the "DIRECT softmax reference" of
    nx_flashattn_scale.nx; ``naive_attention`` in oxios flash_attention.rs.
``softcap(z, kappa)``
    Logit soft-capping ``kappa * tanh(z / kappa)`` ("Module 16: Efficient and Long
    Attention", section 16.5).
``merge(m1, l1, o1, m2, l2, o2)``
    The two-block merge identities of Module 16, section 16.2: the combined sum
    ``l = e^(m1-m) l1 + e^(m2-m) l2`` and the combined output that weights each
    block's normalised output by its share ``e^(mi-m) li / l``.
``flops(...)``
    The attention FLOP count used to convert times into TFLOP/s (4 d per valid
    (query, key) pair; the closed forms 4 B Hq N^2 d, halved for causal, and
    4 B Hq d (N W - W^2/2) for a causal window are reported beside it).

``softmax.softmax(x)``, ``softmax.softmax_topk(x, k)``
    The classical softmax of each row in fp64 and its top-K with probabilities
    ("Online normalizer calculation for softmax"; see ``oracle/softmax.py``).

Every function is pinned by ``tests/test_oracle_pins.py`` against values the pages
print, closed forms, invariants and a library softmax.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_fp64.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_fp64.so")
_lock = threading.Lock()
_lib = None

DTYPE_CODES = {"float64": 0, "float32": 1, "bfloat16": 2}
_ARGTYPES = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
             ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
             ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
             ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]


def build(force: bool = False) -> str:
    """Compile ``attn_fp64.c`` into ``liboracle_fp64.so`` next to it (plain IEEE fp64:
    no fast-math, no FMA contraction, baseline x86-64 so the same file runs on any
    host this repository is copied to)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-pthread", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def load_library(path: str):
    """ctypes handle for an oracle library built from ``attn_fp64.c`` at ``path``."""
    lib = ctypes.CDLL(path)
    f = lib.oracle_attn_fp64
    f.restype = ctypes.c_int
    f.argtypes = _ARGTYPES
    return lib


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _as_host_array(t):
    """(contiguous numpy array, dtype code).  bf16 torch tensors are passed as their raw
    16-bit patterns; the C side widens them exactly."""
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), DTYPE_CODES["bfloat16"]
        if t.dtype == torch.float32:
            return t.numpy(), DTYPE_CODES["float32"]
        if t.dtype == torch.float64:
            return t.numpy(), DTYPE_CODES["float64"]
        raise TypeError(f"oracle: unsupported dtype {t.dtype}")
    a = np.ascontiguousarray(t)
    if a.dtype == np.float64:
        return a, 0
    if a.dtype == np.float32:
        return a, 1
    if a.dtype == np.uint16:  # bf16 bit patterns
        return a, 2
    raise TypeError(f"oracle: unsupported dtype {a.dtype}")


def attention(q, k, v, *, scale: float, causal: bool = False, window: int = 0, n_sink: int = 0,
              softcap: float = 0.0, rows=None, nthreads: int | None = None, _lib=None):
    """Dense fp64 attention.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (torch or numpy; fp64, fp32 or bf16 — all
    three the same type).  Self-attention has Nq == Nk; with Nq < Nk the queries are the
    last Nq positions of the key sequence for the causal and window masks.
    ``n_sink``: the first ``n_sink`` keys are attention sinks, exempt from the window
    (Module 16, section 16.6); they stay under the causal mask.
    ``rows``: optional flat row indices ``(b*Hq + hq)*Nq + i``.
    Returns ``(O, LSE)`` as float64 numpy arrays: ``O[B,Hq,Nq,d]``, ``LSE[B,Hq,Nq]`` for
    all rows, or ``O[len(rows), d]``, ``LSE[len(rows)]`` for a row subset.
    """
    qa, qt = _as_host_array(q)
    ka, kt = _as_host_array(k)
    va, vt = _as_host_array(v)
    if not (qt == kt == vt):
        raise TypeError("oracle: q, k, v must share one dtype")
    if qa.ndim != 4 or ka.ndim != 4 or va.ndim != 4:
        raise ValueError("oracle: expected 4-D [B, H, N, d] inputs")
    B, Hq, N, d = qa.shape
    Bk, Hkv, Nk, dk = ka.shape
    if (Bk, dk) != (B, d) or va.shape != ka.shape:
        raise ValueError("oracle: q/k/v shapes disagree")
    if rows is not None:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = rows_a.size
        o = np.zeros((nrows, d), dtype=np.float64)
        lse = np.zeros((nrows,), dtype=np.float64)
        rows_ptr = rows_a.ctypes.data
    else:
        rows_a = None
        nrows = B * Hq * N
        o = np.zeros((B, Hq, N, d), dtype=np.float64)
        lse = np.zeros((B, Hq, N), dtype=np.float64)
        rows_ptr = None
    if nthreads is None:
        nthreads = host_threads()
    lib = _lib if _lib is not None else _load()
    rc = lib.oracle_attn_fp64(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, qt,
                                  B, Hq, Hkv, N, Nk, d, float(scale), int(bool(causal)), int(window),
                                  int(n_sink), float(softcap), rows_ptr, nrows, o.ctypes.data, lse.ctypes.data,
                                  int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_fp64 failed with status {rc}")
    return o, lse


def softcap(z, kappa):
    """Soft-capped logit ``kappa * tanh(z / kappa)`` (Module 16, section 16.5)."""
    return kappa * np.tanh(np.asarray(z, dtype=np.float64) / kappa)


def merge(m1, l1, o1, m2, l2, o2):
    """Combine two blocks of one softmax row (Module 16, section 16.2).

    Each block i has its own maximum ``mi``, its sum ``li`` of ``exp(x - mi)`` and its
    normalised output ``oi``.  With ``m = max(m1, m2)``:
    ``l = e^(m1-m) l1 + e^(m2-m) l2`` and
    ``o = (e^(m1-m) l1 / l) o1 + (e^(m2-m) l2 / l) o2``.
    Returns ``(m, l, o)``.
    """
    m = np.maximum(m1, m2)
    w1 = np.exp(np.asarray(m1, dtype=np.float64) - m) * l1
    w2 = np.exp(np.asarray(m2, dtype=np.float64) - m) * l2
    l = w1 + w2
    o = (w1 / l)[..., None] * np.asarray(o1, dtype=np.float64) + (w2 / l)[..., None] * np.asarray(o2, dtype=np.float64)
    return m, l, o


def valid_pairs(N: int, causal: bool, window: int) -> int:
    """Number of (query i, key j) pairs that the mask keeps for one head."""
    if not causal and window <= 0:
        return N * N
    total = 0
    for i in range(N):
        lo = 0 if window <= 0 else max(0, i - window + 1)
        hi = i if causal else N - 1
        if hi >= lo:
            total += hi - lo + 1
    return total


def valid_pairs_closed(N: int, causal: bool, window: int) -> int:
    """Closed form of ``valid_pairs`` (same count, O(1))."""
    if not causal:
        if window <= 0:
            return N * N
        raise ValueError("a window without causal masking is not a workload here")
    if window <= 0 or window >= N:
        return N * (N + 1) // 2
    W = window
    return W * (W + 1) // 2 + (N - W) * W


def flops(B: int, Hq: int, N: int, d: int, causal: bool = False, window: int = 0,
          convention: str = "pairs") -> float:
    """Tensor-core FLOPs of one forward pass: 2 d for Q.K^T plus 2 d for P.V per valid
    pair (``convention="pairs"``), or the closed convention 4 B Hq N^2 d, halved for
    causal, 4 B Hq d (N W - W^2/2) for a causal window (``convention="closed"``)."""
    if convention == "pairs":
        return 4.0 * d * B * Hq * valid_pairs_closed(N, causal, window)
    if window > 0:
        return 4.0 * B * Hq * d * (N * window - window * window / 2.0)
    f = 4.0 * B * Hq * N * N * d
    return f / 2.0 if causal else f


def row_flops(N: int, d: int, causal: bool, window: int, i: int) -> float:
    """FLOPs (4 d per valid key) for query row i."""
    lo = 0 if window <= 0 else max(0, i - window + 1)
    hi = i if causal else N - 1
    return 4.0 * d * max(0, hi - lo + 1)


__all__ = ["attention", "softcap", "merge", "flops", "valid_pairs", "valid_pairs_closed",
           "row_flops", "build", "load_library", "host_threads"]

"""B200 (sm_100a) FlashAttention forward pass: Python binding of ``libfa_sm100.so``.

This module only marshals arguments: it checks tensors, takes their device pointers and
the current CUDA stream, and calls the C ABI declared in ``include/fa.h``.  Every step
of the attention itself runs in the library's CUDA kernels; there is no fallback.  If
the library is missing, every call raises.

    import online_softmax_11_b200 as fa
    o, lse = fa.forward(q, k, v, causal=True)                 # bf16, d in {64, 128}
    o, lse = fa.forward(q32, k32, v32)                        # fp32, 1 <= d <= 128

Layout: q [B, Hq, N, d], k and v [B, Hkv, N, d], contiguous CUDA tensors; returns
o [B, Hq, N, d] (same dtype as q) and lse [B, Hq, N] float32 (natural log).
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")

FA_OK = 0
ERRORS = {
    -1: "FA_ERR_NULL_PTR",
    -2: "FA_ERR_BAD_SHAPE",
    -3: "FA_ERR_UNSUPPORTED",
    -4: "FA_ERR_ALIGN",
    -5: "FA_ERR_BAD_ARG",
    -6: "FA_ERR_CUDA",
    -7: "FA_ERR_TIMEOUT",
    -8: "FA_ERR_WORKSPACE",
    -9: "FA_ERR_SCRATCH_LIMIT",
}
STATIC_SCRATCH_BYTES = 32 << 20
MAX_SPLITS = 64
# every symbol include/fa.h declares
EXPORTS = ["fa_fwd", "fa_fwd_f32", "fa_fwd_ext", "fa_softmax", "fa_softmax_topk", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace", "fa_fwd_splitkv_static",
           "fa_check_status", "fa_selftest_wait_timeout", "fa_strerror", "fa_last_cuda_error", "fa_version"]

_lock = threading.Lock()
_lib = None


class FAError(RuntimeError):
    def __init__(self, code: int, lib=None, what: str = ""):
        name = ERRORS.get(code, str(code))
        msg = name
        if lib is not None:
            msg += ": " + lib.fa_strerror(code).decode()
            if code == -6:
                msg += f" (cudaError {lib.fa_last_cuda_error()})"
        if what:
            msg = f"{what}: {msg}"
        super().__init__(msg)
        self.code = code


def load():
    """ctypes handle of ``libfa_sm100.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m online_softmax_11_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        sig = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, f, vp]
        for name in ("fa_fwd", "fa_fwd_f32"):
            fn = getattr(lib, name)
            fn.restype = i
            fn.argtypes = sig
        lib.fa_fwd_splitkv.restype = i
        lib.fa_fwd_splitkv.argtypes = sig[:-1] + [i, vp, ctypes.c_size_t, vp]
        lib.fa_fwd_splitkv_static.restype = i
        lib.fa_fwd_splitkv_static.argtypes = sig[:-1] + [i, vp]
        lib.fa_fwd_ext.restype = i
        lib.fa_fwd_ext.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, f, i, vp, ctypes.c_size_t, vp]
        lib.fa_softmax.restype = i
        lib.fa_softmax.argtypes = [vp, vp, vp, i, i, vp]
        lib.fa_softmax_topk.restype = i
        lib.fa_softmax_topk.argtypes = [vp, vp, vp, vp, i, i, i, vp]
        lib.fa_fwd_splitkv_workspace.restype = ctypes.c_size_t
        lib.fa_fwd_splitkv_workspace.argtypes = [i, i, i, i, i]
        lib.fa_check_status.restype = i
        lib.fa_check_status.argtypes = [vp]
        lib.fa_selftest_wait_timeout.restype = i
        lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        lib.fa_strerror.restype = ctypes.c_char_p
        lib.fa_strerror.argtypes = [i]
        lib.fa_last_cuda_error.restype = i
        lib.fa_last_cuda_error.argtypes = []
        lib.fa_version.restype = i
        lib.fa_version.argtypes = []
        _lib = lib
        return lib


def _stream_handle(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int | None, B: int, Hq: int, Hkv: int,
            N: int, d: int, scale: float, causal: bool, window: int, softcap: float, stream: int,
            dtype: str = "bfloat16") -> int:
    """Direct call of ``fa_fwd`` / ``fa_fwd_f32`` with raw device pointers; returns the
    status code."""
    lib = load()
    fn = lib.fa_fwd if dtype == "bfloat16" else lib.fa_fwd_f32
    return fn(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
              int(window), float(softcap), stream)


def forward(q, k, v, *, scale: float | None = None, causal: bool = False, window: int = 0,
            softcap: float = 0.0, out=None, lse=None, return_lse: bool = True, stream=None):
    """Attention forward through the C ABI.  ``scale`` defaults to 1/sqrt(d) in fp32."""
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] with q's B, N and d")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("q, k, v must all be bfloat16 or all float32")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if scale is None:
        scale = float(torch.tensor(1.0, dtype=torch.float32) / torch.sqrt(torch.tensor(float(d), dtype=torch.float32)))
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    dtype = "bfloat16" if q.dtype == torch.bfloat16 else "float32"
    with torch.cuda.device(q.device):
        rc = fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                     lse.data_ptr() if lse is not None else None, B, Hq, Hkv, N, d, scale, causal, window,
                     softcap, _stream_handle(stream), dtype)
    if rc != FA_OK:
        raise FAError(rc, load(), "fa_fwd" if dtype == "bfloat16" else "fa_fwd_f32")
    return (out, lse) if return_lse else out


def splitkv_workspace_bytes(B: int, Hq: int, N: int, d: int, num_splits: int) -> int:
    """Workspace bytes ``fa_fwd_splitkv`` needs."""
    return int(load().fa_fwd_splitkv_workspace(B, Hq, N, d, num_splits))


def forward_splitkv(q, k, v, *, num_splits: int, scale: float | None = None, causal: bool = False,
                    window: int = 0, softcap: float = 0.0, out=None, lse=None, workspace=None, stream=None):
    """Split-KV attention forward (bf16) through ``fa_fwd_splitkv``; the workspace is a
    caller tensor (allocated here with torch when not given)."""
    import torch
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("fa_fwd_splitkv takes bfloat16 q, k, v")
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] with q's B, N and d")
    for t in (q, k, v):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if scale is None:
        scale = float(torch.tensor(1.0, dtype=torch.float32) / torch.sqrt(torch.tensor(float(d), dtype=torch.float32)))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    need = splitkv_workspace_bytes(B, Hq, N, d, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        rc = load().fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq,
                                   Hkv, N, d, float(scale), int(bool(causal)), int(window), float(softcap),
                                   int(num_splits), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, load(), "fa_fwd_splitkv")
    return out, lse


def forward_ext(q, k, v, *, scale: float | None = None, causal: bool = False, window: int = 0, n_sink: int = 0,
                softcap: float = 0.0, num_splits: int = 0, out=None, lse=None, workspace=None, stream=None):
    """General bf16 forward through ``fa_fwd_ext``: q [B, Hq, Nq, d] against k, v
    [B, Hkv, Nk, d] (queries at the last Nq key positions), attention sinks beside a
    window, and split-KV when ``num_splits`` >= 1 (workspace allocated here with torch
    when not given)."""
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("fa_fwd_ext takes bfloat16 q, k, v")
    if k.shape != (B, Hkv, Nk, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, Nk, d] with q's B and d")
    for t in (q, k, v):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if scale is None:
        scale = float(torch.tensor(1.0, dtype=torch.float32) / torch.sqrt(torch.tensor(float(d), dtype=torch.float32)))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    ws_ptr, ws_bytes = None, 0
    if num_splits > 0:
        if workspace is None:
            need = splitkv_workspace_bytes(B, Hq, Nq, d, num_splits)
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    with torch.cuda.device(q.device):
        rc = load().fa_fwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                               Nq, Nk, d, float(scale), int(bool(causal)), int(window), int(n_sink), float(softcap),
                               int(num_splits), ws_ptr, ws_bytes, _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, load(), "fa_fwd_ext")
    return out, lse


def _check_rows(x, what):
    import torch
    if x.dim() != 2 or x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError(f"{what}: x must be a contiguous float32 CUDA tensor [rows, V]")


def softmax(x, *, out=None, lse=None, return_lse: bool = False, stream=None):
    """Row softmax of float32 ``x`` [rows, V] through ``fa_softmax`` (online normaliser)."""
    import torch
    _check_rows(x, "fa_softmax")
    rows, V = x.shape
    if out is None:
        out = torch.empty_like(x)
    if return_lse and lse is None:
        lse = torch.empty(rows, dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        rc = load().fa_softmax(x.data_ptr(), out.data_ptr(), lse.data_ptr() if lse is not None else None, rows, V,
                               _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, load(), "fa_softmax")
    return (out, lse) if return_lse else out


def softmax_topk(x, k: int, *, stream=None):
    """Fused softmax + top-``k`` of float32 ``x`` [rows, V] through ``fa_softmax_topk``.
    Returns (probs [rows, k] float32, idx [rows, k] int32, lse [rows] float32)."""
    import torch
    _check_rows(x, "fa_softmax_topk")
    rows, V = x.shape
    probs = torch.empty((rows, k), dtype=torch.float32, device=x.device)
    idx = torch.empty((rows, k), dtype=torch.int32, device=x.device)
    lse = torch.empty(rows, dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        rc = load().fa_softmax_topk(x.data_ptr(), probs.data_ptr(), idx.data_ptr(), lse.data_ptr(), rows, V, int(k),
                                    _stream_handle(stream))
    if rc != FA_OK:
        raise FAError(rc, load(), "fa_softmax_topk")
    return probs, idx, lse


def check_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return load().fa_check_status(_stream_handle(stream))


def selftest_wait_timeout(timeout_us: int = 20000, stream=None) -> int:
    """Run the bounded-wait self-test kernel; FA_ERR_TIMEOUT (-7) means it works."""
    return load().fa_selftest_wait_timeout(int(timeout_us), _stream_handle(stream))


def attention_flops(B: int, Hq: int, N: int, d: int, causal: bool = False, window: int = 0) -> float:
    """4 d FLOPs per (query, key) pair the mask keeps (2 d for Q K^T, 2 d for P V)."""
    if not causal:
        pairs = N * N
    elif window <= 0 or window >= N:
        pairs = N * (N + 1) // 2
    else:
        pairs = window * (window + 1) // 2 + (N - window) * window
    return 4.0 * d * B * Hq * pairs


__all__ = ["forward", "forward_ext", "forward_splitkv", "softmax", "softmax_topk", "splitkv_workspace_bytes", "fwd_raw", "load", "check_status",
           "selftest_wait_timeout", "attention_flops", "FAError", "EXPORTS", "LIB_PATH", "MAX_SPLITS"]

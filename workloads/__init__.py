"""Seeded synthetic inputs for the attention forward pass.

This module is shared by the tests, the smoke check and the benchmark, on both sides of
the parity check (the fp64 oracle and the CUDA library).  It holds shapes, seeds and
random-number generation only — none of the attention arithmetic.

Workloads
---------
``modular_n64_d32``  one head, N=64, d=32, fp32, non-causal, with the integer-modular
    inputs of nx_flashattn_scale.nx (``fa_seed``: ``((a i + b c) mod m - m/2) / m`` with
    (a, b, m) = (7, 3, 13) for Q, (5, 2, 11) for K, (3, 1, 9) for V), scale 1/sqrt(32).
``mha_b4_h16_n1k_d64``  B=4, H=16, N=1024, d=64, bf16, non-causal, N(0,1) inputs.
``causal_b8_h32_n4k_d128``  B=8, H=32, N=4096, d=128, bf16, causal, N(0,1) inputs.
``gqa_b1_h32kv8_n16k_d128``  B=1, Hq=32, Hkv=8, N=16384, d=128, bf16, causal; K, V are
    N(0,1) and Q is N(0,1)*8 (large logits, so the running maximum keeps moving).
``local_b2_h16_n32k_d128_w4k_cap50``  B=2, H=16, N=32768, d=128, bf16, causal sliding
    window of 4096 keys, logit soft-cap 50, N(0,1) inputs.

Softmax workloads (``SOFTMAX_WORKLOADS``): 4096 rows of 32000 logits and 1024 rows of
262144 logits, fp32 N(0,1) * 4, top-K with K = 5 (vocabulary-sized rows; the page gives
no sizes).

Further workloads (``EXTRA_WORKLOADS``) for the general entry point: the local workload
with 4 attention sinks ("Module 16", section 16.6); a chunk of 1024 new queries against
a 16384-key cache (the queries are the last 1024 positions, causal); and one decoding
step (one query row per head) against a 16384-key cache, grouped-query heads.

Random inputs are drawn on the CPU with ``torch.Generator().manual_seed(seed)`` as fp32
N(0,1), optionally multiplied by a constant in fp32, then rounded to bf16 (round to
nearest even), so the oracle and the GPU see bit-identical values.  Seeds are
1000 * workload_number + {0, 1, 2} for Q, K, V.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: str  # "float32" or "bfloat16"
    causal: bool
    window: int
    softcap: float
    q_mult: float = 1.0
    modular: bool = False
    nq: int = 0       # query rows per head when they differ from the N key rows (0: N)
    n_sink: int = 0   # attention sinks beside the window

    @property
    def Nq(self) -> int:
        return self.nq if self.nq > 0 else self.N

    @property
    def scale(self) -> float:
        """1/sqrt(d) rounded to fp32 (the value the library receives)."""
        return float(np.float32(1.0) / np.sqrt(np.float32(self.d)))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def seeds(self):
        base = 1000 * self.number
        return base, base + 1, base + 2

    def describe(self) -> dict:
        d = {"workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv, "N": self.N,
             "d": self.d, "dtype": self.dtype, "causal": self.causal, "window": self.window,
             "softcap": self.softcap, "q_mult": self.q_mult}
        if self.nq > 0:
            d["Nq"] = self.nq
        if self.n_sink > 0:
            d["n_sink"] = self.n_sink
        return d


WORKLOADS = {
    w.name: w
    for w in [
        Workload("modular_n64_d32", 1, 1, 1, 1, 64, 32, "float32", False, 0, 0.0, modular=True),
        Workload("mha_b4_h16_n1k_d64", 2, 4, 16, 16, 1024, 64, "bfloat16", False, 0, 0.0),
        Workload("causal_b8_h32_n4k_d128", 3, 8, 32, 32, 4096, 128, "bfloat16", True, 0, 0.0),
        Workload("gqa_b1_h32kv8_n16k_d128", 4, 1, 32, 8, 16384, 128, "bfloat16", True, 0, 0.0, q_mult=8.0),
        Workload("local_b2_h16_n32k_d128_w4k_cap50", 5, 2, 16, 16, 32768, 128, "bfloat16", True, 4096, 50.0),
    ]
}
EXTRA_WORKLOADS = {
    w.name: w
    for w in [
        Workload("sink4_b2_h16_n32k_d128_w4k_cap50", 6, 2, 16, 16, 32768, 128, "bfloat16", True, 4096, 50.0,
                 n_sink=4),
        Workload("chunk_b4_h32kv8_q1k_k16k_d128", 7, 4, 32, 8, 16384, 128, "bfloat16", True, 0, 0.0, nq=1024),
        Workload("decode_b32_h32kv8_q1_k16k_d128", 8, 32, 32, 8, 16384, 128, "bfloat16", True, 0, 0.0, nq=1),
    ]
}
ALL_WORKLOADS = {**WORKLOADS, **EXTRA_WORKLOADS}
BY_NUMBER = {w.number: w for w in WORKLOADS.values()}
HEADLINE = "causal_b8_h32_n4k_d128"


@dataclasses.dataclass(frozen=True)
class SoftmaxWorkload:
    """Rows of logits for the stand-alone softmax / softmax + top-K: fp32 N(0,1) * scale."""
    name: str
    rows: int
    V: int
    k: int
    scale: float = 4.0
    seed: int = 9000

    def describe(self) -> dict:
        return {"workload": self.name, "rows": self.rows, "V": self.V, "k": self.k, "dtype": "float32",
                "values": f"N(0,1) * {self.scale}"}


SOFTMAX_WORKLOADS = {
    w.name: w
    for w in [
        SoftmaxWorkload("softmax_r4k_v32k", 4096, 32000, 5),
        SoftmaxWorkload("softmax_r1k_v256k", 1024, 262144, 5, seed=9100),
    ]
}


def make_logits(w: SoftmaxWorkload, seed=None) -> torch.Tensor:
    """[rows, V] fp32 CPU logits for a softmax workload."""
    return _randn((w.rows, w.V), w.seed if seed is None else seed, w.scale, torch.float32)


def modular_matrix(n: int, d: int, a: int, b: int, m: int) -> np.ndarray:
    """nx_flashattn_scale.nx ``fa_seed``: x = (a i + b c) mod m, value (x - m/2) / m with
    integer m/2, converted to fp32 and divided in fp32 (IEEE, correctly rounded)."""
    i = np.arange(n, dtype=np.int64)[:, None]
    c = np.arange(d, dtype=np.int64)[None, :]
    x = (a * i + b * c) % m
    return (x - m // 2).astype(np.float32) / np.float32(m)


def _randn(shape, seed: int, mult: float, dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if mult != 1.0:
        t = t * torch.tensor(mult, dtype=torch.float32)
    return t.to(dtype)


def make_inputs(w: Workload, seeds=None):
    """(q, k, v) CPU tensors for workload ``w``: q [B,Hq,Nq,d], k/v [B,Hkv,N,d]."""
    if w.modular:
        if (w.B, w.Hq, w.Hkv) != (1, 1, 1):
            raise ValueError("modular inputs are defined for one head")
        q = torch.from_numpy(modular_matrix(w.N, w.d, 7, 3, 13)).reshape(1, 1, w.N, w.d)
        k = torch.from_numpy(modular_matrix(w.N, w.d, 5, 2, 11)).reshape(1, 1, w.N, w.d)
        v = torch.from_numpy(modular_matrix(w.N, w.d, 3, 1, 9)).reshape(1, 1, w.N, w.d)
        dt = torch.float32 if w.dtype == "float32" else torch.bfloat16
        return q.to(dt), k.to(dt), v.to(dt)
    dt = torch.bfloat16 if w.dtype == "bfloat16" else torch.float32
    sq, sk, sv = seeds if seeds is not None else w.seeds()
    q = _randn((w.B, w.Hq, w.Nq, w.d), sq, w.q_mult, dt)
    k = _randn((w.B, w.Hkv, w.N, w.d), sk, 1.0, dt)
    v = _randn((w.B, w.Hkv, w.N, w.d), sv, 1.0, dt)
    return q, k, v


def random_inputs(B, Hq, Hkv, N, d, dtype="bfloat16", seed=0, q_mult=1.0):
    """(q, k, v) for an ad-hoc shape (tests)."""
    w = Workload("adhoc", 0, B, Hq, Hkv, N, d, dtype, False, 0, 0.0, q_mult=q_mult)
    return make_inputs(w, seeds=(seed, seed + 1, seed + 2))


def random_cross_inputs(B, Hq, Hkv, Nq, Nk, d, dtype="bfloat16", seed=0, q_mult=1.0):
    """(q, k, v) with Nq query rows and Nk key rows per head (tests): q [B,Hq,Nq,d] from
    ``seed``, k and v [B,Hkv,Nk,d] from ``seed + 1`` and ``seed + 2``."""
    dt = torch.bfloat16 if dtype == "bfloat16" else torch.float32
    return (_randn((B, Hq, Nq, d), seed, q_mult, dt), _randn((B, Hkv, Nk, d), seed + 1, 1.0, dt),
            _randn((B, Hkv, Nk, d), seed + 2, 1.0, dt))


def sample_rows(w: Workload, per_head_rows, heads=None):
    """Flat row indices (b*Hq + hq)*Nq + i for the given query rows of the given heads
    (all heads by default)."""
    heads = range(w.B * w.Hq) if heads is None else heads
    rows = sorted(set(int(i) for i in per_head_rows if 0 <= int(i) < w.Nq))
    return np.array([bh * w.Nq + i for bh in heads for i in rows], dtype=np.int64)


def standard_row_sample(N: int, head: int = 256, tail: int = 256, stride: int = 61):
    """Query rows 0..head-1, the last ``tail`` rows and every ``stride``-th row."""
    s = set(range(min(head, N))) | set(range(max(0, N - tail), N)) | set(range(0, N, stride))
    return sorted(s)


__all__ = ["SoftmaxWorkload", "SOFTMAX_WORKLOADS", "make_logits", "Workload", "WORKLOADS", "EXTRA_WORKLOADS", "ALL_WORKLOADS", "BY_NUMBER", "HEADLINE", "make_inputs", "random_inputs", "random_cross_inputs",
           "modular_matrix", "sample_rows", "standard_row_sample"]

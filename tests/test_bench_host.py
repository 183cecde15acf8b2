"""Host-side arithmetic of the benchmark (no GPU): the FLOP and byte counts it divides by."""
import numpy as np

import bench
import oracle
import workloads
from tests.pin_suite import _kept_keys


def test_kept_keys_per_row_matches_brute_force():
    """4 d FLOPs per kept pair: the per-row key counts of the general workloads equal the
    key sets built from the mask's words (queries at the last Nq positions, window,
    sinks, causal)."""
    for (N, nq, W, S, causal) in [(50, 0, 7, 3, True), (50, 10, 7, 3, True), (40, 55, 5, 2, True),
                                  (30, 0, 0, 0, False), (30, 12, 0, 0, False), (64, 0, 1, 4, True),
                                  (64, 0, 10, 30, True), (300, 1, 0, 0, True)]:
        w = workloads.Workload("t", 0, 1, 1, 1, N, 8, "bfloat16", causal, W, 0.0, nq=nq, n_sink=S)
        got = bench.kept_keys_per_row(w, np.arange(w.Nq))
        want = [len(_kept_keys(i + N - w.Nq, N, causal, W, S)) for i in range(w.Nq)]
        assert list(got) == want, (N, nq, W, S)


def test_closed_flops_follow_the_convention():
    for n in (2, 3, 4, 5):
        w = workloads.BY_NUMBER[n]
        assert bench.closed_flops(w) == oracle.flops(w.B, w.Hq, w.N, w.d, w.causal, w.window, convention="closed")
    # the general workloads count kept pairs exactly
    w = workloads.EXTRA_WORKLOADS["decode_b32_h32kv8_q1_k16k_d128"]
    assert bench.closed_flops(w) == 4.0 * w.d * w.B * w.Hq * w.N
    w = workloads.EXTRA_WORKLOADS["chunk_b4_h32kv8_q1k_k16k_d128"]
    pairs = w.Nq * (w.N - w.Nq) + w.Nq * (w.Nq + 1) // 2
    assert bench.closed_flops(w) == 4.0 * w.d * w.B * w.Hq * pairs


def test_softmax_bytes():
    sw = workloads.SOFTMAX_WORKLOADS["softmax_r4k_v32k"]
    assert bench.softmax_bytes(sw, "softmax") == sw.rows * sw.V * 8 + sw.rows * 4
    assert bench.softmax_bytes(sw, "softmax_topk") == sw.rows * sw.V * 4 + sw.rows * sw.k * 8 + sw.rows * 4


def test_job_throughput_is_the_whole_job_over_the_slowest_rank():
    assert bench.job_tflops(4, 1e12, 10, 1000.0) == 4 * 1e12 * 10 / 1.0 / 1e12


def test_l2_flush_decision_looks_at_k_and_v():
    """Inputs larger than L2 in total but with K + V inside it (grouped-query attention)
    still get an L2 flush before every step; the headline workload does not need one."""
    import torch

    def meta(w):
        mk = lambda h, n: torch.empty((w.B, h, n, w.d), dtype=torch.bfloat16, device="meta")  # noqa: E731
        return mk(w.Hq, w.Nq), mk(w.Hkv, w.N), mk(w.Hkv, w.N)

    assert not bench.l2_flush_needed(*meta(workloads.BY_NUMBER[3]))
    assert bench.l2_flush_needed(*meta(workloads.BY_NUMBER[4]))   # K + V = 64 MiB
    assert bench.l2_flush_needed(*meta(workloads.BY_NUMBER[2]))   # everything fits


def test_clock_sampler_keeps_only_samples_inside_the_timed_region():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = [(0.5, 1000.0, 1965.0, 300.0, set()), (1.0, 1965.0, 1965.0, 700.0, {"sw_power_cap"}),
                 (1.5, 1900.0, 1965.0, 800.0, set()), (3.0, 800.0, 1965.0, 200.0, {"hw_slowdown"})]
    s.proc = s.thread = None
    s.source = "test"
    s.power_limit_w = 1000.0
    import threading
    s._stop = threading.Event()
    s.t0, s.t1 = 0.9, 2.0
    c = s.stop()
    assert c["samples"] == 2 and c["sm_mhz"] == (1965.0 + 1900.0) / 2 and c["reasons"] == ["sw_power_cap"]
    assert c["sm_mhz_range"] == [1900.0, 1965.0] and c["power_limit_w"] == 1000.0

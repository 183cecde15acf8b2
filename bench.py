"""Attention-forward benchmark on B200: TFLOP/s and fraction of the dense BF16 peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one full attention forward of the workload (all of Q.K^T, masking, online
softmax, P.V and the O / LSE write-back: one launch of the bf16 tensor-core kernel)
over one batch of synthetic inputs already resident in HBM.  The headline workload is
the causal B=8, H=32, N=4096, d=128 bf16 configuration.  FLOPs follow the convention
4 B Hq N^2 d, halved for causal, 4 B Hq d (N W - W^2/2) for a causal window.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream; for N > 1 (torchrun,
one rank per GPU) every rank runs its own independent batch (weak scaling, no data-path
collective) and the maximum time over ranks is used.  The inputs (768 MiB for the
headline workload) are larger than the 126 MB L2, so no flush is needed between steps.

Printed (rank 0, one JSON line): metric, value (whole-job TFLOP/s), roofline of the
kernel against the measured peak, e2e (the same metric with pinned-host inputs copied
in and outputs copied back inside the timed region), the fp64 CPU oracle timed on a
bounded row sample (cpu_baseline), SM clocks sampled during the timed region, and the
number of kernel launches in the timed region.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), as the reference
arm of the comparison.

``--op softmax`` / ``--op softmax_topk`` time the stand-alone softmax (online normaliser)
and the fused softmax + top-K instead, on a softmax workload (default 4096 rows of 32000
fp32 logits); their metric is HBM bandwidth: bytes that must cross HBM (the row read once
and, for softmax, written once; K probabilities and indices for top-K) per second.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "attention fwd TFLOP/s on 1 B200 and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024  # B200 L2 (126 MB)
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
KERNEL_SOURCES = ["online_softmax_11_b200/csrc/fa_fwd_tc.cuh", "online_softmax_11_b200/csrc/sm100_ptx.cuh",
                  "online_softmax_11_b200/csrc/fa_api.cu"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    rec = d.get(workload)
    if not rec or rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def l2_flush_needed(q, k, v) -> bool:
    """Flush L2 before every step unless every input is re-read from HBM anyway.  The
    decision is taken on Q + K + V and, separately, on K + V: with grouped-query
    attention K and V can fit in L2 while Q does not, and K / V tiles left in L2 by one
    launch would then be read warm by the next."""
    nbytes = [t.numel() * t.element_size() for t in (q, k, v)]
    return sum(nbytes) < L2_BYTES or nbytes[1] + nbytes[2] < L2_BYTES


def kept_keys_per_row(w, i):
    """Keys each query row i (numpy array) keeps: positions p = i + N - Nq, keys up to p
    (causal), the window's most recent ones plus the sinks below it."""
    pos = i + (w.N - w.Nq)
    hi = np.minimum(pos, w.N - 1) if w.causal else np.full_like(i, w.N - 1)
    lo = np.maximum(0, pos - w.window + 1) if w.window > 0 else np.zeros_like(i)
    n = np.maximum(0, hi - lo + 1)
    if w.window > 0 and w.n_sink > 0:
        n = n + np.maximum(0, np.minimum(np.minimum(w.n_sink, lo), hi + 1))
    return n


def closed_flops(w) -> float:
    """The convention for the self-attention workloads; 4 d per kept pair for the
    general ones (different query and key lengths, sinks)."""
    if w.nq > 0 or w.n_sink > 0:
        return float(4.0 * w.d * w.B * w.Hq * kept_keys_per_row(w, np.arange(w.Nq, dtype=np.int64)).sum())
    if w.window > 0:
        return 4.0 * w.B * w.Hq * w.d * (w.N * w.window - w.window * w.window / 2.0)
    f = 4.0 * w.B * w.Hq * w.N * w.N * w.d
    return f / 2.0 if w.causal else f


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons sampled while the timed region runs.

    A background thread reads NVML every ``period_ms`` (read-only queries: current and
    maximum SM clock, power draw, active clock-event reasons, and once the enforced power
    limit); ``nvidia-smi -lms`` is the
    fallback when the NVML binding is missing.  Only samples taken between
    ``mark_start()`` and ``mark_end()`` (host times around the timed region, which ends
    with a device synchronisation) are reported.  The GPU is found by the UUID of the
    CUDA device, so a CUDA_VISIBLE_DEVICES remapping cannot point NVML at another GPU.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device, period_ms: float = 2.0):
        import threading
        self.samples = []  # (host time, sm MHz, max sm MHz, power W, set of reason names)
        self.t0 = self.t1 = None
        self.proc = None
        self.thread = None
        self.source = None
        self.power_limit_w = None  # enforced board power limit (read once, NVML only)
        self._stop = threading.Event()
        handle = self._nvml_handle(device)
        if handle is not None:
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, args=(handle, period_ms / 1e3), daemon=True)
            self.thread.start()
            return
        try:
            import torch
            index = device.index if isinstance(device, torch.device) and device.index is not None else 0
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "10"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    @staticmethod
    def _nvml_handle(device):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            uuid = str(getattr(props, "uuid", ""))
            if uuid:
                try:
                    return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
                except pynvml.NVMLError:
                    pass
            if os.environ.get("CUDA_VISIBLE_DEVICES") is None:
                return pynvml.nvmlDeviceGetHandleByIndex(torch.device(device).index or 0)
        except Exception:  # noqa: BLE001 - no NVML: fall back to nvidia-smi
            return None
        return None

    def _poll_nvml(self, handle, period_s):
        import pynvml
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        smax = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
        try:
            self.power_limit_w = pynvml.nvmlDeviceGetEnforcedPowerLimit(handle) / 1e3
        except pynvml.NVMLError:
            pass
        while not self._stop.is_set():
            t = time.perf_counter()
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                power = pynvml.nvmlDeviceGetPowerUsage(handle) / 1e3
            except pynvml.NVMLError:
                break
            self.samples.append((t, sm, smax, power, {n for n, b in bits.items() if mask & b}))
            time.sleep(period_s)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax, power = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            reasons = {n for n, val in zip(self.REASON_NAMES, parts[5:9]) if val.lower() == "active"}
            self.samples.append((time.perf_counter(), sm, smax, power, reasons))

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.source is None:
            return None
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:
            return None
        reasons = set()
        for s in inside:
            reasons |= s[4]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "sm_mhz_range": [min(s[1] for s in inside), max(s[1] for s in inside)],
                "power_w_median": statistics.median(s[3] for s in inside), "power_limit_w": self.power_limit_w,
                "samples": len(inside),
                "reasons": sorted(reasons), "source": self.source,
                "window_ms": (t1 - t0) * 1e3 if self.t0 is not None and self.t1 is not None else None}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample_rows(w, n_rows: int, offset: int = 0):
    """``n_rows`` flat row indices spread evenly over all heads and query positions (so the
    causal / window work per row averages like the full workload), rotated by
    ``offset``."""
    total = w.B * w.Hq * w.Nq
    stride = max(1, total // max(1, n_rows))
    start = (offset * 7919) % stride
    return np.arange(start, total, stride, dtype=np.int64)[:n_rows]


def rows_flops(w, rows) -> float:
    return float(4.0 * w.d * kept_keys_per_row(w, rows % w.Nq).sum())


def time_oracle(w, inputs, seconds: float, offset: int = 0):
    """Time the fp64 oracle on a row sample sized to take about ``seconds``.
    Returns (TFLOP/s, seconds, rows, threads)."""
    import oracle
    q, k, v = inputs
    threads = oracle.host_threads()
    probe = oracle_sample_rows(w, 64 * threads, offset)
    t0 = time.perf_counter()
    oracle.attention(q, k, v, scale=w.scale, causal=w.causal, window=w.window, n_sink=w.n_sink, softcap=w.softcap, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    n = int(max(threads, min(w.B * w.Hq * w.Nq, len(probe) * seconds / dt)))
    rows = oracle_sample_rows(w, n, offset)
    t0 = time.perf_counter()
    oracle.attention(q, k, v, scale=w.scale, causal=w.causal, window=w.window, n_sink=w.n_sink, softcap=w.softcap, rows=rows)
    dt = time.perf_counter() - t0
    return rows_flops(w, rows) / dt / 1e12, dt, len(rows), threads


# ----------------------------------------------------------------------------- distributed

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def emit(obj):
    print(json.dumps(obj), flush=True)


def rank_seeds(w, rank: int):
    """Seeds of rank `rank`'s own batch: every rank processes an independent batch of the
    workload (weak scaling, no data exchange)."""
    return tuple(s + 100 * rank for s in w.seeds())


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank time over all ranks (one all-reduce of one number)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world_size: int, flop_per_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world_size * flop_per_step * steps / (max_ms / 1e3) / 1e12


def reference_arm(args, w):
    """The fp64 CPU oracle as the reference implementation (rank 0 only)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    inputs = workloads.make_inputs(w)
    threads = oracle.host_threads()
    budget = float(args.reference_seconds) / max(1, args.steps + args.warmup)
    # per step: a row sample sized for `budget` seconds of oracle work
    probe = oracle_sample_rows(w, 32 * threads)
    t0 = time.perf_counter()
    oracle.attention(*inputs, scale=w.scale, causal=w.causal, window=w.window, n_sink=w.n_sink, softcap=w.softcap, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    n_rows = int(max(threads, len(probe) * budget / dt))
    total_flop = 0.0
    total_s = 0.0
    for step in range(args.warmup + args.steps):
        rows = oracle_sample_rows(w, n_rows, step)
        t0 = time.perf_counter()
        oracle.attention(*inputs, scale=w.scale, causal=w.causal, window=w.window, n_sink=w.n_sink, softcap=w.softcap, rows=rows)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            total_flop += rows_flops(w, rows)
            total_s += dt
    value = total_flop / total_s / 1e12
    sample = (f"{n_rows} query rows per step spread over all {w.B * w.Hq} heads and positions of "
              f"{w.name} (dense fp64 oracle; FLOPs counted as 4 d per unmasked pair)")
    emit({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, **{k: v for k, v in w.describe().items() if k != "workload"}},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })
    return 0


def gpu_arm(args, w):
    import torch
    import torch.distributed as dist

    import online_softmax_11_b200 as fa

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    fa.load()

    # each rank its own batch: seeds shifted by the rank (weak scaling, no data exchange)
    seeds = rank_seeds(w, rank)
    q_h, k_h, v_h = workloads.make_inputs(w, seeds=seeds)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    general = args.splits > 0 or w.nq > 0 or w.n_sink > 0
    workspace = None
    if general:
        # general entry point (split-KV, cross lengths, sinks); the workspace is
        # allocated once, outside the timed region
        ws_bytes = fa.splitkv_workspace_bytes(w.B, w.Hq, w.Nq, w.d, args.splits) if args.splits > 0 else 0
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        ws_ptr = workspace.data_ptr() if args.splits > 0 else None
        lib = fa.load()

        def launch(qq, kk, vv, oo, ll):
            rc = lib.fa_fwd_ext(qq.data_ptr(), kk.data_ptr(), vv.data_ptr(), oo.data_ptr(), ll.data_ptr(), w.B, w.Hq,
                                w.Hkv, w.Nq, w.N, w.d, w.scale, int(w.causal), w.window, w.n_sink, w.softcap,
                                args.splits, ws_ptr, ws_bytes, sh)
            if rc != 0:
                raise fa.FAError(rc, lib, "fa_fwd_ext")

        def step():
            launch(q, k, v, o, lse)
    else:
        def step():
            rc = fa.fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.Hq, w.Hkv,
                            w.N, w.d, w.scale, w.causal, w.window, w.softcap, sh, w.dtype)
            if rc != 0:
                raise fa.FAError(rc, fa.load(), "fa_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.check_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    sampler = ClockSampler(dev) if not args.no_clocks else None
    if sampler is not None:
        time.sleep(0.3)  # let the sampler start before the timed region
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    small = l2_flush_needed(q, k, v)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.mark_start()
    if not small:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        elapsed_ms = start.elapsed_time(end)
    else:
        # inputs that fit in L2: flush it (write a larger buffer) before every step and
        # time each step alone with its own events
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        elapsed_ms = 0.0
        for _ in range(args.steps):
            flush.zero_()
            start.record(stream)
            step()
            end.record(stream)
            end.synchronize()
            elapsed_ms += start.elapsed_time(end)
        del flush
    if sampler is not None:
        sampler.mark_end()
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    if fa.check_status() != 0:
        raise RuntimeError("device status word set during the timed region")

    max_ms = max_over_ranks(elapsed_ms, dev)
    flop_per_step = closed_flops(w)
    per_launch_ms = elapsed_ms / args.steps
    value = job_tflops(ws, flop_per_step, args.steps, max_ms)

    # ---- e2e: pinned host inputs -> device, forward, outputs -> pinned host, per step
    e2e = None
    if not args.no_e2e:
        # Every step copies its inputs from pinned host memory, runs the forward through
        # the public call and copies O and LSE back.  Steps are pipelined over three
        # streams with two buffer sets: step i's inputs go in while step i-1 computes and
        # step i-2's outputs come back (the two copy directions and the kernels overlap).
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        op = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lp = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        bufs = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(o),
                 torch.empty_like(lse)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            qd, kd, vd, od, ld = bufs[b]
            if used[b]:  # the buffers' previous step has finished computing / copying out
                s_in.wait_event(comp_done[b])
                stream.wait_event(out_done[b])
            with torch.cuda.stream(s_in):
                qd.copy_(qp, non_blocking=True)
                kd.copy_(kp, non_blocking=True)
                vd.copy_(vp, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if general:
                launch(qd, kd, vd, od, ld)
            else:
                fa.forward(qd, kd, vd, scale=w.scale, causal=w.causal, window=w.window, softcap=w.softcap, out=od,
                           lse=ld, stream=stream)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                op.copy_(od, non_blocking=True)
                lp.copy_(ld, non_blocking=True)
                out_done[b].record(s_out)
            used[b] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if ws > 1:
            dist.barrier()
        n_e2e = max(1, min(args.e2e_steps, args.steps))
        es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        es.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        s_out.wait_event(comp_done[(n_e2e - 1) % 2])
        ee.record(s_out)
        torch.cuda.synchronize(dev)
        te_ms = max_over_ranks(es.elapsed_time(ee), dev)
        h2d = (q.numel() * q.element_size() + k.numel() * k.element_size() + v.numel() * v.element_size())
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": job_tflops(ws, flop_per_step, n_e2e, te_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": te_ms / n_e2e, "pipelined": "copies in, kernel, copies out on three streams"}
        if fa.check_status() != 0:
            raise RuntimeError("device status word set during the end-to-end run")
        del qp, kp, vp, op, lp, bufs

    # ---- CPU baseline: the fp64 oracle on a bounded row sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tflops, secs, nrows, threads = time_oracle(w, (q_h, k_h, v_h), args.cpu_seconds)
        cpu = {"value": tflops, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{nrows} query rows spread evenly over all {w.B * w.Hq} heads and positions of "
                         f"{w.name}, {secs:.1f} s of fp64 work; FLOPs counted as 4 d per unmasked pair"}

    peaks, peaks_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_bw = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    if w.dtype == "float32":  # the fp32 CUDA-core path
        kernel = f"fa_fwd_f32_kernel<{(w.d + 31) // 32}>"
    elif (w.Hq // w.Hkv) * w.Nq <= 16:  # the group's query rows fit one 16-row block
        kernel = f"fa_decode_kernel<{w.d}>"
    else:
        kernel = (f"fa_fwd_tc_kernel<{w.d}, {'true' if args.splits > 0 else 'false'}, "
                  f"{'true' if (w.n_sink > 0 and w.window > 0) else 'false'}, "
                  f"{'true' if w.softcap > 0 else 'false'}>")
    # algorithmic bytes: Q, K, V read once, O and LSE written once
    alg_bytes = float(q.numel() * q.element_size() + k.numel() * k.element_size() + v.numel() * v.element_size()
                      + o.numel() * o.element_size() + lse.numel() * lse.element_size())
    if w.dtype == "float32":
        # plain FP32 FMA arithmetic: peak = SMs x 128 FP32 lanes x 2 flop x the SM clock
        # seen (1965 MHz when no sample was taken)
        sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
        peak_alu = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * 2 * sm_mhz * 1e6 / 1e12
        achieved = flop_per_step / (per_launch_ms / 1e3) / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak_alu, "unit": UNIT,
                    "frac": achieved / peak_alu, "traffic": None,
                    "peak_source": "SMs x 128 FP32 lanes x 2 flop x SM clock (derived, no tensor cores)",
                    "kernel": kernel, "algorithmic_flop_per_launch": flop_per_step,
                    "note": "n = 64, d = 32: one launch of a few microseconds, bound by launch latency"}
    elif flop_per_step / alg_bytes >= peak * 1e12 / (peak_bw * 1e9):
        achieved = flop_per_step / (per_launch_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                    "traffic": load_traffic(w.name), "peak_source": f"bf16_tflops (burst) of {peaks_src}",
                    "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                    "kernel": kernel, "algorithmic_flop_per_launch": flop_per_step}
    else:  # below the ridge point (one query row per head): bound by reading K and V
        achieved = alg_bytes / (per_launch_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak_bw, "unit": "GB/s",
                    "frac": achieved / peak_bw, "traffic": load_traffic(w.name),
                    "peak_source": f"hbm_gbs of {peaks_src}", "kernel": kernel,
                    "algorithmic_bytes_per_launch": alg_bytes}

    if rank == 0:
        cfg = {"workload": w.name, **{k: v for k, v in w.describe().items() if k != "workload"},
               "flop_convention": ("4 d per kept (query, key) pair" if (w.nq > 0 or w.n_sink > 0) else
                                   "4 B Hq N^2 d, /2 causal; 4 B Hq d (N W - W^2/2) with a window"),
               "l2": ("L2 flushed before every step (inputs, or K and V, smaller than L2); steps timed one by one"
                      if small else "inputs and K + V larger than L2 (no flush needed)"),
               "parallelism": f"replicas x{ws} (independent batches)"}
        if args.splits > 0:
            cfg["split_kv"] = args.splits
        emit({
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if w.dtype == "float32" else "bf16",
            "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": args.steps * (2 if args.splits > 0 else 1),
        })
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


SOFTMAX_METRIC = {"softmax": "stand-alone softmax GB/s (rows read and written once) on 1 B200",
                  "softmax_topk": "fused softmax + top-K GB/s (rows read once) on 1 B200"}


def softmax_bytes(sw, op: str) -> float:
    """Bytes that must cross HBM per step: x read once; y written (softmax) or K
    probabilities + K int32 indices (top-K); one fp32 LSE per row."""
    out = sw.rows * sw.V * 4 if op == "softmax" else sw.rows * sw.k * 8
    return float(sw.rows * sw.V * 4 + out + sw.rows * 4)


def softmax_oracle_time(sw, op: str, x, seconds: float, offset: int = 0):
    """The fp64 oracle on a bounded row sample: returns (GB/s of the same accounting,
    seconds, rows, threads=1: numpy on one core)."""
    from oracle import softmax as osm
    t0 = time.perf_counter()
    osm.softmax(x[:4]) if op == "softmax" else osm.softmax_topk(x[:4], sw.k)
    dt = max(time.perf_counter() - t0, 1e-4)
    n = int(max(1, min(sw.rows, 4 * seconds / dt)))
    start = (offset * 97) % max(1, sw.rows - n + 1)
    t0 = time.perf_counter()
    osm.softmax(x[start:start + n]) if op == "softmax" else osm.softmax_topk(x[start:start + n], sw.k)
    dt = time.perf_counter() - t0
    return softmax_bytes(sw, op) * n / sw.rows / dt / 1e9, dt, n


def softmax_arm(args, sw):
    """Time fa_softmax / fa_softmax_topk (ours) or the oracle (reference) on ``sw``."""
    import torch
    op = args.op
    ws, rank, local = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        x = workloads.make_logits(sw)
        total_b, total_s = 0.0, 0.0
        budget = float(args.reference_seconds) / max(1, args.steps + args.warmup)
        for step in range(args.warmup + args.steps):
            gbs, dt, n = softmax_oracle_time(sw, op, x, budget, step)
            if step >= args.warmup:
                total_b += gbs * dt
                total_s += dt
        value = total_b / total_s
        sample = f"{n} of {sw.rows} rows per step, numpy fp64 on one core"
        emit({"impl": "reference", "metric": SOFTMAX_METRIC[op], "value": value, "unit": "GB/s", "n_gpus": ws,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3,
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
              "config": sw.describe(),
              "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
              "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        return 0
    import torch.distributed as dist
    import online_softmax_11_b200 as fa
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    lib = fa.load()
    x_h = workloads.make_logits(sw, seed=sw.seed + 100 * rank)
    x = x_h.to(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    y = torch.empty_like(x)
    probs = torch.empty((sw.rows, sw.k), dtype=torch.float32, device=dev)
    idx = torch.empty((sw.rows, sw.k), dtype=torch.int32, device=dev)
    lse = torch.empty(sw.rows, dtype=torch.float32, device=dev)

    def step(xx):
        if op == "softmax":
            rc = lib.fa_softmax(xx.data_ptr(), y.data_ptr(), lse.data_ptr(), sw.rows, sw.V, sh)
        else:
            rc = lib.fa_softmax_topk(xx.data_ptr(), probs.data_ptr(), idx.data_ptr(), lse.data_ptr(), sw.rows, sw.V,
                                     sw.k, sh)
        if rc != 0:
            raise fa.FAError(rc, lib, "fa_" + op)

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev) if not args.no_clocks else None
    if sampler is not None:
        time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.mark_start()
    ev0.record(stream)
    for _ in range(args.steps):
        step(x)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.mark_end()
    if ws > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    clocks = sampler.stop() if sampler is not None else None
    max_ms = max_over_ranks(ms, dev)
    nbytes = softmax_bytes(sw, op)
    value = ws * nbytes * args.steps / (max_ms / 1e3) / 1e9
    per_launch = ms / args.steps

    e2e = None
    if not args.no_e2e:
        # pinned input copied in, the kernel, outputs copied back, every step; steps are
        # pipelined over three streams with two buffer sets (as in the attention arm)
        xp = x_h.pin_memory()
        outp = torch.empty(y.shape if op == "softmax" else probs.shape, dtype=torch.float32, pin_memory=True)
        ip = torch.empty(idx.shape, dtype=torch.int32, pin_memory=True)
        bufs = [(torch.empty_like(x), torch.empty_like(y) if op == "softmax" else None, torch.empty_like(probs),
                 torch.empty_like(idx), torch.empty_like(lse)) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            xd, yd, pd, idd, ld = bufs[b]
            if used[b]:
                s_in.wait_event(comp_done[b])
                stream.wait_event(out_done[b])
            with torch.cuda.stream(s_in):
                xd.copy_(xp, non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if op == "softmax":
                rc = lib.fa_softmax(xd.data_ptr(), yd.data_ptr(), ld.data_ptr(), sw.rows, sw.V, sh)
            else:
                rc = lib.fa_softmax_topk(xd.data_ptr(), pd.data_ptr(), idd.data_ptr(), ld.data_ptr(), sw.rows, sw.V,
                                         sw.k, sh)
            if rc != 0:
                raise fa.FAError(rc, lib, "fa_" + op)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                if op == "softmax":
                    outp.copy_(yd, non_blocking=True)
                else:
                    outp.copy_(pd, non_blocking=True)
                    ip.copy_(idd, non_blocking=True)
                out_done[b].record(s_out)
            used[b] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if ws > 1:
            dist.barrier()
        n_e2e = max(1, min(args.e2e_steps, args.steps))
        es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        es.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        ee.record(s_out)
        torch.cuda.synchronize(dev)
        te = max_over_ranks(es.elapsed_time(ee), dev)
        d2h = y.numel() * 4 if op == "softmax" else probs.numel() * 4 + idx.numel() * 4
        e2e = {"value": ws * nbytes * n_e2e / (te / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": x.numel() * 4,
               "d2h_bytes_per_step": d2h, "steps": n_e2e, "ms_per_step": te / n_e2e,
               "pipelined": "copies in, kernel, copies out on three streams"}
        del xp, outp, ip, bufs

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        gbs, secs, n = softmax_oracle_time(sw, op, x_h, min(args.cpu_seconds, 10.0))
        cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} of {sw.rows} rows, numpy fp64 on one core, {secs:.1f} s"}
    peaks, src = load_peaks()
    peak_bw = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = nbytes / (per_launch / 1e3) / 1e9
    kmax = next(c for c in (4, 8, 16, 32) if sw.k <= c)
    kernel = ("softmax_online_kernel" if op == "softmax" else
              f"softmax_topk_kernel<{kmax}, {512 if sw.V <= 131072 else 1024}>")
    if rank == 0:
        emit({"metric": SOFTMAX_METRIC[op], "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
              "config": {**sw.describe(), "l2": "inputs larger than L2 (no flush needed)",
                         "parallelism": f"replicas x{ws} (independent batches)"},
              "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak_bw, "unit": "GB/s",
                           "frac": achieved / peak_bw, "traffic": None, "peak_source": f"hbm_gbs of {src}",
                           "kernel": kernel, "algorithmic_bytes_per_launch": nbytes},
              "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": args.steps})
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["attention", "softmax", "softmax_topk"], default="attention")
    ap.add_argument("--workload", default=None,
                    choices=sorted(workloads.ALL_WORKLOADS) + sorted(workloads.SOFTMAX_WORKLOADS))
    ap.add_argument("--batch", type=int, default=None, help="override B (profiling on a smaller case)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="total oracle time budget of the reference arm")
    ap.add_argument("--splits", type=int, default=0,
                    help="time the split-KV path with this many key chunks (0: the plain forward)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    args = ap.parse_args(argv)
    ws, _, _ = dist_env()
    if args.gpus != ws:
        ap.error(f"--gpus {args.gpus} needs one process per GPU: launch with torchrun --nproc-per-node "
                 f"{args.gpus} (WORLD_SIZE is {ws})")
    if args.op != "attention":
        name = args.workload or "softmax_r4k_v32k"
        if name not in workloads.SOFTMAX_WORKLOADS:
            ap.error(f"--op {args.op} takes a softmax workload: {sorted(workloads.SOFTMAX_WORKLOADS)}")
        return softmax_arm(args, workloads.SOFTMAX_WORKLOADS[name])
    if args.workload in workloads.SOFTMAX_WORKLOADS:
        ap.error("softmax workloads need --op softmax or --op softmax_topk")
    w = workloads.ALL_WORKLOADS[args.workload or workloads.HEADLINE]
    if args.batch is not None:
        w = w.with_(B=args.batch)
    if args.impl == "reference":
        return reference_arm(args, w)
    return gpu_arm(args, w)


if __name__ == "__main__":
    sys.exit(main())

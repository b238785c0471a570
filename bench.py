"""Benchmark of the quantized Delta-rule decode step (one JSON line on stdout).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

A step is one decode step (unpack, dequant + decay, delta rule, readout,
requant + repack in place) over every page of the workload's batch.  The
default workload is the largest: the DAMP-style state (16 FP16 key rows, 112
INT8 rows with stochastic rounding), 4,096 requests x 32 heads; the other
workloads (uniform INT8, 256 x 32; STEPQuant 6-bit, 1,024 x 32; STEPQuant
4-bit with the KDA gate, 2,048 x 32) are measured in the same run, each with
its own roofline, clock record and CPU baseline.  The K timed steps run as
five back-to-back repetitions whose mean and best are reported.

Inputs for all steps are generated on the device before timing; every step
streams the whole state and its inputs (0.29-5.2 GB moved per step, the
state alone 138 MB-2.5 GB) through the 126 MB L2, so no flush is needed
between steps.  Under torchrun each rank runs its own batch (weak
scaling, no collective on the data path); time is the max over ranks.

The same line also reports the per-window path (stq_window_step, windows
of 4, 8 and 16 steps) and the prefill (stq_prefill) on the default workload,
each with its own roofline.

--impl reference times the CPU oracle (single thread, as written) on a
bounded sample of the same workload; only rank 0 runs it.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_recurrent_delta_b200 import ranks as R  # noqa: E402
from linear_attention_recurrent_delta_b200 import workloads as W  # noqa: E402

METRIC = "decode state-update head-steps/s"
UNIT = "head-steps/s"


def algorithmic_bytes_per_page(spec):
    """Bytes one page-step must move: codes + r read and written, c read,
    q, k, v, the gate(s) and beta read, o written (the precision map is
    L2-resident and not counted)."""
    code = sum(rows * 128 * (16 if kind == "fp16" else bits) // 8 for rows, kind, bits in spec["groups"])
    n_int = sum(rows for rows, kind, _ in spec["groups"] if kind == "int")
    b = 2 * code + 2 * 4 * n_int + (512 if spec["col_scales"] else 0)
    b += 3 * 512 + (512 if spec["gate_vector"] else 4) + 4 + 512
    return b


def window_bytes_per_page(spec, window):
    """Bytes one page-step of the per-window path must move, averaged over a
    window of ``window`` steps (the last one commits).  Every step reads the
    page (codes, r, c), q, k, v, the gate(s), beta and (t > 0) the buffer's P,
    K[0..t-1], D[0..t-1]; it writes o and, unless it commits, P', K[0..t] and
    D[t]; the committing step writes the requantized codes and r instead."""
    code = sum(rows * 128 * (16 if kind == "fp16" else bits) // 8 for rows, kind, bits in spec["groups"])
    n_int = sum(rows for rows, kind, _ in spec["groups"] if kind == "int")
    page_read = code + 4 * n_int + (512 if spec["col_scales"] else 0)
    inputs = 3 * 512 + (512 if spec["gate_vector"] else 4) + 4
    total = 0
    for t in range(window):
        read = page_read + inputs + (512 + 1024 * t if t > 0 else 0)
        write = 512 + (code + 4 * n_int if t == window - 1 else 512 + 512 * (t + 1) + 512)
        total += read + write
    return total / window


DECODE_SOURCES = ("stq_decode.cu", "stq_device.cuh", "stq_internal.h", "stq_slices.cuh")


def kernel_source_hash(names=DECODE_SOURCES):
    """Hash of the sources the decode kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_recurrent_delta_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# The B200's nominal HBM3e bandwidth (HGX figure, 7.7 TB/s; 8 TB/s in DGX
# material).  The roofline divides by the measured copy bandwidth; the
# fraction of the rounder nominal 8 TB/s figure is reported beside it.
NOMINAL_HBM_GBS = 8000.0


def ncu_traffic(workload_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
    except (OSError, ValueError):
        return None
    e = d.get(workload_name)
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def hbm_roofline(spec, pages, ms_per_step, workload_name):
    """The decode kernel's roofline object: algorithmic bytes per page x pages
    per launch / the launch's average CUDA-event time, against the measured
    copy bandwidth (and, beside it, the nominal 8 TB/s)."""
    bpp = algorithmic_bytes_per_page(spec)
    achieved = bpp * pages / (ms_per_step / 1000.0) / 1e9
    peak, peak_kind = measured_peak()
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": ncu_traffic(workload_name), "peak_kind": peak_kind,
            "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "bytes_per_head_step": bpp, "pages_per_launch": pages, "kernel": "stq::decode_kernel"}


class ClockSampler:
    """SM clock, its maximum and the clock-event (throttle) reasons of one GPU,
    read through NVML every millisecond from a thread, so that even a timed
    region of a few tens of milliseconds holds samples; nvidia-smi at 200 ms
    if NVML cannot be loaded.  Read-only: no setting of the GPU is changed."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.rows = []          # (monotonic time, sm MHz, max MHz, [reason names])
        self.proc = None
        self.stop_ev = threading.Event()
        self.thread = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.cuda_index)
            bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            nv = None
        if nv is not None:
            self.source = "nvml, 1 ms"

            def poll():
                while not self.stop_ev.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h) \
                            if hasattr(nv, "nvmlDeviceGetCurrentClocksEventReasons") \
                            else nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                        self.rows.append((time.monotonic(), float(sm), float(mx),
                                          [n for n, b in self.REASONS if bits & b]))
                    except Exception:
                        pass
                    time.sleep(0.001)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi, 200 ms"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def read():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[0] == str(self.cuda_index):
                    try:
                        self.rows.append((time.monotonic(), float(parts[1]), float(parts[2]),
                                          [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]))
                    except ValueError:
                        pass
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def stop(self, t0=None, t1=None):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        self.stop_ev.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.thread.join(timeout=5)
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        inside = True
        if not rows:   # region shorter than one sampling period: keep the nearest samples
            rows = self.rows[-2:]
            inside = False
        sm = [r[1] for r in rows]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in rows) if rows else None,
                "reasons": sorted({n for r in rows for n in r[3]}), "samples": len(rows),
                "inside_timed_region": inside, "source": self.source}


def dist_setup(n_gpus):
    world, rank, local = R.rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        R.init("nccl", timeout_s=120, device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    R.barrier(world)


def max_over_ranks(x, world):
    return R.max_over_ranks(x, world, device="cuda")


def split_reps(steps, reps=5):
    """K timed steps as `reps` back-to-back repetitions (fewer if K < reps):
    the repetition sizes, summing to K."""
    n = max(1, min(reps, steps))
    return [steps // n + (1 if i < steps % n else 0) for i in range(n)]


def run_gpu(w, steps, warmup, rank, world, sample_clocks=True, e2e_steps=16, paged=False):
    """Decode steps of workload w: `warmup` untimed steps, then exactly `steps`
    timed steps as five repetitions, each bracketed by its own CUDA events on
    the launching stream (barrier + synchronize around the whole region).
    Returns the total and per-repetition device times (max over ranks), the
    clock record of the region and, if e2e_steps, the end-to-end time of the
    host-buffer entry point."""
    from linear_attention_recurrent_delta_b200 import binding as B
    dev = torch.device("cuda", torch.cuda.current_device())
    wr = R.rank_workload(w, rank)   # this rank's own requests: no exchange on the data path
    qs = B.QuantizedState(wr.format, wr.batch, wr.heads, device=dev)
    S = W.initial_state(wr, device=dev)
    qs.calibrate_and_quantize(S)
    del S
    torch.cuda.synchronize()
    n_in = min(wr.steps, max(steps, warmup, 1))
    inputs = [W.step_inputs(wr, t, device=dev) for t in range(n_in)]
    o = torch.empty(wr.batch, wr.heads, 128, device=dev)
    seed = W.sr_seed(wr)
    stream = torch.cuda.current_stream()

    # paged: every request through the slot table, in a random order of slots
    table = torch.randperm(wr.batch, generator=torch.Generator().manual_seed(wr.seed)).to(
        device=dev, dtype=torch.int32) if paged else None

    def step(t):
        x = inputs[t % n_in]
        if paged:
            B.stq_decode_step_slots(qs.state, table, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o, seed, t,
                                    stream)
        else:
            B.stq_decode_step(qs.state, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o, seed, t, stream)

    for t in range(warmup):
        step(t)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device()) if sample_clocks else None
    if clocks:
        clocks.start()
        time.sleep(0.05)
    sizes = split_reps(steps)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(sizes) + 1)]
    h0 = time.monotonic()
    evs[0].record(stream)
    t = warmup
    for i, n in enumerate(sizes):
        for _ in range(n):
            step(t)
            t += 1
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    barrier(world)
    torch.cuda.synchronize()
    rep_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(sizes))]
    ms = evs[0].elapsed_time(evs[-1])
    clk = clocks.stop(h0, h1) if clocks else None
    status = B.stq_device_status(qs.state)
    if status != B.STQ_OK:
        raise RuntimeError("device status: %s" % B.stq_status_string(status))
    ms_max = max_over_ranks(ms, world)
    rep_ms = [max_over_ranks(x, world) for x in rep_ms]
    per_step = [m / n for m, n in zip(rep_ms, sizes)]
    reps = {"n": len(sizes), "steps_each": sizes, "ms_per_step_mean": statistics.mean(per_step),
            "ms_per_step_best": min(per_step), "ms_per_step_worst": max(per_step)}

    if e2e_steps == 0:
        del qs, inputs
        torch.cuda.empty_cache()
        return {"ms": ms_max, "clocks": clk, "reps": reps}
    # end to end through the pipelined host-buffer entry point: every step's
    # H2D of its inputs from pinned memory, the step and the D2H of its o,
    # all inside the timed region; the copies of neighbouring steps overlap
    # the step (stq_decode_steps_host).  8 distinct steps of inputs, passed
    # e2e_steps / 8 times (a call's copies start after the work before it on
    # the stream, the previous call's last copy-out included, so the
    # pipeline refills once per call).
    chunk = 8
    host = {k: torch.stack([x[k] for x in [W.step_inputs(wr, t) for t in range(chunk)]]).contiguous().pin_memory()
            for k in inputs[0]}
    del inputs
    o_host = torch.empty(chunk, wr.batch, wr.heads, 128).pin_memory()
    io_bytes = 2 * B.stq_decode_io_bytes(qs.state)
    io_buf = torch.empty(io_bytes + 256, dtype=torch.uint8, device=dev)
    off = (-io_buf.data_ptr()) % 256
    io = io_buf[off:off + io_bytes]
    h2d = sum(v[0].numel() * v.element_size() for v in host.values())
    d2h = o_host[0].numel() * o_host.element_size()
    n_calls = max(1, e2e_steps // chunk)
    B.stq_decode_steps_host(qs.state, host["q"], host["k"], host["v"], host["alpha"], host["beta"], o_host, io,
                            seed, 0, stream)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for r in range(n_calls):
        B.stq_decode_steps_host(qs.state, host["q"], host["k"], host["v"], host["alpha"], host["beta"], o_host, io,
                                seed, r * chunk, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_steps = n_calls * chunk
    barrier(world)
    # the same inputs' host-to-device copies alone, from the same pinned
    # buffers: the PCIe bound of the end-to-end rate
    del io_buf
    dst = {k: torch.empty(v[0].shape, dtype=v.dtype, device=dev) for k, v in host.items()}
    for k in host:
        dst[k].copy_(host[k][0], non_blocking=True)
    torch.cuda.synchronize()
    n_copy = 8
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for r in range(n_copy):
        for k in host:
            dst[k].copy_(host[k][r % chunk], non_blocking=True)
    c1.record(stream)
    torch.cuda.synchronize()
    h2d_ms = max_over_ranks(c0.elapsed_time(c1), world) / n_copy
    # and with each step's o copied back at the same time on a second stream
    # (both directions of the link busy, as in the pipelined steps)
    o_dev = torch.empty(o_host[0].shape, dtype=o_host.dtype, device=dev)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    torch.cuda.synchronize()
    c0.record(stream)
    side.wait_event(c0)
    for r in range(n_copy):
        for k in host:
            dst[k].copy_(host[k][r % chunk], non_blocking=True)
        with torch.cuda.stream(side):
            o_host[r % chunk].copy_(o_dev, non_blocking=True)
    stream.wait_stream(side)
    c1.record(stream)
    torch.cuda.synchronize()
    both_ms = max_over_ranks(c0.elapsed_time(c1), world) / n_copy
    barrier(world)
    del qs, host, dst, o_dev
    torch.cuda.empty_cache()
    return {"ms": ms_max, "clocks": clk, "reps": reps, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h,
            "e2e_steps": e2e_steps, "h2d_copy_ms": h2d_ms, "copies_ms": both_ms}


def run_window(w, window, steps, warmup, rank, world):
    """Per-window decode steps (stq_window_step), t cycling 0 .. window-1 with
    a commit at window-1; steps and warmup are rounded up to whole windows.
    Returns the device time of the timed steps (max over ranks) and the mean
    time of each window position from a second, per-launch-timed pass."""
    from linear_attention_recurrent_delta_b200 import binding as B
    dev = torch.device("cuda", torch.cuda.current_device())
    wr = R.rank_workload(w, rank)
    qs = B.QuantizedState(wr.format, wr.batch, wr.heads, device=dev)
    S = W.initial_state(wr, device=dev)
    qs.calibrate_and_quantize(S)
    del S
    nbuf = B.stq_window_buffer_bytes(qs.state, window)
    buf_raw = torch.empty(nbuf + 256, dtype=torch.uint8, device=dev)
    off = (-buf_raw.data_ptr()) % 256
    buf = buf_raw[off:off + nbuf]
    n_in = min(wr.steps, 16)
    inputs = [W.step_inputs(wr, t, device=dev) for t in range(n_in)]
    o = torch.empty(wr.batch, wr.heads, 128, device=dev)
    seed = W.sr_seed(wr)
    stream = torch.cuda.current_stream()
    steps = -(-steps // window) * window
    warmup = -(-max(warmup, 3) // window) * window

    def step(i):
        x = inputs[i % n_in]
        t = i % window
        B.stq_window_step(qs.state, buf, window, t, t == window - 1, x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                          o, seed, i, stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        step(warmup + i)
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    # per position: an event pair around each launch (this pass only)
    reps = max(1, min(50, steps // window))
    per_t = [0.0] * window
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps * window)]
    for i in range(reps * window):
        evs[i][0].record(stream)
        step(warmup + steps + i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    for i in range(reps * window):
        per_t[i % window] += evs[i][0].elapsed_time(evs[i][1]) / reps
    status = B.stq_device_status(qs.state)
    if status != B.STQ_OK:
        raise RuntimeError("device status: %s" % B.stq_status_string(status))
    barrier(world)
    del qs, inputs, buf_raw
    torch.cuda.empty_cache()
    return {"ms": ms, "steps": steps, "per_t_ms": per_t}


def tf32_peak():
    """Dense tf32 tensor-core peak: the measured bf16 GEMM rate (burst) x the
    nominal tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s dense)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            bf16 = float(json.load(fh)["bf16_tflops"])
        return bf16 * 1.1 / 2.25, "measured bf16 x nominal tf32/bf16 ratio"
    except (OSError, KeyError, ValueError):
        return 1590.0 * 1.1 / 2.25, "fallback bf16 x nominal tf32/bf16 ratio"


# FP32 peak of the CUDA cores for the prefill's plain arithmetic: 148 SMs x
# 128 FP32 lanes x 2 flops per fma x 1.965 GHz (clocks.max.sm).
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def prefill_flops_per_head_token():
    """Per page and token: the decay (one multiply per element; the first
    token's dequantization instead), the prediction, the update and the
    readout (one fma each per element)."""
    return 128 * 128 * (1 + 2 + 2 + 2)


def chunked_flops_per_head_token():
    """Tensor-core work per page and token of the chunkwise prefill, counted
    as the fp32 products it computes (each run as three tf32 MMAs on split
    operands): per 128-token chunk, K K^T, S^T K^T, (gam Q) K^T, S^T (gam Q)^T,
    E^T P~^T and E^T K~, six 128 x 128 x 128 products, divided by 128 tokens."""
    return 6 * 2 * 128 * 128 * 128 // 128


def run_prefill(w, L, steps, warmup, rank, world, chunked=False):
    """stq_prefill (or, chunked, stq_prefill_chunked) of an L-token prompt over
    the whole batch, K times (each from the state the previous left).  Returns
    the device time (max over ranks)."""
    from linear_attention_recurrent_delta_b200 import binding as B
    dev = torch.device("cuda", torch.cuda.current_device())
    wr = R.rank_workload(w, rank)
    qs = B.QuantizedState(wr.format, wr.batch, wr.heads, device=dev)
    S = W.initial_state(wr, device=dev)
    qs.calibrate_and_quantize(S)
    del S
    x = None
    for l in range(L):   # [L][B][H][...] filled token by token (no second copy)
        xl = W.step_inputs(wr, l, device=dev)
        if x is None:
            x = {k: torch.empty((L,) + tuple(v.shape), dtype=v.dtype, device=dev) for k, v in xl.items()}
        for k in xl:
            x[k][l].copy_(xl[k])
    o = torch.empty(L, wr.batch, wr.heads, 128, device=dev)
    seed = W.sr_seed(wr)
    stream = torch.cuda.current_stream()
    fn = B.stq_prefill_chunked if chunked else B.stq_prefill
    for i in range(max(warmup, 3)):
        fn(qs.state, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o, None, seed, i, stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        fn(qs.state, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o, None, seed, 100 + i, stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    status = B.stq_device_status(qs.state)
    if status != B.STQ_OK:
        raise RuntimeError("device status: %s" % B.stq_status_string(status))
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    barrier(world)
    del qs, x, o
    torch.cuda.empty_cache()
    return {"ms": ms, "steps": steps}


def run_lifetime(samples=32, batch=64, reps=20):
    """stq_lifetime_weights over `samples` gate samples of a `batch`-request
    stepquant4-kda state (vector gates): device time per call."""
    from linear_attention_recurrent_delta_b200 import binding as B
    w = [x for x in W.WORKLOADS if x.fmt == "stepquant4_kda"][0].resized(batch=batch)
    dev = torch.device("cuda", torch.cuda.current_device())
    qs = B.QuantizedState(w.format, w.batch, w.heads, device=dev)
    alpha = torch.stack([W.step_inputs(w, t, device=dev)["alpha"] for t in range(samples)]).contiguous()
    out = torch.empty(w.heads, 128, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        B.stq_lifetime_weights(qs.state, alpha, out, stream)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(reps):
        B.stq_lifetime_weights(qs.state, alpha, out, stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / reps
    nbytes = alpha.numel() * 4
    del qs, alpha
    return {"ms": ms, "gbs": nbytes / (ms / 1000.0) / 1e9, "samples": samples, "requests": batch,
            "heads": w.heads, "format": w.fmt, "bytes_read": nbytes}


def run_quantizer(batch=256, reps=3, iters=4):
    """The quantizer side on a stepquant6 state of `batch` requests (column
    scales, so the joint fit has both scales to fit): device time per call of
    stq_calibrate, stq_quantize_state, stq_quantize_state_fit (`iters`
    rounds, impact weights = the mean q^2 of 8 steps' queries per head and
    channel) and stq_dequantize_state, with the HBM rate of the bytes each
    call must move (fp32 state 64 KiB per page, the packed page)."""
    from linear_attention_recurrent_delta_b200 import binding as B
    w = [x for x in W.WORKLOADS if x.fmt == "stepquant6" and x.index > 0][0].resized(batch=batch)
    dev = torch.device("cuda", torch.cuda.current_device())
    qs = B.QuantizedState(w.format, w.batch, w.heads, device=dev)
    S = W.initial_state(w, device=dev)
    imp = torch.stack([W.step_inputs(w, t, device=dev)["q"] for t in range(8)]).square().mean(dim=(0, 1)).contiguous()
    ws = torch.empty(max(B.stq_calibrate_workspace_bytes(qs.state), 8), dtype=torch.uint8, device=dev)
    S_back = torch.empty_like(S)
    stream = torch.cuda.current_stream()
    calls = {
        "stq_calibrate": lambda: B.stq_calibrate(qs.state, S, None, ws, stream),
        "stq_quantize_state": lambda: B.stq_quantize_state(qs.state, S, stream),
        "stq_quantize_state_fit": lambda: B.stq_quantize_state_fit(qs.state, S, imp, iters, stream),
        "stq_dequantize_state": lambda: B.stq_dequantize_state(qs.state, S_back, stream),
    }
    state_b = 128 * 128 * 4
    page_b = B.stq_page_bytes(B.format_from_spec(w.format))
    moved = {"stq_calibrate": state_b, "stq_quantize_state": state_b + page_b,
             "stq_quantize_state_fit": state_b + page_b, "stq_dequantize_state": page_b + state_b}
    out = {"workload": w.name, "pages": w.pages, "fit_rounds": iters}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(reps):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / reps
        gbs = moved[name] * w.pages / (ms / 1000.0) / 1e9
        out[name] = {"ms": ms, "bytes_per_page": moved[name], "hbm_gbs": gbs}
    status = B.stq_device_status(qs.state)
    if status != B.STQ_OK:
        raise RuntimeError("device status: %s" % B.stq_status_string(status))
    del qs, S, S_back, ws
    torch.cuda.empty_cache()
    return out


class OracleSample:
    """The CPU oracle (single thread, as written) stepping a sample of the
    workload's pages: the first ``n_pages`` pages of a batch whose fp32 state
    comes from the workload generator and is quantized by the oracle."""

    def __init__(self, w, n_pages):
        import oracle as O
        self.O = O
        self.fmt = O.format_from_spec(w.format)
        n_pages = max(1, min(n_pages, w.pages))
        b_s = -(-n_pages // w.heads)
        self.ws = w.resized(batch=b_s)
        S = W.initial_state(self.ws).numpy()
        self.perm = O.rank_rows(self.fmt, S)
        pb = O.page_bytes(self.fmt)
        self.n = n_pages
        self.pages = np.zeros(self.ws.pages * pb, np.uint8)
        for i in range(n_pages):
            b, h = divmod(i, w.heads)
            self.pages[i * pb:(i + 1) * pb] = O.pack_page(self.fmt, O.quantize_page(self.fmt, S[b, h], self.perm[h]))
        m = self.ws.pages
        x = W.step_inputs(self.ws, 0)
        self.x = {k: np.ascontiguousarray(v.numpy().reshape(m, -1)) for k, v in x.items()}
        self.o = np.zeros((m, 128), np.float32)
        self.seed = W.sr_seed(w)
        self.t = 0
        self.desc = "%d of %d pages (%s, %d heads)" % (n_pages, w.pages, w.name, w.heads)

    def step(self):
        x = self.x
        self.O.decode_step_pages(self.fmt, self.ws.batch, self.ws.heads, self.pages, self.perm, x["q"], x["k"],
                                 x["v"], np.ascontiguousarray(x["alpha"].reshape(-1)),
                                 np.ascontiguousarray(x["beta"].reshape(-1)), self.o, self.seed, self.t,
                                 0, self.n)
        self.t += 1
        return self.n


def oracle_rate(w, budget_s, n_pages=64):
    """CPU-oracle head-steps/s over about budget_s seconds of work."""
    smp = OracleSample(w, n_pages)
    smp.step()
    done, steps = 0, 0
    t0 = time.perf_counter()
    while True:
        done += smp.step()
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return done / el, "%s x %d steps" % (smp.desc, steps), el


def _oracle_worker(args):
    """One host process of the all-cores baseline: its own 64-page sample of the
    workload (pages differ per process through the batch offset), stepped for
    about budget_s seconds.  Returns (pages stepped, seconds)."""
    index, batch, proc, budget_s = args
    w = W.WORKLOADS[index]
    if batch:
        w = w.resized(batch=batch)
    w = R.rank_workload(w, 1000 + proc)          # a distinct sample per process
    smp = OracleSample(w, 64)
    smp.step()
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        done += smp.step()
    return done, time.perf_counter() - t0


def oracle_rate_all_cores(w, budget_s):
    """The same oracle on the host cores: one spawned process per core this
    process may use (at most 32: each process imports torch), each stepping
    its own sample; head-steps/s = all pages / the slowest process."""
    import multiprocessing as mp
    n = max(1, min(32, len(os.sched_getaffinity(0))))
    ctx = mp.get_context("spawn")   # never fork after the GPU is in use
    jobs = [(w.index, w.batch if w.batch != W.WORKLOADS[w.index].batch else 0, i, budget_s) for i in range(n)]
    with ctx.Pool(n) as pool:
        try:   # bounded: a worker that dies must not hold the bench
            res = pool.map_async(_oracle_worker, jobs).get(timeout=4 * budget_s + 180)
        except Exception:
            pool.terminate()
            return None, n
    done = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    return done / el, n


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-other-seconds", type=float, default=4.0,
                    help="the oracle's single-core run on each other workload")
    ap.add_argument("--cpu-all-seconds", type=float, default=8.0,
                    help="the oracle on every host core (0: skip)")
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    ap.add_argument("--only", action="store_true", help="skip the other workloads")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--paged", action="store_true",
                    help="with --profile: step through the slot table (stq_decode_step_slots)")
    ap.add_argument("--window", type=int, default=0,
                    help="with --profile: per-window steps (stq_window_step) of this window length")
    ap.add_argument("--prefill", type=int, default=0,
                    help="with --profile: stq_prefill of a prompt of this many tokens")
    ap.add_argument("--chunked", action="store_true",
                    help="with --profile --prefill: the chunkwise tensor-core form (stq_prefill_chunked)")
    ap.add_argument("--profile", action="store_true",
                    help="decode steps only: no clock sampling, e2e, CPU baseline or other workloads")
    args = ap.parse_args()
    w = W.WORKLOADS[args.config]
    if args.batch:
        w = w.resized(batch=args.batch)
    spec = w.format
    dtype = "f32"

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        # one step = the oracle over a sample of pages sized so that the whole
        # run (warm-up + timed steps) takes about args.ref_seconds
        probe = OracleSample(w, 8)
        t0 = time.perf_counter()
        for _ in range(3):
            probe.step()
        t_page = (time.perf_counter() - t0) / (3 * probe.n)
        n_pages = int(max(1, min(w.pages, args.ref_seconds / (max(1, args.steps + args.warmup) * t_page))))
        smp = OracleSample(w, n_pages)
        for _ in range(args.warmup):
            smp.step()
        t0 = time.perf_counter()
        done = 0
        for _ in range(args.steps):
            done += smp.step()
        el = time.perf_counter() - t0
        value = done / el
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1000.0 * w.pages / value, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
                "impl": "reference",
                "config": {"workload": w.name, "batch": w.batch, "heads": w.heads, "d_k": 128, "d_v": 128,
                           "format": w.fmt, "parallelism": "pages per rank"},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                                 "sample": "%s per step, %d steps" % (smp.desc, args.steps)},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    world, rank, local = dist_setup(args.gpus)
    from linear_attention_recurrent_delta_b200 import build as build_mod
    if rank == 0:
        build_mod.build()
    barrier(world)
    if args.profile and args.prefill:
        r = run_prefill(w, args.prefill, args.steps, args.warmup, rank, world, chunked=args.chunked)
        if rank == 0:
            print(json.dumps({"workload": w.name, "batch": w.batch, "prompt": args.prefill,
                              "chunked": args.chunked, "ms_per_prefill": r["ms"] / r["steps"]}))
        R.finish(world)
        return
    if args.profile and args.window:
        r = run_window(w, args.window, args.steps, args.warmup, rank, world)
        if rank == 0:
            print(json.dumps({"workload": w.name, "batch": w.batch, "window": args.window,
                              "ms_per_step": r["ms"] / r["steps"], "per_t_ms": r["per_t_ms"]}))
        R.finish(world)
        return
    if args.profile:
        res = run_gpu(w, args.steps, args.warmup, rank, world, sample_clocks=False, e2e_steps=0, paged=args.paged)
        if rank == 0:
            print(json.dumps({"workload": w.name, "batch": w.batch, "ms_per_step": res["ms"] / args.steps}))
        R.finish(world)
        return
    res = run_gpu(w, args.steps, args.warmup, rank, world)
    value = R.aggregate_rate(w.pages, world, args.steps, res["ms"])
    ms_step = res["ms"] / args.steps
    roof = hbm_roofline(spec, w.pages, ms_step, w.name)
    roof["frac_best_repetition"] = roof["frac"] * ms_step / res["reps"]["ms_per_step_best"]
    bpp = roof["bytes_per_head_step"]
    peak, peak_kind = roof["peak"], roof["peak_kind"]
    e2e_value = R.aggregate_rate(w.pages, world, res["e2e_steps"], res["e2e_ms"])
    # the rate the host-to-device copies alone allow (one step's inputs per copy)
    pcie_value = R.aggregate_rate(w.pages, world, 1, res["h2d_copy_ms"])
    copies_value = R.aggregate_rate(w.pages, world, 1, res["copies_ms"])

    paged = None
    if not args.only:
        r = run_gpu(w, args.steps, args.warmup, rank, world, sample_clocks=False, e2e_steps=0, paged=True)
        paged = {"value": R.aggregate_rate(w.pages, world, args.steps, r["ms"]), "unit": UNIT,
                 "entry_point": "stq_decode_step_slots", "table": "random permutation of all %d slots" % w.batch,
                 "frac_of_%s_peak" % peak_kind: bpp * w.pages * args.steps / (r["ms"] / 1000.0) / 1e9 / peak}

    windows = {}
    if not args.only:
        for wl in (4, 8, 16):
            r = run_window(w, wl, max(96, args.steps // 5), args.warmup, rank, world)
            b = window_bytes_per_page(spec, wl)
            gbs = b * w.pages * r["steps"] / (r["ms"] / 1000.0) / 1e9
            windows["W%d" % wl] = {"value": R.aggregate_rate(w.pages, world, r["steps"], r["ms"]), "unit": UNIT,
                                   "hbm_gbs": gbs, "frac_of_%s_peak" % peak_kind: gbs / peak,
                                   "bytes_per_head_step": b, "ms_per_position": r["per_t_ms"]}

    prefill = {}
    if not args.only:
        fl = prefill_flops_per_head_token()
        for L in (16, 64):
            r = run_prefill(w, L, max(10, args.steps // 500), args.warmup, rank, world)
            rate = R.aggregate_rate(w.pages * L, world, r["steps"], r["ms"])
            prefill["L%d" % L] = {"value": rate, "unit": "head-tokens/s", "prompt": L,
                                  "ms_per_prefill": r["ms"] / r["steps"],
                                  "roofline": {"bound": "alu", "achieved": rate * fl / 1e12,
                                               "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                                               "frac": rate * fl / 1e12 / FP32_PEAK_TFLOPS,
                                               "flops_per_head_token": fl}}
        # the chunkwise tensor-core form against the recurrent one: the
        # headline batch with a 512-token prompt, and one request x 32 heads
        # with a 1,024-token prompt (32 pages: few CTAs for the recurrent form);
        # for a scalar-gate headline also one request of the KDA workload
        tf = chunked_flops_per_head_token()
        tc_peak = tf32_peak()
        cases = [("batch256_L512", w.resized(batch=min(w.batch, 256)), 512, 3),
                 ("one_request_L1024", w.resized(batch=1), 1024, 5)]
        if not spec["gate_vector"]:   # the gate-vector form too
            kda = [x for x in W.WORKLOADS if x.format["gate_vector"]][0]
            cases.append(("kda_one_request_L1024", kda.resized(batch=1), 1024, 5))
        for tag, wl, L, n in cases:
            rr = run_prefill(wl, L, n, 2, rank, world)
            rc = run_prefill(wl, L, n, 2, rank, world, chunked=True)
            rate_r = R.aggregate_rate(wl.pages * L, world, rr["steps"], rr["ms"])
            rate_c = R.aggregate_rate(wl.pages * L, world, rc["steps"], rc["ms"])
            prefill["chunked_" + tag] = {
                "workload": wl.name, "value": rate_c, "unit": "head-tokens/s", "prompt": L, "pages": wl.pages,
                "entry_point": "stq_prefill_chunked", "kernel": "stq::prefill_tc_kernel",
                "ms_per_prefill": rc["ms"] / rc["steps"],
                "recurrent_value": rate_r, "speedup_vs_recurrent": rate_c / rate_r,
                "roofline": {"bound": "tensor", "achieved": rate_c * tf / 1e12, "peak": tc_peak[0],
                             "unit": "TFLOP/s", "frac": rate_c * tf / 1e12 / tc_peak[0],
                             "peak_kind": tc_peak[1], "flops_per_head_token": tf,
                             "note": "fp32 products counted once; each runs as three tf32 MMAs"}}

    lifetime = run_lifetime() if not args.only else None
    quantizer = run_quantizer() if (not args.only and rank == 0) else None

    # every other workload of the metric, each with its own roofline, clock
    # record and (rank 0, one GPU) CPU baseline
    others = {}
    if not args.only:
        for i in (1, 2, 3, 4):
            if i == args.config:
                continue
            wi = W.WORKLOADS[i]
            n_steps = max(200, args.steps // 3)
            r = run_gpu(wi, n_steps, args.warmup, rank, world, sample_clocks=True, e2e_steps=0)
            ms_i = r["ms"] / n_steps
            roof_i = hbm_roofline(wi.format, wi.pages, ms_i, wi.name)
            roof_i["frac_best_repetition"] = roof_i["frac"] * ms_i / r["reps"]["ms_per_step_best"]
            others[wi.name] = {"value": R.aggregate_rate(wi.pages, world, n_steps, r["ms"]), "unit": UNIT,
                               "steps": n_steps, "ms_per_step": ms_i, "repetitions": r["reps"],
                               "roofline": roof_i, "clocks": r["clocks"],
                               "target_70pct": i in (2, 3, 4)}

    if rank != 0:
        R.finish(world)
        return
    cpu_v, cpu_sample, _ = oracle_rate(w, args.cpu_seconds) if world == 1 else (None, None, None)
    cpu_all = None
    if world == 1 and args.cpu_all_seconds > 0:
        v_all, n_all = oracle_rate_all_cores(w, args.cpu_all_seconds)
        if v_all:
            cpu_all = {"value": v_all, "unit": UNIT, "cores": n_all, "cpu": cpu_model(),
                       "gbs": v_all * bpp / 1e9, "sample": "64 pages per process (own requests), %.0f s" %
                       args.cpu_all_seconds}
    if world == 1 and args.cpu_other_seconds > 0:
        for name, e in others.items():
            wi = [x for x in W.WORKLOADS if x.name == name][0]
            v_i, s_i, _ = oracle_rate(wi, args.cpu_other_seconds)
            e["cpu_baseline"] = {"value": v_i, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": s_i,
                                 "gbs": v_i * e["roofline"]["bytes_per_head_step"] / 1e9, "cpu": cpu_model()}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "heads": w.heads, "d_k": 128, "d_v": 128,
                   "format": w.fmt, "groups": spec["groups"], "col_scales": spec["col_scales"],
                   "stochastic": spec["stochastic"], "gate_vector": spec["gate_vector"],
                   "parallelism": "pages per rank" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (%.0f MB moved per step)" % (bpp * w.pages / 1e6)},
        "repetitions": res["reps"],
        "roofline": roof,
        "cpu_baseline": ({"value": cpu_v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": cpu_sample,
                          "gbs": cpu_v * bpp / 1e9, "cpu": cpu_model(), "all_cores": cpu_all}
                         if cpu_v else None),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                "steps": res["e2e_steps"], "entry_point": "stq_decode_steps_host",
                "overlap": "copies of neighbouring steps overlap the step (two staging slots)",
                "h2d_copy": {"ms_per_step": res["h2d_copy_ms"],
                             "gbs": res["h2d"] / (res["h2d_copy_ms"] / 1000.0) / 1e9,
                             "bound_value": pcie_value, "frac": e2e_value / pcie_value,
                             "note": "the step's input copies alone from the same pinned buffers, "
                                     "timed by CUDA events: the PCIe bound of value"},
                "copies_both_ways": {"ms_per_step": res["copies_ms"], "bound_value": copies_value,
                                     "frac": e2e_value / copies_value,
                                     "note": "the input copies with o copied back at the same time on a "
                                             "second stream, no kernel"}},
        "gpu_launches": args.steps * world,   # one decode_kernel launch per step and rank (timed region)
        "clocks": res["clocks"],
        "other_workloads": others,
        "paged_step": paged,
        "quantizer": quantizer,
        "lifetime_weights": ({"entry_point": "stq_lifetime_weights", "kernel": "stq::lifetime_kernel",
                              "note": "cold path, once per calibration; one thread per (head, channel)",
                              **lifetime} if lifetime else None),
        "prefill": ({"entry_point": "stq_prefill", "kernel": "stq::prefill_kernel",
                     "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz", "prompts": prefill}
                    if prefill else None),
        "window_decode": ({"entry_point": "stq_window_step",
                           "kernels": ["stq::window_step_kernel", "stq::window_commit_kernel"],
                           "windows": windows} if windows else None),
    }
    print(json.dumps(line))
    R.finish(world)


if __name__ == "__main__":
    main()

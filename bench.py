"""Benchmark of the LLM.int8() decomposed linear layer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one i8_linear_forward over one batch (outlier scan, activation quantisation,
int8 tcgen05 GEMM with the fused fp16 outlier product, dequantisation and bias).  The
weight is quantised once before timing (i8_quantize_weight; timed separately and reported
under "weight_quant").  Inputs are synthetic (numpy PCG64, see synth.py) with the shape of
the named workload; the default, and the line's headline, is the OPT-175B-shaped layer,
X [8192, 12288] x W [49152, 12288] with 8 planted outlier columns at threshold 6 (the
largest of the layer shapes, and the one the outlier-density sweep is quoted on).

Timing: W untimed warm-up steps; then K timed steps, each bracketed by CUDA events on the
launching stream, with a 256 MiB buffer written between steps (outside the events) to
flush the 126 MB L2 when the step's inputs (X and CB) are smaller than twice the L2 --
larger inputs stream from HBM every step anyway, and the config line says which was
done; barrier + synchronize around the loop; value = total effective ops of all ranks /
the slowest rank's summed step time.  A second loop of the same steps records events
around the dominant kernel alone (the "roofline" record).  "e2e" is the same metric
through the public call with host buffers: each step uploads X from pinned host memory
and reads the whole C back, with the copies on two streams of their own overlapping the
forward (two buffer slots); the read-backs are checked bit for bit.

At one GPU, with the default workload, the same run also measures the rest of the layer
shapes (unless --no-extras): "sweep" holds the OPT-175B outlier-density sweep (planted
columns {0, 8, 64, 256} x threshold {6, +inf}) and "per_config" the BLOOM-176B FFN decode
batches (T = 1, 8, 16; bound by HBM), the BLOOM-176B QKV prefill and the OPT-6.7B FFN-up
prefill, each with its step time, effective TOPS and dominant-kernel roofline fraction.

Multi-GPU: one process per GPU (torchrun).  At N GPUs the layer is N times as wide (N x
49152 output channels by default) and rank r holds output channels [r*N0, (r+1)*N0) of
that one layer -- its own rows of the one weight, scales and bias -- with the hidden
states replicated: every rank computes the same outlier mask and row scales and writes its
own columns of C, with no collective on the data path (weak scaling).

--impl reference times the CPU oracle (oracle/, plain C) on this host's cores on the
same workload, each step a bounded row sample, and prints the same line with
"impl": "reference".  Only rank 0 runs it.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_matmul_decomposition_b200 import synth  # noqa: E402

METRIC = "int8 decomposed linear: effective TOPS & HBM GB/s, % of sm_100a roofline"
DEFAULT_WORKLOAD = "opt175b_cols8_thr6"
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 1000 * 1000      # B200 L2 capacity (nominal)
# int8 (and e4m3) dense tensor ops per SM per clock of tcgen05 (8192 multiply-adds), the
# instruction rate ncu reports for the int8 pipe; x SMs x SM clock = the pipe's peak
PIPE_OPS_PER_SM_CLK = 16384
# NVIDIA's dense B200 figures, for context: int8 4.5 POPS, HBM3e 8 TB/s class
DATASHEET_I8_TOPS = 4500.0
DATASHEET_HBM_GBS = 8000.0


def l2_policy(mode, T, N, K):
    """(flush?, description) for the timed loops: a 256 MiB buffer is written between
    steps unless the step's inputs (CB and X) are at least twice the L2, in which case each
    step streams them from HBM anyway (and a written flush would only leave dirty lines for
    the next step to write back)."""
    inputs = N * K + 2 * T * K
    if mode == "always" or inputs < 2 * L2_BYTES:
        return True, "256 MiB buffer written between timed steps (outside the events)"
    return False, ("no flush: the step's inputs (CB %.0f MB + X %.1f MB) are %.1fx the 126 MB "
                   "L2, so every step streams them from HBM" %
                   (N * K / 1e6, 2 * T * K / 1e6, inputs / L2_BYTES))


def workloads():
    w = {"opt_ffn_up": synth.opt_ffn_up_prefill(), "bloom_qkv": synth.bloom_qkv_prefill(),
         "tiny": synth.tiny()}
    for T in (1, 8, 16):
        w["bloom_decode_%d" % T] = synth.bloom_ffn_decode(T)
    for c in (0, 8, 64, 256):
        for thr in (6.0, math.inf):
            w["opt175b_cols%d_thr%s" % (c, "inf" if math.isinf(thr) else "6")] = \
                synth.opt175b_sweep(c, thr)
    return w


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def tensor_peak(pk, clk, e4m3=False):
    """The 8-bit tensor peak (TOPS) the GEMM is held to: twice a measured bf16 cuBLAS
    figure (the nominal dense int8 : bf16 and fp8 : bf16 rates are 2 : 1).  The burst
    figure serves a kernel that ran at burst clocks; when the clocks sampled during the
    timed region show the power cap (sw_power_cap), the sustained figure, measured under
    that cap, is the fair one.  Without a clock record the burst figure, the larger, is
    used.  Returns (peak, basis)."""
    capped = clk is not None and "sw_power_cap" in (clk.get("reasons") or [])
    bf16 = pk["bf16_sus"] if capped else pk["bf16"]
    why = ("sw_power_cap seen in the timed region" if capped else
           "no clock record" if clk is None else "no power cap seen in the timed region")
    basis = "%s %s bf16 %.1f TF/s x 2 (nominal %s:bf16 ratio); %s" % (
        pk["source"], "sustained" if capped else "burst", bf16, "fp8" if e4m3 else "int8", why)
    return 2.0 * bf16, basis


def json_threshold(t):
    """A threshold for the JSON line: +inf as the string "inf" (JSON has no infinity)."""
    return "inf" if math.isinf(t) else t


def pipe_peak_tops(sms, sm_mhz):
    """The tensor pipe's int8 instruction rate at the given SM clock (TOPS)."""
    if not sms or not sm_mhz:
        return None
    return PIPE_OPS_PER_SM_CLK * sms * sm_mhz * 1e6 / 1e12


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks of the default process group
    (identity without one).  Used for every device time the line reports."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def rank_workload(w, rank, world):
    """Weak scaling over one layer: with `world` GPUs the layer has world * N output
    channels, and rank r holds rows synth.shard_rows(world * N, r, world) of its weight,
    scales and bias (N of them).  Returns (layer, rows): the layer's workload and the rank's
    [r0, r1).  The hidden states are the same on every rank."""
    import dataclasses
    layer = w if world == 1 else dataclasses.replace(
        w, N=w.N * world, name="%s_x%d_wide" % (w.name, world))
    return layer, synth.shard_rows(layer.N, rank, world)


# ----------------------------------------------------------------------------- clocks
NVML_REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                ("hw_thermal_slowdown", 0x40))


def summarise_clock_samples(samples, t0, t1):
    """Clock record of the samples taken inside [t0, t1]: samples are (time, sm_mhz,
    max_mhz, reason_bits, power_w).  None when no sample falls inside."""
    inside = [x for x in samples if t0 <= x[0] <= t1]
    if not inside:
        return None
    reasons = sorted({name for x in inside for name, bit in NVML_REASONS if x[3] & bit})
    return {"sm_mhz": statistics.median(x[1] for x in inside),
            "sm_max_mhz": inside[0][2], "reasons": reasons, "samples": len(inside),
            "power_w_max": max(x[4] for x in inside),
            "source": "NVML every ~2 ms, timed region only"}


class ClockSampler:
    """SM clock, throttle reasons and power of the GPU, read through NVML by a background
    thread every ~2 ms; begin() / end() delimit the timed region, and stop() summarises
    the samples inside it (NVML reads only: nothing is set)."""

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.samples = []
        self.t0 = self.t1 = None
        self.thread = None
        self.running = False

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                if (u.decode() if isinstance(u, bytes) else u) == self.uuid:
                    return pynvml, h
        import torch
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())

    def start(self):
        import threading
        try:
            nv, h = self._handle()
            max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            return

        def run():
            while self.running:
                try:
                    self.samples.append((time.monotonic(),
                                         float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         max_mhz,
                                         int(nv.nvmlDeviceGetCurrentClocksEventReasons(h)),
                                         nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception:
                    return
                time.sleep(0.002)

        self.running = True
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def begin(self):
        self.t0 = time.monotonic()

    def end(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.thread is None:
            return None
        self.running = False
        self.thread.join(timeout=5)
        if self.t0 is None or self.t1 is None:
            return None
        return summarise_clock_samples(self.samples, self.t0, self.t1)


# ----------------------------------------------------------------------------- helpers
def work_counts(T, N, K, n_o):
    """Algorithmic work and bytes of one forward."""
    i8_ops = 2.0 * T * N * (K - n_o)
    f16_flops = 2.0 * T * N * n_o
    eff_ops = 2.0 * T * N * K
    # X read twice (scan, quantise), Xq written and read, CB read, SCB/bias, C written,
    # the fp16 outlier slices written and read
    bytes_ = (2 * 2 * T * K + 2 * T * K + N * K + 4 * N + 2 * N + 2 * T * N
              + 2 * (2 * T * n_o + 2 * N * n_o))
    return i8_ops, f16_flops, eff_ops, bytes_


def traffic_record(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary (profiles/dram_traffic.txt), if
    it was taken on this workload and on the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(path) as f:
            lines = [l.split(None, 4) for l in f if l.strip() and not l.startswith("#")]
    except OSError:
        return None
    for parts in lines:
        if (len(parts) >= 4 and parts[0] == kernel and parts[2] == source_hash(kernel)
                and parts[3] == workload):
            return {"dram_bytes_per_launch": int(parts[1]),
                    "note": parts[4].strip() if len(parts) > 4 else ""}
    return None


# The CUDA sources that decide a kernel's code and launch: its own header, the headers it
# includes, and the host code that sizes its launch.
CUDA_SOURCES = ("api.cu", "common.cuh", "quant.cuh", "gemm.cuh", "gemm_wide.cuh", "gemv.cuh",
                "bwd.cuh")
KERNEL_SOURCES = {
    "decode_kernel": ("api.cu", "common.cuh", "quant.cuh", "gemv.cuh"),
    "prepare_kernel": ("api.cu", "common.cuh", "quant.cuh"),
    "i8_gemm_tcgen05_kernel": ("api.cu", "common.cuh", "gemm.cuh"),
    "i8_gemm_wide_kernel": ("api.cu", "common.cuh", "gemm.cuh", "gemm_wide.cuh"),
}


def source_hash(kernel=None):
    """sha256 over the sources of `kernel` (all CUDA sources for an unknown kernel)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, CUDA_SOURCES):
        with open(os.path.join(ROOT, "bit_matmul_decomposition_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def fp16_tensor(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).to(device)


# ----------------------------------------------------------------------------- CPU oracle
def sample_rows(w, X, CB, SCB, b, budget_s):
    """Rows of the oracle's row sample that take about budget_s: a call costs a fixed part
    (the scan and row quantisation of all T rows; the mask needs every row) plus a part per
    sampled row, both fitted from two short calls."""
    from oracle import oracle as O
    T = X.shape[0]
    r2 = min(T, 8)
    t = []
    for r in (1, r2):
        t0 = time.perf_counter()
        O.linear_forward(X, CB, SCB, b, w.threshold, rows=np.arange(r))
        t.append(time.perf_counter() - t0)
    per_row = max((t[1] - t[0]) / max(r2 - 1, 1), 1e-6)
    fixed = max(t[0] - per_row, 0.0)
    return int(max(1, min(T, (budget_s - fixed) / per_row)))


def oracle_sample(w, X, CB, SCB, b, budget_s):
    """Time the oracle on a row sample of the workload: the whole scan + row quantisation
    (the mask needs every row) and the int8 product/dequant/outlier/bias for `rows` rows,
    sized to take about budget_s.  Returns (seconds, rows, effective ops)."""
    from oracle import oracle as O
    T = X.shape[0]
    rows = sample_rows(w, X, CB, SCB, b, budget_s)
    sel = np.linspace(0, T - 1, rows).astype(np.int64)
    calls = 0
    t0 = time.perf_counter()
    while True:   # (when all T rows take less than the budget, whole calls are repeated)
        O.linear_forward(X, CB, SCB, b, w.threshold, rows=sel)
        calls += 1
        dt = time.perf_counter() - t0
        if dt >= 0.8 * budget_s or rows < T:
            break
    return dt, rows * calls, 2.0 * rows * calls * w.N * w.K


def run_reference(args, w):
    """--impl reference: the oracle on the host cores, same workload, per-step row sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle as O
    X, W, b = synth.make_x(w), synth.make_w(w), synth.make_bias(w)
    CB, SCB = O.quantize_weight(W)
    per_step = max(0.05, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = sample_rows(w, X, CB, SCB, b, per_step)
    sel = np.linspace(0, w.T - 1, rows).astype(np.int64)
    for _ in range(args.warmup):
        O.linear_forward(X, CB, SCB, b, w.threshold, rows=sel)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.linear_forward(X, CB, SCB, b, w.threshold, rows=sel)
    dt = time.perf_counter() - t0
    ops = 2.0 * rows * w.N * w.K * args.steps
    val = ops / dt / 1e12
    sample = ("per step: scan + row quantisation of all %d rows, then int8 product, "
              "dequant, fp64 outlier part and bias for %d of %d rows" % (w.T, rows, w.T))
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": dict(w.describe(), sample_rows=rows),
            "cpu_baseline": {"value": val, "unit": "TOPS", "cores": O.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
class Layer:
    """One workload's device tensors: X, CB/SCB (quantised here, timed), bias, C and the
    forward's workspace."""

    def __init__(self, abi, w, dev, rows=None, e4m3=False, X=None, CB=None, SCB=None):
        import torch
        self.w, self.dev, self.e4m3 = w, dev, e4m3
        r0, r1 = (0, w.N) if rows is None else rows
        self.T, self.K, self.N = w.T, w.K, r1 - r0
        self.X_h = synth.make_x(w) if X is None else X
        self.X = fp16_tensor(self.X_h, dev)
        b = synth.make_bias(w, (r0, r1))
        self.b = None if b is None else fp16_tensor(b, dev)
        self.wq_ms = None
        if CB is None:
            W = fp16_tensor(synth.make_w(w, (r0, r1)), dev)
            self.CB = torch.empty((self.N, self.K), dtype=torch.uint8 if e4m3 else torch.int8,
                                  device=dev)
            self.SCB = torch.empty((self.N,), dtype=torch.float32, device=dev)
            quantize = abi.i8_quantize_weight_e4m3 if e4m3 else abi.i8_quantize_weight
            quantize(W, self.CB, self.SCB)
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            reps = 5
            ev[0].record()
            for _ in range(reps):
                quantize(W, self.CB, self.SCB)
            ev[1].record()
            torch.cuda.synchronize()
            self.wq_ms = ev[0].elapsed_time(ev[1]) / reps
            del W
        else:
            self.CB, self.SCB = CB, SCB
        size = abi.i8_linear_workspace_size_e4m3 if e4m3 else abi.i8_linear_workspace_size
        self.ws = torch.empty((size(self.T, self.N, self.K),), dtype=torch.uint8, device=dev)
        self.C = torch.empty((self.T, self.N), dtype=torch.float16, device=dev)
        # outlier count of this input (the scan's device scalar), for the work accounting
        mask = torch.empty(((self.K + 31) // 32,), dtype=torch.int32, device=dev)
        idx = torch.empty((self.K,), dtype=torch.int32, device=dev)
        n_o = torch.empty((4,), dtype=torch.int32, device=dev)
        abi.i8_outlier_scan(self.X, w.threshold, mask, idx, n_o)
        self.n_o = int(n_o[0].item())

    def weight_quant(self, pk):
        if self.wq_ms is None:
            return None
        gbs = 3.0 * self.N * self.K / (self.wq_ms * 1e-3) / 1e9
        return {"ms": self.wq_ms, "gbs": gbs, "frac_hbm": gbs / pk["hbm"],
                "frac_of_datasheet_hbm": gbs / DATASHEET_HBM_GBS,
                "bytes": 3 * self.N * self.K + 4 * self.N}


def time_forward(abi, forward, steps, warmup, flush_l2, stream, uuid, barrier=lambda: None):
    """`steps` whole steps, each bracketed by events (clocks sampled meanwhile), with events
    around the dominant kernel inside every fourth step (and the last), so that the kernel's
    time and the step's come from the same loop in the same power and thermal state.  (Kernel
    events cost their step the launch overlap of its two kernels, ~10 us; sampling one step
    in four keeps that out of the step time almost entirely.)  Returns (summed step ms,
    kernel ms averaged over the sampled steps x steps, clock record)."""
    import torch
    for _ in range(warmup):
        flush_l2()
        forward()
    st = abi.i8_sync_status()
    if st != 0:
        raise RuntimeError("device error during warm-up: %s" % abi.STATUS.get(st, st))
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    kv_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    kv_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in kv_s + kv_e:          # torch creates the CUDA event on its first record
        e.record(stream)
    clocks = ClockSampler(uuid)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.05)
    clocks.begin()
    sampled = [i for i in range(steps) if i % 4 == 3 or i == steps - 1]
    for i in range(steps):
        flush_l2()
        ev_s[i].record(stream)
        if i in sampled:
            abi.i8_set_profile_events(kv_s[i], kv_e[i])
        forward()
        abi.i8_set_profile_events(None, None)
        ev_e[i].record(stream)
    torch.cuda.synchronize()
    clocks.end()
    barrier()
    clk = clocks.stop()
    st = abi.i8_sync_status()
    if st != 0:
        raise RuntimeError("device error in the timed loop: %s" % abi.STATUS.get(st, st))
    step_ms = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(steps))
    kern_ms = steps * sum(kv_s[i].elapsed_time(kv_e[i]) for i in sampled) / len(sampled)
    return step_ms, kern_ms, clk


def roofline(abi, L, kern_per, clk, pk, sms):
    """The dominant kernel against its roofline: the decode kernel (the whole forward of a
    decode batch, one stream of CB) against HBM bandwidth, else the tcgen05 GEMM against
    the 8-bit tensor peak.  `peak` is the measured figure; the pipe instruction rate at the
    sampled SM clock and the datasheet figure are given beside it."""
    T, N, K, n_o = L.T, L.N, L.K, L.n_o
    i8_ops, f16_flops, _, _ = work_counts(T, N, K, n_o)
    if T <= 16 and not L.e4m3:
        nbytes = N * K + 2 * T * K + 4 * N + (2 * N if L.b is not None else 0) + 2 * T * N
        achieved = nbytes / (kern_per * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "kernel": "decode_kernel",
                "peak_basis": "%s HBM copy bandwidth" % pk["source"],
                "frac_of_datasheet_peak": achieved / DATASHEET_HBM_GBS,
                "algorithmic_bytes_per_launch": nbytes, "kernel_ms": kern_per}
    # int8 (or e4m3) ops plus the fp16 flops counted at the 8-bit rate x 2 (the nominal
    # fp16 : int8 : fp8 dense rates are 1 : 2 : 2)
    equiv = i8_ops + 2.0 * f16_flops
    achieved = equiv / (kern_per * 1e-3) / 1e12
    peak_i8, basis = tensor_peak(pk, clk, L.e4m3)
    mhz = clk.get("sm_mhz") if clk else None
    pipe = pipe_peak_tops(sms, mhz)
    # the GEMM variant the library picks for these sizes on this device (the e4m3 forward
    # runs a GEMM at every T)
    kernel = abi.i8_forward_kernel(T, N, K)
    if kernel == "decode_kernel":
        kernel = "i8_gemm_tcgen05_kernel"
    return {"bound": "tensor", "achieved": achieved, "peak": peak_i8, "unit": "TOPS",
            "frac": achieved / peak_i8, "kernel": kernel,
            "peak_basis": basis,
            "frac_of_burst_peak": achieved / (2.0 * pk["bf16"]),
            "frac_of_sustained_peak": achieved / (2.0 * pk["bf16_sus"]),
            "frac_of_pipe_peak": None if pipe is None else achieved / pipe,
            "pipe_peak_basis": None if pipe is None else (
                "%d ops/clk/SM x %d SMs x median %.0f MHz sampled in the timed loop = %.0f TOPS"
                % (PIPE_OPS_PER_SM_CLK, sms, mhz, pipe)),
            "frac_of_datasheet_peak": achieved / DATASHEET_I8_TOPS,
            "algorithmic_ops_per_launch": equiv, "kernel_ms": kern_per}


def measure_layer(abi, L, steps, warmup, l2_mode, stream, uuid, pk, sms, forward=None):
    """Step time, effective TOPS and the dominant kernel's roofline of one layer."""
    import torch
    use_flush, l2_desc = l2_policy(l2_mode, L.T, L.N, L.K)
    flush = torch.empty((L2_FLUSH_BYTES if use_flush else 16,), dtype=torch.uint8,
                        device=L.dev)

    def flush_l2():
        if use_flush:
            flush.zero_()

    if forward is None:
        def forward():
            abi.i8_linear_forward(L.X, L.CB, L.SCB, L.b, L.w.threshold, L.C, L.ws)
    step_ms, kern_ms, clk = time_forward(abi, forward, steps, warmup, flush_l2, stream, uuid)
    ms = step_ms / steps
    _, _, eff, nbytes = work_counts(L.T, L.N, L.K, L.n_o)
    roof = roofline(abi, L, kern_ms / steps, clk, pk, sms)
    return {"workload": L.w.name, "T": L.T, "N": L.N, "K": L.K,
            "threshold": json_threshold(L.w.threshold),
            "n_outliers": L.n_o, "steps": steps, "ms_per_step": ms,
            "effective_tops": eff / (ms * 1e-3) / 1e12,
            "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "l2": l2_desc,
            "roofline": {k: v for k, v in roof.items()
                         if k not in ("pipe_peak_basis", "peak_basis")},
            "clocks": None if clk is None else {"sm_mhz": clk["sm_mhz"],
                                                "reasons": clk["reasons"]}}


def run_extras(abi, head, dev, stream, uuid, pk, sms, steps):
    """The other layer shapes, measured in the same run: the OPT-175B density sweep (same
    weight as the headline) and the BLOOM decode / QKV and OPT-6.7B FFN-up layers."""
    import torch
    sweep = []
    xs = {}
    for c in (0, 8, 64, 256):
        for thr in (6.0, math.inf):
            w = synth.opt175b_sweep(c, thr)
            if w.name == head.w.name:
                continue
            if c not in xs:      # the two thresholds share their hidden states
                xs = {c: synth.make_x(w)}
            L = Layer(abi, w, dev, X=xs[c], CB=head.CB, SCB=head.SCB)
            sweep.append(measure_layer(abi, L, max(5, steps // 2), 3, "auto", stream, uuid,
                                       pk, sms))
            del L
            torch.cuda.empty_cache()
    per = {}
    jobs = [("bloom_ffn_decode_T%d" % T, synth.bloom_ffn_decode(T), 100) for T in (1, 8, 16)]
    jobs += [("bloom_qkv_prefill", synth.bloom_qkv_prefill(), max(5, steps // 2)),
             ("opt6.7b_ffn_up_prefill", synth.opt_ffn_up_prefill(), 200)]
    shared = None      # the three decode batches share one weight
    for key, w, n in jobs:
        if shared is not None and w.seed == shared.w.seed:
            L = Layer(abi, w, dev, CB=shared.CB, SCB=shared.SCB)
        else:
            shared = None
            torch.cuda.empty_cache()
            L = Layer(abi, w, dev)
        rec = measure_layer(abi, L, n, 5, "auto", stream, uuid, pk, sms)
        wq = L.weight_quant(pk)
        if wq is not None:
            rec["weight_quant"] = wq
        per[key] = rec
        if w.T <= 16:
            shared = L
        del L
    del shared
    torch.cuda.empty_cache()
    return sweep, per


def run_gpu(args, w0):
    import torch
    import torch.distributed as dist

    from bit_matmul_decomposition_b200 import abi

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    layer, rows = rank_workload(w0, rank, world)
    abi.load()
    stream = torch.cuda.current_stream()
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    e4m3 = args.format == "e4m3"
    if e4m3 and args.outlier_cache:
        raise SystemExit("--outlier-cache applies to the int8 forward only")
    L = Layer(abi, layer, dev, rows=rows, e4m3=e4m3)
    T, K, N = L.T, L.K, L.N
    use_flush, l2_desc = l2_policy(args.l2_flush, T, N, K)
    flush = torch.empty((L2_FLUSH_BYTES if use_flush else 16,), dtype=torch.uint8, device=dev)

    def flush_l2():
        if use_flush:
            flush.zero_()

    cache = None
    if args.outlier_cache:
        # capacity: every column, so any outlier set of this layer is cached
        cache = torch.empty((abi.i8_outlier_cache_size(N, K, K),), dtype=torch.uint8,
                            device=dev)
        abi.i8_outlier_cache_reset(cache)

    def forward(X_in, C_out):
        if e4m3:
            abi.i8_linear_forward_e4m3(X_in, L.CB, L.SCB, L.b, layer.threshold, C_out, L.ws)
        elif cache is None:
            abi.i8_linear_forward(X_in, L.CB, L.SCB, L.b, layer.threshold, C_out, L.ws)
        else:
            abi.i8_linear_forward_cached(X_in, L.CB, L.SCB, L.b, layer.threshold, C_out, L.ws,
                                         cache)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    K_steps = args.steps
    step_ms, kern_ms, clk = time_forward(abi, lambda: forward(L.X, L.C), K_steps, args.warmup,
                                         flush_l2, stream, uuid, barrier)
    step_ms, kern_ms = max_over_ranks([step_ms, kern_ms], dev)

    i8_ops, f16_flops, eff_ops, bytes_ = work_counts(T, N, K, L.n_o)
    ms_per_step = step_ms / K_steps
    value = world * eff_ops / (ms_per_step * 1e-3) / 1e12
    hbm_gbs = bytes_ / (ms_per_step * 1e-3) / 1e9

    # ---------------------------------------------------------------- end to end
    # Through the public call with host buffers: every step uploads its X from pinned host
    # memory and reads its whole C back into pinned host memory.  The forward stays on one
    # stream (calls that share a workspace must be ordered); uploads and read-backs run on
    # two copy streams, and two buffer slots let step i+1's upload and step i-1's read-back
    # overlap step i's forward, as a serving loop would.  The L2 flush, when the policy
    # asks for one, runs on the forward stream inside the timed region.
    e2e_steps = max(3, min(K_steps, 50))
    depth = 2
    X_h = torch.from_numpy(np.ascontiguousarray(L.X_h).view(np.int16)).view(
        torch.float16).pin_memory()
    C_h = [torch.empty((T, N), dtype=torch.float16).pin_memory() for _ in range(depth)]
    X_in = [torch.empty_like(L.X) for _ in range(depth)]
    C_out = [torch.empty_like(L.C) for _ in range(depth)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(depth)]
    ev_fw = [torch.cuda.Event() for _ in range(depth)]
    ev_dn = [torch.cuda.Event() for _ in range(depth)]
    issued = [0]

    def e2e_step():
        i = issued[0]
        j = i % depth
        if i >= depth:
            up.wait_event(ev_fw[j])        # the forward that last read X_in[j] is done
        with torch.cuda.stream(up):
            X_in[j].copy_(X_h, non_blocking=True)
            ev_up[j].record(up)
        flush_l2()
        stream.wait_event(ev_up[j])
        if i >= depth:
            stream.wait_event(ev_dn[j])    # C_out[j] has been read back
        forward(X_in[j], C_out[j])
        ev_fw[j].record(stream)
        down.wait_event(ev_fw[j])
        with torch.cuda.stream(down):
            C_h[j].copy_(C_out[j], non_blocking=True)
            ev_dn[j].record(down)
        issued[0] = i + 1

    def e2e_drain(ev):
        for j in range(min(depth, issued[0])):
            stream.wait_event(ev_dn[j])
        ev.record(stream)

    for _ in range(2 * depth):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    down.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    e2e_drain(e1)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    torch.cuda.synchronize()
    st = abi.i8_sync_status()
    if st != 0:
        raise RuntimeError("device error in the e2e loop: %s" % abi.STATUS.get(st, st))
    # every read-back holds the forward's output (the forward is deterministic)
    C_ref_bits = L.C.cpu().view(torch.int16)
    for j in range(depth):
        if not torch.equal(C_h[j].view(torch.int16), C_ref_bits):
            raise RuntimeError("e2e read-back %d differs from the device-timed output" % j)
    del C_h, X_in, C_out, X_h, C_ref_bits
    e2e_per = max_over_ranks([e2e_ms], dev)[0] / e2e_steps
    e2e_value = world * eff_ops / (e2e_per * 1e-3) / 1e12

    decode = T <= 16 and not e4m3   # (the e4m3 forward runs the GEMM for every T)
    pk = peaks()
    roof = roofline(abi, L, kern_ms / K_steps, clk, pk, sms)
    tr = traffic_record(roof["kernel"], w0.name) if not e4m3 else None
    roof["traffic"] = None if tr is None else tr["dram_bytes_per_launch"]
    if tr is not None:
        roof["traffic_note"] = tr.get("note", "")

    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": K_steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if e4m3 else "int8", "data": "synthetic",
            "config": dict(w0.describe(), n_outliers=L.n_o,
                           parallelism=("one layer of %d x %d output channels split by output "
                                        "channel over %d GPUs; this rank holds [%d, %d)"
                                        % (world, w0.N, world, rows[0], rows[1])
                                        if world > 1 else "one GPU, the whole layer"),
                           l2=l2_desc,
                           **({"code_format": "e4m3 (the FP8 variant of the decomposition)"}
                              if e4m3 else {}),
                           **({"outlier_cache": "on: the fixed input's outlier set is cached "
                                                "during warm-up, every timed step hits"}
                              if cache is not None else {})),
            "hbm_gbs": hbm_gbs * world, "hbm_frac": hbm_gbs / pk["hbm"],
            "roofline": roof,
            "weight_quant": L.weight_quant(pk),
            "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": 2 * T * K,
                    "d2h_bytes_per_step": 2 * T * N, "ms_per_step": e2e_per,
                    "steps": e2e_steps,
                    "pipeline": "forward on one stream; X uploads and C read-backs on two "
                                "copy streams, %d buffer slots; read-backs checked "
                                "bit-exact against the device-timed output" % depth},
            # launches of this library's kernels per step: fused prepare + GEMM, or the one
            # decode kernel (the memsets before them are not kernels of this library)
            "gpu_launches": K_steps * (1 if decode else 2),
            "clocks": clk}

    # CPU baseline: the oracle on this host, rank 0 at N = 1 only
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not e4m3:
        from oracle import oracle as O
        CB_h = L.CB.cpu().numpy()
        SCB_h = L.SCB.cpu().numpy()
        b_h = None if L.b is None else L.b.cpu().view(torch.int16).numpy().view(np.float16)
        dt, nrows, ops = oracle_sample(layer, L.X_h, CB_h, SCB_h, b_h, args.cpu_budget)
        del CB_h
        line["cpu_baseline"] = {
            "value": ops / dt / 1e12, "unit": "TOPS", "cores": O.num_threads(),
            "kind": "oracle",
            "sample": "scan + row quantisation of all %d rows, then int8 product, dequant, "
                      "fp64 outlier part and bias for %d evenly spaced rows (repeated calls "
                      "count again) x all %d outputs (%.1f s)" % (T, nrows, N, dt)}

    if (world == 1 and not args.no_extras and not e4m3 and cache is None
            and w0.name == workloads()[DEFAULT_WORKLOAD].name):
        keep = L
        del L
        sweep, per = run_extras(abi, keep, dev, stream, uuid, pk, sms, K_steps)
        head = {"workload": keep.w.name, "threshold": json_threshold(keep.w.threshold),
                "n_outliers": keep.n_o, "ms_per_step": ms_per_step,
                "effective_tops": value, "roofline": {k: roof[k] for k in (
                    "achieved", "peak", "frac", "frac_of_pipe_peak",
                    "frac_of_datasheet_peak", "kernel_ms")}}
        line["sweep"] = sorted([head] + sweep,
                               key=lambda r: (r["threshold"] == "inf", r["n_outliers"]))
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_train(args, w):
    """--mode train (one GPU): a training step of the fp16-weight mode of the nn.Module
    front end -- re-quantise the fp16 weight, the int8 decomposed forward (library kernels)
    and the straight-through backward (dx = dy W, dW = dy^T x, db = sum dy; fp16 GEMMs) --
    on the workload's shapes.  Reports 3 x 2TNK / step time (forward + two backward
    products), separately from the forward benchmark."""
    import torch

    from bit_matmul_decomposition_b200.linear import Linear8bitLt

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, K, N = w.T, w.K, w.N
    X = fp16_tensor(synth.make_x(w), dev).requires_grad_(True)
    m = Linear8bitLt(K, N, bias=True, threshold=w.threshold, device=dev, has_fp16_weights=True)
    with torch.no_grad():
        m.weight.copy_(fp16_tensor(synth.make_w(w), dev))
        b = synth.make_bias(w)
        if b is not None:
            m.bias.copy_(fp16_tensor(b, dev))
    gy = torch.randn((T, N), device=dev, dtype=torch.float16) * 0.01
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)

    def step():
        X.grad = None
        m.weight.grad = None
        m.bias.grad = None
        m(X).backward(gy)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler()
    clocks.start()
    time.sleep(0.05)
    clocks.begin()
    for e0, e1 in ev:
        flush.zero_()
        e0.record()
        step()
        e1.record()
    torch.cuda.synchronize()
    clocks.end()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    flops = 3.0 * 2.0 * T * N * K
    print(json.dumps({
        "metric": "int8 decomposed linear, training step (fp16 weights re-quantised, "
                  "int8 forward, straight-through fp16 backward)",
        "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "mode": "train", "data": "synthetic",
        "config": dict(w.describe(), l2="256 MiB buffer written between timed steps"),
        "clocks": clk}), flush=True)
    st = abi_status()
    if st != 0:
        raise RuntimeError("device error in the training loop: %s" % st)
    return 0


def abi_status():
    from bit_matmul_decomposition_b200 import abi
    return abi.i8_sync_status()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads()))
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other layer shapes (sweep and per_config records) that the "
                         "default workload's run also measures")
    ap.add_argument("--l2-flush", default="auto", choices=["auto", "always"],
                    help="auto: flush the L2 between timed steps only when the inputs are "
                         "smaller than twice the L2")
    ap.add_argument("--format", default="int8", choices=["int8", "e4m3"],
                    help="code format of the decomposition's 8-bit part (e4m3: the FP8 "
                         "variant, not the benchmark's headline configuration)")
    ap.add_argument("--outlier-cache", action="store_true",
                    help="forward through i8_linear_forward_cached (the weight's outlier "
                         "columns kept across calls)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count T (a smaller case of the same "
                         "layer, e.g. for profiler captures); the line then names T")
    ap.add_argument("--mode", default="forward", choices=["forward", "train"],
                    help="train: one GPU, the fp16-weight training step of the module "
                         "front end (not the forward benchmark)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = workloads()[args.workload]
    if args.tokens is not None:
        import dataclasses
        if args.tokens < 1:
            raise SystemExit("--tokens must be positive")
        w = dataclasses.replace(w, T=args.tokens, name="%s_T%d" % (w.name, args.tokens))
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "train":
        return run_train(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())

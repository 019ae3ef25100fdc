#!/usr/bin/env python
"""Benchmark of the MXFP8 training hot path on B200.

One step = the MoE grouped layer forward + backward on the MoE benchmark
shape of ao PR #4705 ("Wire MoE and MXFP8Linear training paths to CuTeDSL by
default", roofline benchmark at K=N=4096, G=8, M=16384), run through every
cast and GEMM of the path:

  1. X   [16384, 4096]      fused dim0 + dim1 cast into padded groups (pad path;
                            the dim1 codes are kept for the wgrad)
  2. W   [8, 4096, 4096]    32x32 cast (codes + forward and dgrad scale views)
  3. fwd grouped GEMM       Y  = X_g W_g^T          (M groups)
  4. dY  [16384, 4096]      fused dim0 + dim1 cast into padded groups
  5. dgrad grouped GEMM     dX = dY_g W_g           (M groups, W codes read MN-major)
  6. wgrad grouped GEMM     dW_g = dY_g^T X_g       (K groups)

value = 3 * 2*M*N*K FLOPs per step / step time (TFLOP/s, whole job). Inputs
are seeded synthetic bf16 tensors on the device (512 MB > the 126 MB L2, so
no explicit flush between steps). The cast bandwidth of the four cast modes
on the 1024^2 ... 16384^2 sweep tensors and the [64, 2048, 7168] expert stack
is reported beside it (L2 flushed before every launch; in-stream and isolated
launch timings), and so are the GEMMs
alone (CUDA-graph replays), the MXFP8 linear at M=4096, N=4096, K=2048, the
unaligned geometry (casts of a [16384, 576] gradient; the grouped GEMMs at
G=32, K=7168, N=2048, M=32768 with skewed groups), the backward-override
arms, and (one GPU only) the same GEMMs through cuBLASLt's MXFP8 kernel and
the high-precision arm's through torch._grouped_mm, timed interleaved with
this library's as context.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs the same step on its own GPU (replicas: the
path has no data exchange) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MXFP8 cast GB/s and grouped-GEMM TFLOPS on 1 B200, as % of HBM / MXFP8 peak"
G, M, N, K = 8, 16384, 4096, 4096
STEP_FLOPS = 3 * 2 * M * N * K
GEMM_FLOPS = 2 * M * N * K
WORKLOAD = "MoE grouped GEMM fwd+bwd with MXFP8 casts, G=8, K=N=4096, M=16384 (Dirichlet(1) groups)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0     # nominal dense ratio (4.5 / 2.25 PFLOP/s)


# ------------------------------------------------------------------ utils --
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(value, world):
    """Max of a float over ranks (control plane only)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(step_ms_local, steps, world):
    """Whole-job throughput from per-rank timings: every rank did the same work."""
    total_ms = reduce_max(step_ms_local * steps, world)
    ms_per_step = total_ms / steps
    value = world * STEP_FLOPS * steps / (total_ms * 1e-3) / 1e12
    return value, ms_per_step


# The sampler runs in a process of its own: NVML readings stamped with the
# system-wide monotonic clock by that process, so a busy host thread holding
# the interpreter lock cannot thin them out. One per device, shared by every
# measured region; each region keeps the readings stamped inside it.
_SAMPLER_SRC = r"""
import os, sys, time
import pynvml
pynvml.nvmlInit()
dev, period, deadline, path = sys.argv[1], float(sys.argv[2]), time.monotonic() + float(sys.argv[3]), sys.argv[4]
parent = int(sys.argv[6])
try:
    h, how = pynvml.nvmlDeviceGetHandleByUUID(dev), "uuid"
except Exception:
    h, how = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[5])), "index"
with open(path, "a", buffering=1) as out:
    out.write("# " + how + "\n")
    while time.monotonic() < deadline and os.getppid() == parent:    # ends with its parent, however that ends
        try:
            mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            out.write("%.6f %d %d\n" % (time.monotonic(), mhz, mask))
        except Exception:
            pass
        time.sleep(period)
"""
_samplers = {}


def start_clock_sampler(local, period_s=0.0005, lifetime_s=1800.0):
    """Start (once) the NVML sampler process of CUDA device `local`; returns its
    (output path, max SM MHz) or None without NVML. NVML does not see
    CUDA_VISIBLE_DEVICES, so the device is named by its UUID (index as fallback)."""
    if local in _samplers:
        return _samplers[local]
    import atexit
    import subprocess
    import tempfile
    try:
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
        try:
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(local)
        max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:
        _samplers[local] = None
        return None
    fd, path = tempfile.mkstemp(prefix="mx_clocks_", suffix=".txt")
    os.close(fd)
    proc = subprocess.Popen([sys.executable, "-c", _SAMPLER_SRC, uuid, str(period_s), str(lifetime_s), path,
                             str(local), str(os.getpid())], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)

    def _stop():
        proc.terminate()
        try:
            proc.wait(timeout=5)
        except Exception:
            proc.kill()
        try:
            os.remove(path)
        except OSError:
            pass
    atexit.register(_stop)
    t_end = time.monotonic() + 20.0          # until its first reading is in
    while time.monotonic() < t_end and proc.poll() is None:
        with open(path) as fh:
            if sum(1 for line in fh if not line.startswith("#")) > 0:
                break
        time.sleep(0.01)
    _samplers[local] = (path, max_mhz)
    return _samplers[local]


class ClockSampler:
    """SM clock and clock-event reasons of one device during a region (readings
    of the sampler process whose stamps fall between entry and exit)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, local):
        self.sampler = start_clock_sampler(local)
        self.t0 = self.t1 = None

    def __enter__(self):
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        self.t1 = time.monotonic()

    def summary(self):
        if self.sampler is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        path, max_mhz = self.sampler
        t1 = self.t1 if self.t1 is not None else time.monotonic()
        mhz, reasons, device = [], set(), None
        with open(path) as fh:
            for line in fh:
                if line.startswith("#"):
                    device = line[1:].strip()
                    continue
                parts = line.split()
                if len(parts) != 3 or not (self.t0 <= float(parts[0]) <= t1):
                    continue
                mhz.append(int(parts[1]))
                mask = int(parts[2])
                reasons.update(n for n, bit in self.REASONS.items() if mask & bit and n != "gpu_idle")
        out = {"sm_mhz": sorted(mhz)[len(mhz) // 2] if mhz else None, "sm_max_mhz": max_mhz,
               "reasons": sorted(reasons), "samples": len(mhz)}
        if device is not None:
            out["nvml_device_by"] = device
        return out


def profile_traffic(name, source_files):
    """Per-launch DRAM bytes from a committed ncu summary, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", name)
    h = hashlib.sha256()
    for f in source_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    fields = dict(line.split(":", 1) for line in text.splitlines() if ":" in line and not line.startswith(" "))
    if fields.get("kernel_source_sha256_16", "").strip() != digest:
        return None
    try:
        return float(fields["traffic_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


class L2Flush:
    """Empties the 126 MB L2 between timed iterations: writes a 256 MB buffer, then
    reads a second one, so that the written lines are evicted (and written back)
    before the timed kernel starts rather than during it."""

    def __init__(self, device, nbytes=256 * 1024 * 1024):
        import torch
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.r = torch.zeros(nbytes // 4, dtype=torch.int32, device=device)

    def zero_(self):
        self.w.zero_()
        self.r.max()


# ------------------------------------------------------------ our step ----
class MoEStep:
    """Preallocated buffers and the six launches of one MoE fwd+bwd step.

    `problem` builds (x, w, dy, offs) for groups G, tokens M, output width N and
    input width K; the default is the MoE benchmark shape."""

    def __init__(self, mx, device, seed=0, shape=(G, M, N, K), problem=None):
        import torch
        from mxfp8_block_scaled_cast_b200 import synthetic as S
        self.mx, self.torch = mx, torch
        g, m, n, k = self.G, self.M, self.N, self.K = shape
        make = problem or S.moe_problem
        self.x, self.w, self.dy, offs = make(G=g, M=m, N=n, K=k, seed=seed, device=device)
        self.offs = offs.to(device)
        cap = self.cap = mx.mx_padded_rows_capacity(m, g)
        u8 = lambda *s: torch.empty(*s, dtype=torch.uint8, device=device)
        bf = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device=device)
        self.xq, self.xs = u8(cap, k), u8(mx.mx_scale_bytes(cap, k // 32))
        self.xqt, self.xst = u8(k, cap), u8(mx.mx_scale_bytes(k, cap // 32))
        self.wq, self.wsf = u8(g, n, k), u8(g * mx.mx_scale_bytes(n, k // 32))
        self.wsd = u8(g * mx.mx_scale_bytes(k, n // 32))
        self.dq, self.ds = u8(cap, n), u8(mx.mx_scale_bytes(cap, n // 32))
        self.dqt, self.dst = u8(n, cap), u8(mx.mx_scale_bytes(n, cap // 32))
        self.y, self.dx, self.dw = bf(m, n), bf(m, k), bf(g, n, k)
        self.launches_per_step = 6
        self.gemm_flops = 2 * m * n * k
        self.gemm_events = []

    def gemms(self):
        """The three grouped GEMMs of the step, as callables (fwd, dgrad, wgrad)."""
        mx, g, m, n, k = self.mx, self.G, self.M, self.N, self.K
        return {
            "fwd": lambda: mx.mx_grouped_mm(self.xq, self.xs, self.wq, self.wsf, self.offs, g, mx.MX_GROUPS_M,
                                            self.y, m, n, k, self.cap),
            "dgrad": lambda: mx.mx_grouped_mm(self.dq, self.ds, self.wq, self.wsd, self.offs, g,
                                              mx.MX_GROUPS_M_KN, self.dx, m, k, n, self.cap),
            "wgrad": lambda: mx.mx_grouped_mm(self.dqt, self.dst, self.xqt, self.xst, self.offs, g,
                                              mx.MX_GROUPS_K, self.dw, m, n, k, self.cap),
        }

    def run(self, timed_gemms=False):
        mx, t = self.mx, self.torch
        mx.mx_cast_2d_grouped(self.x, self.offs, self.cap, self.xq, self.xs, self.xqt, self.xst)
        mx.mx_cast_w32x32(self.w, self.wq, self.wsf, None, self.wsd)
        calls = self.gemms()
        for name in ("fwd", None, "dgrad", "wgrad"):
            if name is None:
                mx.mx_cast_2d_grouped(self.dy, self.offs, self.cap, self.dq, self.ds, self.dqt, self.dst)
                continue
            if timed_gemms:
                a, b = t.cuda.Event(enable_timing=True), t.cuda.Event(enable_timing=True)
                a.record()
                calls[name]()
                b.record()
                self.gemm_events.append((a, b))
            else:
                calls[name]()


def select_peak(region_ms, reasons, peaks):
    """The measured bf16 peak the in-step GEMM rate is held against.

    A timed region of tens of milliseconds is a burst: the burst figure. A long
    one (beyond 100 ms, or one that saw the power cap engage) takes the
    sustained figure, as do the seconds-long back-to-back replays of
    `gemm_only`. Returns (kind, bf16 TFLOP/s, why); a peak missing from the
    measured file falls back to FALLBACK_PEAKS."""
    capped = "sw_power_cap" in reasons
    sustained = region_ms > 100.0 or capped
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    why = f"the timed region lasts {region_ms:.1f} ms" + (" with the power cap engaged" if capped else "")
    return ("sustained" if sustained else "burst"), float(peaks.get(key, FALLBACK_PEAKS[key])), why


def flushed_time(fn, flush, reps=20, pairs=40, runs=15):
    """Seconds per launch of `fn` with the L2 flushed before it, measured two ways.

    isolated   CUDA events around one launch issued after a flush, median of `reps`.
               The stream has drained when the start event fires, so this includes the
               latency of a launch into an idle stream (about 5 us here), which dominates
               tensors of a few MB.
    in_stream  a CUDA graph of `pairs` (flush, launch) pairs minus a graph of `pairs`
               flushes alone, replayed alternately `runs` times, median difference per
               launch: the launch queued behind other work, as inside a training step;
               the write-back of its dirty lines during the next flush is charged to it.
    """
    import torch
    iso = isolated_time(fn, flush, reps)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graphs = []
    with torch.cuda.stream(s):
        for with_fn in (True, False):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                for _ in range(pairs):
                    flush.zero_()
                    if with_fn:
                        fn()
            graphs.append(g)
    torch.cuda.synchronize()

    def replay(g):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    for g in graphs:
        replay(g)
    diffs = sorted((replay(graphs[0]) - replay(graphs[1])) / pairs for _ in range(runs))
    del graphs
    return iso, max(diffs[len(diffs) // 2], 1e-6) * 1e-3


def isolated_time(fn, flush, reps=20):
    """Seconds per launch of `fn`: CUDA events around one launch issued after an
    L2 flush, median of `reps` (3 unflushed warm-up launches first)."""
    import torch
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ts.sort()
    return ts[len(ts) // 2] * 1e-3


CAST_METHOD = ("gbs: in-stream, a CUDA graph of 40 (L2 flush, cast) pairs minus 40 flushes alone, "
               "median of 15 alternating replays; gbs_isolated: CUDA events around one launch after a "
               "flush, median of 20 (includes about 5 us of launch latency into an idle stream)")


def cast_rates(nbytes, times, hbm):
    """GB/s of a cast moving `nbytes`, in-stream and isolated, with the in-stream
    figure's fractions of the measured copy bandwidth and of the 8 TB/s spec."""
    iso, ins = times
    gbs = nbytes / ins / 1e9
    return {"gbs": round(gbs, 1), "gbs_isolated": round(nbytes / iso / 1e9, 1),
            "frac_of_measured_hbm": round(gbs / hbm, 3), "frac_of_8tbs_spec": round(gbs / 8000, 3)}


def cast_sweep(mx, device, flush, hbm):
    """GB/s of each cast mode on the 1024^2 ... 16384^2 sweep tensors and the expert
    stack, L2 flushed before every launch (8192^2, 16384^2 and the stack also
    exceed the L2); bytes are the tensor read plus codes and scales written."""
    import torch
    from mxfp8_block_scaled_cast_b200 import synthetic as S

    out = {"method": CAST_METHOD}
    for n in (1024, 4096, 8192, 16384):
        x = S.sweep_tensor((n, n), seed=0, device=device)
        u8 = lambda *s: torch.empty(*s, dtype=torch.uint8, device=device)
        q, s, qt, st = u8(n, n), u8(mx.mx_scale_bytes(n, n // 32)), u8(n, n), u8(mx.mx_scale_bytes(n, n // 32))
        E = n * n
        modes = {
            "dim0": (lambda: mx.mx_cast_dim0(x, q, s), 2 + 1 + 1 / 32),
            "dim1": (lambda: mx.mx_cast_dim1(x, qt, st), 2 + 1 + 1 / 32),
            "2d": (lambda: mx.mx_cast_2d(x, q, s, qt, st), 2 + 2 + 2 / 32),
            "32x32": (lambda: mx.mx_cast_w32x32(x, q, s, None, st), 2 + 1 + 2 / 32),
        }
        for name, (fn, bpe) in modes.items():
            pairs = 40 if n < 16384 else 10
            out[f"{name}_{n}x{n}_gbs"] = cast_rates(E * bpe, flushed_time(fn, flush, pairs=pairs), hbm)
    del x, q, s, qt, st
    # the pad-path launch of the MoE step: the fused cast of X [16384, 4096] into
    # the padded groups of the Dirichlet(1) sizes (bytes: X read, both padded code
    # copies and both blocked scale buffers written)
    xm, wm, dym, offs = S.moe_problem(seed=0, device=device)
    del wm, dym
    offs = offs.to(device)
    mm, km = xm.shape
    cap = mx.mx_padded_rows_capacity(mm, offs.numel())
    gq, gs = u8(cap, km), u8(mx.mx_scale_bytes(cap, km // 32))
    gqt, gst = u8(km, cap), u8(mx.mx_scale_bytes(km, cap // 32))
    nbytes = mm * km * 2 + 2 * cap * km + gs.numel() + gst.numel()
    out["2d_grouped_moe_16384x4096_gbs"] = cast_rates(
        nbytes, flushed_time(lambda: mx.mx_cast_2d_grouped(xm, offs, cap, gq, gs, gqt, gst), flush), hbm)
    del xm, gq, gs, gqt, gst
    g3, n3, k3 = 64, 2048, 7168
    w = S.sweep_tensor((g3, n3, k3), seed=0, device=device)
    wq = u8(g3, n3, k3)
    sf, sd = u8(g3 * mx.mx_scale_bytes(n3, k3 // 32)), u8(g3 * mx.mx_scale_bytes(k3, n3 // 32))
    out["32x32_64x2048x7168_gbs"] = cast_rates(
        g3 * n3 * k3 * (2 + 1 + 2 / 32),
        flushed_time(lambda: mx.mx_cast_w32x32(w, wq, sf, None, sd), flush, reps=5, pairs=5, runs=5), hbm)
    return out


def graph_time(fn, iters=100, runs=5):
    """Seconds per call of `fn`: a CUDA graph of `iters` back-to-back calls, replayed
    `runs` times, median."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
            for _ in range(iters):
                fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(runs):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / iters)
    ts.sort()
    del g
    return ts[len(ts) // 2] * 1e-3


def gemm_only(mx, step, peaks, iters=100, runs=5):
    """The three grouped GEMMs of a step alone, on the step's prequantized
    operands: each captured as a CUDA graph of `iters` launches and replayed
    `runs` times; median time per launch. No flush (the MoE launches move
    201-335 MB of operands, above the 126 MB L2)."""
    import torch
    step.run()
    torch.cuda.synchronize()
    out = {}
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP8_OVER_BF16
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * FP8_OVER_BF16
    for name, fn in step.gemms().items():
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                for _ in range(iters):
                    fn()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        with ClockSampler(torch.cuda.current_device()) as ck:
            for _ in range(runs):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / iters)
        ts.sort()
        tf = step.gemm_flops / (ts[len(ts) // 2] * 1e-3) / 1e12
        out[name] = {"us_per_launch": round(ts[len(ts) // 2] * 1e3, 1), "tflops": round(tf, 1),
                     "frac_of_measured_sustained_fp8": round(tf / sustained, 3),
                     "frac_of_measured_burst_fp8": round(tf / burst, 3), "frac_of_4500_spec": round(tf / 4500.0, 3),
                     "clocks": ck.summary()}
        del g
    mx.mx_device_error()
    out["method"] = (f"CUDA graph of {iters} back-to-back launches, median of {runs} replays (about 0.1 s "
                     f"of load per GEMM: the sustained regime; `clocks` per GEMM); "
                     f"fp8 peaks = measured bf16 (sustained, burst) x {FP8_OVER_BF16}")
    return out


def library_mxfp8(mx, step, device, iters=(20, 10), rounds=8):
    """The same GEMMs through cuBLASLt's MXFP8 kernel (torch._scaled_mm with E8M0
    scales in the blocked layout this library writes), timed interleaved with this
    library's kernel in one process (CUDA graphs, order flipped each round, median),
    so both see the same power state. Dense 8192^3, and the MoE forward as one
    cuBLASLt call per group (its padded rows; the library has no grouped MXFP8 GEMM)
    against the one grouped launch. Outputs are compared bitwise."""
    import torch
    from mxfp8_block_scaled_cast_b200 import synthetic as S
    f8, e8 = torch.float8_e4m3fn, torch.float8_e8m0fnu

    def capture(fn, n):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                for _ in range(n):
                    fn()
        torch.cuda.synchronize()
        return g

    def replay_ms(g):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    def interleaved(f_ours, f_lib, n, flops):
        ga, gb = capture(f_ours, n), capture(f_lib, n)
        replay_ms(ga)
        replay_ms(gb)
        t = {0: [], 1: []}
        for r in range(rounds):
            for k in ((0, 1) if r % 2 == 0 else (1, 0)):
                t[k].append(replay_ms((ga, gb)[k]) / n)
        del ga, gb
        med = [sorted(v)[len(v) // 2] for v in (t[0], t[1])]
        return {"ours_tflops": round(flops / med[0] / 1e9, 1), "cublaslt_tflops": round(flops / med[1] / 1e9, 1),
                "ours_over_cublaslt": round(med[1] / med[0], 4)}

    out = {"method": "CUDA graphs of back-to-back launches (power-capped), this library and cuBLASLt "
                     f"alternating over {rounds} rounds, median per launch"}
    try:
        n = 8192
        x = S.normal_bf16((n, n), 1.0, seed=1, device=device)
        w = S.normal_bf16((n, n), 0.02, seed=2, device=device)
        xq, xs = mx.cast_dim0(x)
        wq, wsf, _, _ = mx.cast_w32x32(w, transposed=False)
        del x, w
        y = torch.empty(n, n, dtype=torch.bfloat16, device=device)
        ours = lambda: mx.mx_grouped_mm(xq, xs, wq, wsf, None, 1, mx.MX_GROUPS_M, y, n, n, n, 0)
        a8, b8, sa, sb = xq.view(f8), wq.view(f8), xs.view(e8), wsf.view(e8)
        lib = lambda: torch._scaled_mm(a8, b8.t(), sa, sb, out_dtype=torch.bfloat16)
        ours()
        same = bool(torch.equal(lib(), y))
        out["dense_8192"] = dict(interleaved(ours, lib, iters[0], 2 * n ** 3), bitwise_equal=same)
        del xq, xs, wq, wsf, y, a8, b8, sa, sb

        offs = step.offs.cpu().tolist()
        sizes = [offs[0]] + [offs[i] - offs[i - 1] for i in range(1, len(offs))]
        pads = [(v + 127) // 128 * 128 for v in sizes]
        starts = [sum(pads[:i]) for i in range(len(pads))]
        band = mx.mx_scale_bytes(128, step.K // 32)            # one 128-row scale band of X
        per_w = mx.mx_scale_bytes(step.N, step.K // 32)        # one expert's forward scales
        y_pad = torch.empty(sum(pads), step.N, dtype=torch.bfloat16, device=device)
        calls = [(step.xq[p:p + m].view(f8), step.wq[g].view(f8),
                  step.xs[p // 128 * band:(p + m) // 128 * band].view(e8),
                  step.wsf[g * per_w:(g + 1) * per_w].view(e8), y_pad[p:p + m])
                 for g, (p, m) in enumerate(zip(starts, pads)) if m]

        def lib_moe():
            for a8_, b8_, sa_, sb_, yv in calls:
                torch._scaled_mm(a8_, b8_.t(), sa_, sb_, out_dtype=torch.bfloat16, out=yv)
        fwd = step.gemms()["fwd"]
        fwd()
        lib_moe()
        same = all(torch.equal(y_pad[p:p + v], step.y[o - v:o]) for p, v, o in zip(starts, sizes, offs) if v)
        out["moe_fwd_per_group"] = dict(interleaved(fwd, lib_moe, iters[1], step.gemm_flops), bitwise_equal=same,
                                        library_calls=len(calls))
        del y_pad, calls
    except Exception as exc:          # reported, not fatal: the comparison is context
        out["error"] = repr(exc)[:300]
    mx.mx_device_error()
    torch.cuda.empty_cache()
    return out


def library_bf16(mx, step, iters=10, rounds=8):
    """The high-precision arm's bf16 grouped GEMMs against torch._grouped_mm (a
    library grouped GEMM) on the same bf16 operands: dX_g = dY_g W_g over row
    groups and dW_g = dY_g^T X_g over token groups, interleaved CUDA graphs as
    in library_mxfp8, outputs compared bitwise."""
    import torch
    G_, M_, N_, K_ = step.G, step.M, step.N, step.K
    dx = torch.empty(M_, K_, dtype=torch.bfloat16, device=step.dy.device)
    dw = torch.empty(G_, N_, K_, dtype=torch.bfloat16, device=step.dy.device)
    ours = {"dgrad": (lambda: mx.mx_grouped_mm_bf16(step.dy, step.w, step.offs, G_, mx.MX_GROUPS_M, dx, M_, K_, N_), dx),
            "wgrad": (lambda: mx.mx_grouped_mm_bf16(step.dy, step.x, step.offs, G_, mx.MX_GROUPS_K, dw, M_, N_, K_), dw)}
    out = {"method": f"CUDA graphs of {iters} launches, this library and torch._grouped_mm alternating over "
                     f"{rounds} rounds, median per launch"}
    try:
        lib = {"dgrad": lambda: torch._grouped_mm(step.dy, step.w, offs=step.offs, out_dtype=torch.bfloat16),
               "wgrad": lambda: torch._grouped_mm(step.dy.t(), step.x, offs=step.offs, out_dtype=torch.bfloat16)}

        def capture(fn):
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                    for _ in range(iters):
                        fn()
            torch.cuda.synchronize()
            return g

        def replay_ms(g):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b)

        for name in ("dgrad", "wgrad"):
            fn, res = ours[name]
            fn()
            same = bool(torch.equal(lib[name](), res))
            ga, gb = capture(fn), capture(lib[name])
            replay_ms(ga)
            replay_ms(gb)
            t = {0: [], 1: []}
            for r in range(rounds):
                for k in ((0, 1) if r % 2 == 0 else (1, 0)):
                    t[k].append(replay_ms((ga, gb)[k]) / iters)
            del ga, gb
            med = [sorted(v)[len(v) // 2] for v in (t[0], t[1])]
            out[name] = {"ours_tflops": round(GEMM_FLOPS / med[0] / 1e9, 1),
                         "torch_grouped_mm_tflops": round(GEMM_FLOPS / med[1] / 1e9, 1),
                         "ours_over_torch": round(med[1] / med[0], 4), "bitwise_equal": same}
    except Exception as exc:          # reported, not fatal: the comparison is context
        out["error"] = repr(exc)[:300]
    mx.mx_device_error()
    return out


def unaligned_bench(mx, device, flush, peaks):
    """The unaligned geometry: the casts of a [16384, 576] gradient (576 = 18
    blocks of 32, scale columns padded to 20; L2 flushed between iterations; the
    tensor is L2-sized, so this is reported, not graded) and the three grouped
    GEMMs at G=32, K=7168, N=2048, M=32768 with Zipf(1.2) group sizes that are
    not multiples of 128 and three empty groups (pad path; graph-replayed like
    the GEMM-only timing)."""
    import torch
    from mxfp8_block_scaled_cast_b200 import synthetic as S

    out = {}
    r, c = 16384, 576
    dy = S.sweep_tensor((r, c), seed=0, device=device)
    u8 = lambda *s: torch.empty(*s, dtype=torch.uint8, device=device)
    q, s, qt, st = u8(r, c), u8(mx.mx_scale_bytes(r, c // 32)), u8(c, r), u8(mx.mx_scale_bytes(c, r // 32))
    modes = {
        "dim0": (lambda: mx.mx_cast_dim0(dy, q, s), 2 + 1 + 1 / 32),
        "dim1": (lambda: mx.mx_cast_dim1(dy, qt, st), 2 + 1 + 1 / 32),
        "2d": (lambda: mx.mx_cast_2d(dy, q, s, qt, st), 2 + 2 + 2 / 32),
    }
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    for name, (fn, bpe) in modes.items():
        out[f"{name}_{r}x{c}_gbs"] = cast_rates(r * c * bpe, flushed_time(fn, flush), hbm)
    del dy, q, s, qt, st
    out["kva_linear_M16384_N576_K7168"] = kva_gemms(mx, device, peaks)
    step = MoEStep(mx, device, seed=0, shape=(32, 32768, 2048, 7168), problem=S.unaligned_grouped_problem)
    out["grouped_gemm_G32_K7168_N2048_M32768"] = gemm_only(mx, step, peaks)
    out["grouped_gemm_G32_K7168_N2048_M32768"]["gflop_per_launch"] = round(step.gemm_flops / 1e9, 1)
    del step
    torch.cuda.empty_cache()
    return out


def ep_fused_kernels(mx, device, flush, peaks, W=8, tokens=16384, K=4096, N=4096, seed=0, rounds=4):
    """What fusing the expert-parallel exchange into the kernels costs the kernels,
    on one GPU (prime-rl PR #3388, Overview: enable_a2a; ao PR #4705, the
    expert-parallel pipeline benchmark). W ranks of one expert each, `tokens` per
    rank spread evenly over the W experts; rank 0's view:
      dispatch  its tokens cast rowwise into the W receiving ranks' buffers (the
                scatter cast) against the same grouped cast into one send buffer;
      dispatch_dy  in backward, its dY [tokens, N] cast rowwise and columnwise
                into the W ranks' buffers against the same fused grouped cast
                into one buffer;
      combine   its expert GEMM over the groups received from the W senders,
                storing each output row into its sender's buffer, against the
                same GEMM into one output.
    Local buffers stand in for the peers' mapped buffers, so the NVLink transfer
    is not in these numbers (every run here has one GPU). Casts are timed
    in-stream after an L2 flush, GEMMs as CUDA-graph replays; each pair
    alternates over `rounds` rounds, median per variant. Both forms of each
    write the same bytes (checked)."""
    import numpy as np
    import torch
    from mxfp8_block_scaled_cast_b200 import ep, synthetic as S
    E = 1
    rng = np.random.default_rng(seed)
    counts = np.stack([rng.multinomial(tokens, np.full(W * E, 1.0 / (W * E))) for _ in range(W)])
    plan = ep.DirectPlan(W, E, 0, counts)
    ex = plan.exchange
    band = ep.scale_band_bytes(K)
    u8 = lambda n: torch.empty(int(n), dtype=torch.uint8, device=device)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    med = lambda v: sorted(v)[len(v) // 2]

    # ---- dispatch ----
    x = S.normal_bf16((ex.M, K), seed=seed, device=device)
    offs_s = torch.as_tensor(ex.offs_send(), device=device)
    recv_q = [u8(plan.recv_rows_of[d] * K) for d in range(W)]
    recv_s = [u8(plan.recv_rows_of[d] // 128 * band) for d in range(W)]
    dst_q, dst_s = plan.destinations([b.data_ptr() for b in recv_q], [b.data_ptr() for b in recv_s], K)
    one_q, one_s = u8(ex.m_cap_send * K), u8(ex.m_cap_send // 128 * band)
    cast_one = lambda: mx.mx_cast_dim0_grouped(x, offs_s, ex.m_cap_send, one_q, one_s)
    cast_scatter = lambda: mx.mx_cast_dim0_grouped_scatter(x, offs_s, ex.m_cap_send, dst_q, dst_s)
    t = {"one": [], "scatter": []}
    for r in range(rounds):
        for k in (("one", "scatter") if r % 2 == 0 else ("scatter", "one")):
            t[k].append(flushed_time(cast_one if k == "one" else cast_scatter, flush, reps=5, pairs=20, runs=7)[1])
    nbytes = ex.M * K * 2 + ex.m_cap_send * K + ex.m_cap_send // 128 * band
    pads = [ep._pad(c) for c in counts[0]]
    starts = np.concatenate([[0], np.cumsum(pads)[:-1]])
    same_cast = all(
        torch.equal(one_q[int(starts[d]) * K:int(starts[d] + pads[d]) * K],
                    recv_q[d][int(plan.dst_row[d]) * K:int(plan.dst_row[d] + pads[d]) * K]) and
        torch.equal(one_s[int(starts[d]) // 128 * band:int(starts[d] + pads[d]) // 128 * band],
                    recv_s[d][int(plan.dst_row[d]) // 128 * band:int(plan.dst_row[d] + pads[d]) // 128 * band])
        for d in range(W))
    rate = lambda sec: {"gbs": round(nbytes / sec / 1e9, 1), "frac_of_measured_hbm": round(nbytes / sec / 1e9 / hbm, 3)}
    dispatch = {"bytes_per_launch": nbytes, "one_buffer": rate(med(t["one"])),
                "scattered_to_ranks": rate(med(t["scatter"])),
                "scattered_over_one": round(med(t["one"]) / med(t["scatter"]), 4), "same_bytes": same_cast}
    del x, recv_q, recv_s, one_q, one_s

    # ---- backward dispatch: dY cast rowwise and columnwise into the W ranks' buffers ----
    dy = S.normal_bf16((ex.M, N), 0.1, seed=seed + 3, device=device)
    band_n = ep.scale_band_bytes(N)
    caps = [int(plan.recv_rows_of[d]) for d in range(W)]
    rq_ = [u8(c * N) for c in caps]
    rs_ = [u8(c // 128 * band_n) for c in caps]
    rqt = [u8(N * c) for c in caps]
    rst = [u8(mx.mx_scale_bytes(N, c // 32)) for c in caps]
    d4 = plan.destinations_2d(*[[b.data_ptr() for b in bufs] for bufs in (rq_, rs_, rqt, rst)], N)
    cm = ex.m_cap_send
    o_q, o_s, o_qt, o_st = u8(cm * N), u8(cm // 128 * band_n), u8(N * cm), u8(mx.mx_scale_bytes(N, cm // 32))
    cast2_one = lambda: mx.mx_cast_2d_grouped(dy, offs_s, cm, o_q, o_s, o_qt, o_st)
    cast2_scatter = lambda: mx.mx_cast_2d_grouped_scatter(dy, offs_s, cm, *d4)
    t = {"one": [], "scatter": []}
    for r in range(rounds):
        for k in (("one", "scatter") if r % 2 == 0 else ("scatter", "one")):
            t[k].append(flushed_time(cast2_one if k == "one" else cast2_scatter, flush, reps=5, pairs=20, runs=7)[1])
    nbytes = ex.M * N * 2 + 2 * cm * N + cm // 128 * band_n + o_st.numel()
    pads_n = [ep._pad(c) for c in counts[0]]
    starts_n = np.concatenate([[0], np.cumsum(pads_n)[:-1]])
    same_2d = all(
        torch.equal(o_q[int(starts_n[d]) * N:int(starts_n[d] + pads_n[d]) * N],
                    rq_[d][int(plan.dst_row[d]) * N:int(plan.dst_row[d] + pads_n[d]) * N]) and
        torch.equal(o_qt.view(N, cm)[:, int(starts_n[d]):int(starts_n[d] + pads_n[d])],
                    rqt[d].view(N, caps[d])[:, int(plan.dst_row[d]):int(plan.dst_row[d] + pads_n[d])])
        for d in range(W))
    dispatch_dy = {"bytes_per_launch": nbytes, "one_buffer": rate(med(t["one"])),
                   "scattered_to_ranks": rate(med(t["scatter"])),
                   "scattered_over_one": round(med(t["one"]) / med(t["scatter"]), 4), "same_bytes": same_2d}
    del dy, rq_, rs_, rqt, rst, o_q, o_s, o_qt, o_st

    # ---- combine ----
    M_recv, cap, G = ex.M_recv, ex.m_cap_recv, ex.G_recv
    offs_r = torch.as_tensor(ex.offs_recv(), device=device)
    rq, rs = mx.cast_dim0_grouped(S.normal_bf16((M_recv, K), seed=seed + 1, device=device), offs_r, cap)
    wq, wsf, _, _ = mx.cast_w32x32(S.normal_bf16((E, N, K), 0.02, seed=seed + 2, device=device), transposed=False)
    y_one = torch.empty(M_recv, N, dtype=torch.bfloat16, device=device)
    y_send = [torch.empty(int(counts[s_].sum()), N, dtype=torch.bfloat16, device=device) for s_ in range(W)]
    rows = plan.combine_destinations([b.data_ptr() for b in y_send], N)
    gemm_one = lambda: mx.mx_grouped_mm_experts(rq, rs, wq, wsf, offs_r, G, E, mx.MX_GROUPS_M, y_one, M_recv, N, K,
                                                cap)
    gemm_rows = lambda: mx.mx_grouped_mm_experts_to_rows(rq, rs, wq, wsf, offs_r, G, E, mx.MX_GROUPS_M, rows,
                                                         M_recv, N, K, cap)
    t = {"one": [], "rows": []}
    for r in range(rounds):
        for k in (("one", "rows") if r % 2 == 0 else ("rows", "one")):
            t[k].append(graph_time(gemm_one if k == "one" else gemm_rows, iters=20, runs=5))
    mx.mx_device_error()
    ends = np.cumsum(counts[:, 0])
    same_gemm = all(torch.equal(y_one[int(ends[s_] - counts[s_, 0]):int(ends[s_])], y_send[s_][:int(counts[s_, 0])])
                    for s_ in range(W))
    flops = 2 * M_recv * N * K
    combine = {"flops_per_launch": flops,
               "one_output_tflops": round(flops / med(t["one"]) / 1e12, 1),
               "rows_to_senders_tflops": round(flops / med(t["rows"]) / 1e12, 1),
               "rows_over_one": round(med(t["one"]) / med(t["rows"]), 4), "same_bytes": same_gemm}
    del rq, rs, wq, wsf, y_one, y_send
    torch.cuda.empty_cache()
    return {"ranks_emulated": W, "experts_per_rank": E, "tokens_per_rank": tokens, "K": K, "N": N,
            "method": "local buffers stand in for the peers' mapped buffers (NVLink not measured: one GPU); casts "
                      "in-stream after an L2 flush, GEMMs as CUDA-graph replays, the two forms alternating",
            "dispatch": dispatch, "dispatch_dy": dispatch_dy, "combine": combine}


def kva_gemms(mx, device, peaks, Mk=16384, Nk=576, Kk=7168):
    """The GEMMs around the 576-wide output gradient (torchtitan PR #5334, review
    thread: the KV-A projection, y [16384, 576] = x [16384, 7168] w [576, 7168]^T):
    forward (576 output columns: two full 256-column tiles and a 64-column one),
    dgrad (contraction over 576: four 128-deep K steps and a half one) and wgrad
    (576 output rows), on the pad path, each timed alone as graph replays."""
    import torch
    from mxfp8_block_scaled_cast_b200 import synthetic as S
    x, w, _ = S.linear_problem(Mk, Nk, Kk, seed=0, device=device)
    dy = S.sweep_tensor((Mk, Nk), seed=0, device=device)
    u8 = lambda *sh: torch.empty(*sh, dtype=torch.uint8, device=device)
    bf = lambda *sh: torch.empty(*sh, dtype=torch.bfloat16, device=device)
    xq, xs = u8(Mk, Kk), u8(mx.mx_scale_bytes(Mk, Kk // 32))
    xqt, xst = u8(Kk, Mk), u8(mx.mx_scale_bytes(Kk, Mk // 32))
    wq, wsf, wsd = u8(Nk, Kk), u8(mx.mx_scale_bytes(Nk, Kk // 32)), u8(mx.mx_scale_bytes(Kk, Nk // 32))
    dq, ds = u8(Mk, Nk), u8(mx.mx_scale_bytes(Mk, Nk // 32))
    dqt, dst = u8(Nk, Mk), u8(mx.mx_scale_bytes(Nk, Mk // 32))
    mx.mx_cast_2d(x, xq, xs, xqt, xst)
    mx.mx_cast_w32x32(w, wq, wsf, None, wsd)
    mx.mx_cast_2d(dy, dq, ds, dqt, dst)
    y, dx, dw = bf(Mk, Nk), bf(Mk, Kk), bf(Nk, Kk)
    calls = {
        "fwd": lambda: mx.mx_grouped_mm(xq, xs, wq, wsf, None, 1, mx.MX_GROUPS_M, y, Mk, Nk, Kk, 0),
        "dgrad": lambda: mx.mx_grouped_mm(dq, ds, wq, wsd, None, 1, mx.MX_GROUPS_M_KN, dx, Mk, Kk, Nk, 0),
        "wgrad": lambda: mx.mx_grouped_mm(dqt, dst, xqt, xst, None, 1, mx.MX_GROUPS_K, dw, Mk, Nk, Kk, 0),
    }
    flops = 2 * Mk * Nk * Kk
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP8_OVER_BF16
    out = {"gflop_per_launch": round(flops / 1e9, 1)}
    for name, fn in calls.items():
        sec = graph_time(fn, iters=50)
        tf = flops / sec / 1e12
        out[name] = {"us_per_launch": round(sec * 1e6, 1), "tflops": round(tf, 1),
                     "frac_of_measured_burst_fp8": round(tf / burst, 3), "frac_of_4500_spec": round(tf / 4500.0, 3)}
    mx.mx_device_error()
    return out


def linear_bench(mx, device, flush, peaks, reps=20, graph_steps=10):
    """MXFP8 linear forward + backward at M=4096, N=4096, K=2048 (the MXFP8Linear
    benchmark shape of ao PR #4705): y = x w^T, dx = dy w, dw = dy^T x, each step
    re-quantizing w (no cache) or reusing its cached quantization (cache hit, as in
    activation-checkpoint recompute); as separate forward and backward calls (each
    casting what it reads, w included) and as the training pair (the backward
    reusing the forward's casts of x and w, as the autograd linear does). A step is ~0.15 ms of GPU work in seven
    launches, so it is timed both as issued from Python (eager, median of
    L2-flushed repetitions, includes host submission) and as CUDA-graph replays of
    `graph_steps` steps (median of 5 replays, per step)."""
    import torch
    from mxfp8_block_scaled_cast_b200 import synthetic as S
    Ml, Nl, Kl = 4096, 4096, 2048
    x, w, dy = S.linear_problem(Ml, Nl, Kl, seed=0, device=device)
    ws = mx.linear_workspace(Ml, Nl, Kl, device)
    ws_train = mx.linear_workspace(Ml, Nl, Kl, device, train=True)
    y = torch.empty(Ml, Nl, dtype=torch.bfloat16, device=device)
    dx = torch.empty(Ml, Kl, dtype=torch.bfloat16, device=device)
    dw = torch.empty(Nl, Kl, dtype=torch.bfloat16, device=device)
    cache = mx.WeightCache()

    def step(c):
        mx.mx_linear_fwd(x, w, c, 0, y, ws)
        mx.mx_linear_bwd(dy, x, w, c, 0, dx, dw, ws)

    def train_step(c):              # the forward's casts of x and w serve the backward
        mx.mx_linear_fwd_train(x, w, c, 0, y, ws_train)
        mx.mx_linear_bwd_after_fwd(dy, w, c, 0, dx, dw, ws_train)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2] * 1e-3

    def graphed(fn):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
                for _ in range(graph_steps):
                    fn()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / graph_steps)
        ts.sort()
        del g
        return ts[2] * 1e-3

    t_nc, g_nc = timed(lambda: step(None)), graphed(lambda: step(None))
    t_hit, g_hit = timed(lambda: step(cache)), graphed(lambda: step(cache))
    tp_nc, gp_nc = timed(lambda: train_step(None)), graphed(lambda: train_step(None))
    tp_hit, gp_hit = timed(lambda: train_step(cache)), graphed(lambda: train_step(cache))
    mx.mx_device_error()
    hits = cache.stats()["hits"]
    cache.close()
    flops = 3 * 2 * Ml * Nl * Kl
    entry = lambda te, tg: {"ms_per_step_graph": round(tg * 1e3, 4), "tflops_graph": round(flops / tg / 1e12, 1),
                            "ms_per_step_eager": round(te * 1e3, 4), "tflops_eager": round(flops / te / 1e12, 1)}
    return {"shape": {"M": Ml, "N": Nl, "K": Kl}, "flops_per_step": flops,
            "no_cache": entry(t_nc, g_nc), "cache_hit": dict(entry(t_hit, g_hit), hits=hits),
            "training_pair": {"no_cache": entry(tp_nc, gp_nc), "cache_hit": entry(tp_hit, gp_hit),
                              "what": "mx_linear_fwd_train + mx_linear_bwd_after_fwd: the backward "
                                      "casts dY only (x's columnwise cast and w's quantization are the "
                                      "forward's)"}}


def override_arms(mx, step, flush, peaks):
    """Backward of the same MoE layer under the two backward overrides and
    wgrad_with_hp.

    high_precision: dX = dY_g W_g and dW_g = dY_g^T X_g as bf16 grouped GEMMs
    on the bf16 operands; dequantized: the same GEMMs on the forward's codes
    dequantized to bf16 (X from the padded dim0 codes, W from the 32x32 codes);
    wgrad_with_hp: the rowwise cast of dY and the MXFP8 dgrad, with the bf16
    wgrad. Every launch is timed after an L2 flush both in-stream (queued behind
    the flush, as inside a backward step: the figures reported) and isolated (into
    an idle stream, about 5 us of launch latency more: the *_isolated figures).
    """
    import torch

    dev = step.x.device
    dx = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dw = torch.empty(G, N, K, dtype=torch.bfloat16, device=dev)
    xd = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    wd = torch.empty(G, N, K, dtype=torch.bfloat16, device=dev)
    step.run()     # the forward codes of this step are what the dequantized arm reads
    timed = lambda fn: flushed_time(fn, flush, reps=10, pairs=20, runs=9)      # (isolated, in-stream)
    # the wgrad before the dgrad and W before X: the first launches of their kernels
    # in this program are then 3 warm-ups and a flushed launch (what the committed
    # ncu captures select with -s 3)
    i_wgrad, t_wgrad = timed(lambda: mx.mx_grouped_mm_bf16(step.dy, step.x, step.offs, G, mx.MX_GROUPS_K, dw, M, N, K))
    i_dgrad, t_dgrad = timed(lambda: mx.mx_grouped_mm_bf16(step.dy, step.w, step.offs, G, mx.MX_GROUPS_M, dx, M, K, N))
    i_dqw, t_dqw = timed(lambda: mx.mx_dequant_dim0(step.wq, step.wsf, G, N, K, wd))
    i_dqx, t_dqx = timed(lambda: mx.mx_dequant_dim0_grouped(step.xq, step.xs, step.offs, M, K, step.cap, xd))
    # wgrad_with_hp: dY cast rowwise only, the MXFP8 dgrad, and the bf16 wgrad above
    i_dyc, t_dyc = timed(lambda: mx.mx_cast_dim0_grouped(step.dy, step.offs, step.cap, step.dq, step.ds))
    i_mxd, t_mxd = timed(step.gemms()["dgrad"])
    mx.mx_device_error()
    bf16_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])     # burst: single launches
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    deq_gbs = lambda elems, sec: round(elems * (3 + 1 / 32) / sec / 1e9, 1)
    return {
        "method": "in-stream after an L2 flush (a CUDA graph of 20 flush + launch pairs minus 20 flushes, "
                  "median of 9); *_isolated: one launch into an idle stream after a flush, median of 10",
        "high_precision": {
            "backward_ms": round((t_dgrad + t_wgrad) * 1e3, 4),
            "backward_ms_isolated": round((i_dgrad + i_wgrad) * 1e3, 4),
            "dgrad_bf16_tflops": round(GEMM_FLOPS / t_dgrad / 1e12, 1),
            "wgrad_bf16_tflops": round(GEMM_FLOPS / t_wgrad / 1e12, 1),
            "frac_of_measured_bf16_burst": round(2 * GEMM_FLOPS / (t_dgrad + t_wgrad) / 1e12 / bf16_peak, 3),
        },
        "dequantized": {
            "backward_ms": round((t_dgrad + t_wgrad + t_dqx + t_dqw) * 1e3, 4),
            "backward_ms_isolated": round((i_dgrad + i_wgrad + i_dqx + i_dqw) * 1e3, 4),
            "dequant_x_gbs": deq_gbs(M * K, t_dqx),
            "dequant_w_gbs": deq_gbs(G * N * K, t_dqw),
            "dequant_x_gbs_isolated": deq_gbs(M * K, i_dqx),
            "dequant_w_gbs_isolated": deq_gbs(G * N * K, i_dqw),
            "dequant_frac_of_measured_hbm": round(deq_gbs(G * N * K, t_dqw) / hbm, 3),
        },
        "wgrad_with_hp": {
            "backward_ms": round((t_dyc + t_mxd + t_wgrad) * 1e3, 4),
            "backward_ms_isolated": round((i_dyc + i_mxd + i_wgrad) * 1e3, 4),
            "dy_dim0_cast_ms": round(t_dyc * 1e3, 4),
            "dgrad_mxfp8_tflops": round(GEMM_FLOPS / t_mxd / 1e12, 1),
            "wgrad_bf16_tflops": round(GEMM_FLOPS / t_wgrad / 1e12, 1),
        },
    }


# ------------------------------------------------------ CPU (the oracle) --
def oracle_sample(tokens=512, seed=0):
    """One bounded sample of the step on the host: one expert, `tokens` tokens.

    Runs the oracle's casts and float64 GEMMs for the forward, dgrad and wgrad
    of that slice and returns (FLOPs, seconds).
    """
    import numpy as np
    from mxfp8_block_scaled_cast_b200 import synthetic as S
    from oracle import mx_oracle as O
    x = S.bf16_bits(S.normal_bf16((tokens, K), 1.0, seed=seed))
    w = S.bf16_bits(S.normal_bf16((N, K), 0.02, seed=seed + 1))
    dy = S.bf16_bits(S.normal_bf16((tokens, N), 1e-2, seed=seed + 2))
    t0 = time.perf_counter()
    offs = np.array([tokens])
    cap = O.padded_rows_capacity(tokens, 1)
    qx, sx = O.cast_dim0_grouped(x, offs, cap)
    qw, st = O.cast_32x32(w)
    s_fwd, s_dg = O.w32_scale_views(st)
    wf = O.dequant(qw, s_fwd)
    wt = O.dequant(np.ascontiguousarray(qw.T), s_dg)
    O.mm(O.dequant(qx, sx), wf)
    qd, sd = O.cast_dim0_grouped(dy, offs, cap)
    qdt, sdt = O.cast_dim1_grouped(dy, offs, cap)
    qxt, sxt = O.cast_dim1_grouped(x, offs, cap)
    O.mm(O.dequant(qd, sd), wt)
    O.mm(O.dequant(qdt, sdt), O.dequant(qxt, sxt))
    return 3 * 2 * tokens * N * K, time.perf_counter() - t0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def blas_threads():
    """Threads of the BLAS numpy's float64 matmuls run on (None if unknown)."""
    try:
        import numpy  # noqa: F401  (loads the BLAS the oracle uses)
        from threadpoolctl import threadpool_info
        counts = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(counts) if counts else None
    except Exception:
        return None


def cpu_baseline(budget_s=12.0, tokens=512):
    flops, secs, n = 0, 0.0, 0
    while secs < budget_s:
        f, s = oracle_sample(tokens, seed=n)
        flops += f
        secs += s
        n += 1
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "blas_threads": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} x (one expert, {tokens} tokens, K=N=4096: oracle casts (single-threaded numpy) + "
                      f"float64 fwd/dgrad/wgrad (BLAS))"}


def run_reference(args, rank):
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(args.ref_tokens, seed=0)
    flops, secs = 0, 0.0
    for i in range(args.steps):
        f, s = oracle_sample(args.ref_tokens, seed=i)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "G": G, "M": M, "N": N, "K": K,
                   "sample": f"one expert, {args.ref_tokens} tokens per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "blas_threads": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{args.steps} x (one expert, {args.ref_tokens} tokens)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- main ---
def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-sweep", action="store_true", help="skip the cast bandwidth sweep")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--no-arms", action="store_true", help="skip timing the backward-override arms")
    p.add_argument("--no-linear", action="store_true", help="skip timing the MXFP8 linear")
    p.add_argument("--no-gemm-only", action="store_true", help="skip the graph-replayed GEMM-only timing")
    p.add_argument("--no-ep", action="store_true",
                   help="skip timing the expert-parallel exchange fused into the kernels (ranks emulated)")
    p.add_argument("--no-library", action="store_true",
                   help="skip the interleaved comparisons with library GEMMs (cuBLASLt MXFP8, torch bf16 grouped)")
    p.add_argument("--no-unaligned", action="store_true",
                   help="skip the unaligned geometry ([16384, 576] casts, G=32 skewed grouped GEMMs)")
    p.add_argument("--e2e-steps", type=int, default=None, help="end-to-end steps (default: --steps)")
    p.add_argument("--ref-tokens", type=int, default=512)
    args = p.parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    import torch.distributed as dist
    from mxfp8_block_scaled_cast_b200 import mx
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    mx.lib()
    dev = torch.device("cuda", local)
    start_clock_sampler(local)          # running well before any timed region
    peaks, peak_src = load_peaks()
    step = MoEStep(mx, dev, seed=0)

    for _ in range(args.warmup):
        step.run()
    mx.mx_device_error()
    torch.cuda.synchronize()

    # ---- timed region: K steps ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        start.record()
        for _ in range(args.steps):
            step.run(timed_gemms=True)
        end.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mx.mx_device_error()
    total_ms = start.elapsed_time(end)
    value, ms_per_step = aggregate(total_ms / args.steps, args.steps, world)
    gemm_ms = [a.elapsed_time(b) for a, b in step.gemm_events]
    gemm_avg_s = sum(gemm_ms) / len(gemm_ms) * 1e-3
    gemm_tflops = GEMM_FLOPS / gemm_avg_s / 1e12
    peak_kind, bf16_peak, peak_why = select_peak(total_ms, clocks.summary()["reasons"], peaks)
    fp8_peak = bf16_peak * FP8_OVER_BF16
    traffic = profile_traffic("mx_gemm_kernel_moe_G8_K4096_N4096.txt",
                              ["mxfp8_block_scaled_cast_b200/csrc/mx_gemm.cuh",
                               "mxfp8_block_scaled_cast_b200/csrc/mx_sm100.cuh"])

    # ---- end to end through the public API with host buffers ----
    # A training step's per-step host traffic: the activations X, the upstream
    # gradient dY and the routing offsets come in from pinned host memory, the
    # layer's outputs Y and dX go back; the expert weights are parameters,
    # resident in HBM (uploaded once, before the timed region), and dW stays on
    # the device for the optimizer. Two device buffer sets let the copies
    # overlap the compute: while step i runs, the inputs of step i + 1 arrive
    # and the outputs of step i - 1 leave, on their own streams (PCIe is full
    # duplex). A set's inputs are refilled once the step that read them has
    # run; a step runs once its own inputs have arrived and the outputs its
    # set held before have left.
    pin = lambda t: t.cpu().pin_memory()
    hx, hw, hdy, hoffs = pin(step.x), pin(step.w), pin(step.dy), pin(step.offs)
    sets = [step, MoEStep(mx, dev, seed=1)]
    for st_ in sets:
        st_.w.copy_(hw)
    hout = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (step.y, step.dx)] for _ in sets]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hdy, hoffs))
    d2h = sum(t.numel() * t.element_size() for t in hout[0])
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n, start_event=None):
        ev_out = [None, None]
        ev_used = [None, None]          # the last step that read each set's inputs
        for i in range(n):
            b = i % 2
            st = sets[b]
            with torch.cuda.stream(s_in):
                if start_event is not None and i == 0:
                    s_in.wait_event(start_event)
                if ev_used[b] is not None:
                    s_in.wait_event(ev_used[b])
                st.x.copy_(hx, non_blocking=True)
                st.dy.copy_(hdy, non_blocking=True)
                st.offs.copy_(hoffs, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            if ev_out[b] is not None:
                comp.wait_event(ev_out[b])
            st.run()
            ev_comp = torch.cuda.Event()
            ev_comp.record(comp)
            ev_used[b] = ev_comp
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp)
                for h, d in zip(hout[b], (st.y, st.dx)):
                    h.copy_(d, non_blocking=True)
                ev_out[b] = torch.cuda.Event()
                ev_out[b].record(s_out)
        for e in ev_out:
            if e is not None:
                comp.wait_event(e)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    e2e_steps = args.steps if args.e2e_steps is None else args.e2e_steps
    e2e_run(e2e_steps, start_event=a)
    b.record()
    torch.cuda.synchronize()
    mx.mx_device_error()
    e2e_value, _ = aggregate(a.elapsed_time(b) / e2e_steps, e2e_steps, world)
    del sets[1]

    # The linear runs first after the step: its GEMMs are short, so its figures
    # move with the power state the seconds-long GEMM replays below leave behind.
    linear = None
    if not args.no_linear:
        flush = L2Flush(dev)
        with ClockSampler(local) as lin_clocks:
            linear = linear_bench(mx, dev, flush, peaks)
        linear["clocks"] = lin_clocks.summary()
        del flush
    casts = None
    if not args.no_sweep:
        flush = L2Flush(dev)
        casts = cast_sweep(mx, dev, flush, peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        del flush
    gemm_alone = None if args.no_gemm_only else gemm_only(mx, step, peaks)
    # a library's kernel is context, measured on a single GPU only
    library = None if (args.no_library or world > 1) else library_mxfp8(mx, step, dev)
    library_hp = None if (args.no_library or world > 1) else library_bf16(mx, step)
    unaligned = None
    if not args.no_unaligned:
        flush = L2Flush(dev)
        unaligned = unaligned_bench(mx, dev, flush, peaks)
        del flush
    arms = None
    if not args.no_arms:
        flush = L2Flush(dev)
        arms = override_arms(mx, step, flush, peaks)
    ep_fused = None
    if not args.no_ep and world == 1:      # ranks emulated on one GPU: context, single-GPU runs only
        flush = L2Flush(dev)
        ep_fused = ep_fused_kernels(mx, dev, flush, peaks)
        del flush

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0
    cpu = None if (args.no_cpu or world > 1) else cpu_baseline()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": WORKLOAD, "G": G, "M": M, "N": N, "K": K, "step_flops": STEP_FLOPS,
                   "l2": "inputs 512 MB > 126 MB L2 (no flush between steps)", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "mx_gemm_kernel (fwd, dgrad, wgrad launches)",
                     "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp8_peak,
                     "peak_source": f"{peak_src} bf16 {peak_kind} {bf16_peak} x {FP8_OVER_BF16} (nominal fp8/bf16); "
                                    f"{peak_kind} because {peak_why}",
                     "frac_of_4500_spec": gemm_tflops / 4500.0, "traffic": traffic,
                     "flops_per_launch": GEMM_FLOPS, "avg_launch_ms": gemm_avg_s * 1e3},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "copied": "in: X, dY, offs; out: Y, dX (weights resident, dW left on the device)"},
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
        "casts": casts,
        "backward_overrides": arms,
        "linear": linear,
        "gemm_only": gemm_alone,
        "library_mxfp8_cublaslt": library,
        "library_bf16_grouped_mm": library_hp,
        "unaligned": unaligned,
        "ep_fused_kernels": ep_fused,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

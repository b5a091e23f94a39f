"""Benchmark of the fp16 GEMM (+bias+ReLU) path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one call of the GEMM entry point on one synthetic, HBM-resident
problem of the chosen workload (default: M = N = K = 4096 with the fused
bias+ReLU epilogue and fp16 output).  The L2 cache (126 MB) is flushed by
writing a 256 MiB buffer before every step, outside the timed kernel.

Timing: CUDA events on the launching stream around each step's launch, W
untimed warm-up steps, K timed steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, max over ranks.  `value` is the whole
job's TFLOP/s = (2 M N K x K steps x ranks) / max-over-ranks GEMM time.

With --gpus N > 1 (launched by torchrun) every rank solves its own problem of
the same size: the problems are independent, there is no collective on the
data path ("scaling": "weak").

--impl reference times the CPU oracle (fp64 triple loop, OpenMP over rows) on
a bounded row sample of the same workload, on the host cores; rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import tlg_workloads as wl  # noqa: E402

METRIC = "TFLOP/s (fp16 GEMM, fp32 acc; +bias+ReLU) and % of B200 dense FP16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "gemm_bias_relu_4096_f16"
DATASHEET_FP16_TFLOPS = 2250.0  # dense fp16 tensor peak, NVIDIA B200 datasheet
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20


KERNEL_SOURCES = ("tlg_device.cuh", "tlg_gemm_kernel.cuh")  # device code of the GEMM kernel


def strip_comments(src: str) -> str:
    """C++ source without its comments and blank lines (the device code only)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())


def kernel_source_hash() -> str:
    """Hash of the GEMM kernel's device code, comments excluded: DRAM counters recorded for
    another hash are stale."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_dense_gemm_tlg_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch recorded from an ncu capture of the current kernel sources, else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def nvsmi_id(dev) -> str:
    """nvidia-smi -i argument for a torch device (its UUID, independent of CUDA_VISIBLE_DEVICES)."""
    import torch

    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


class NvmlClockSampler:
    """Polls the SM clock, its maximum, the clock-event (throttle) reasons and the power draw
    through NVML every ~2 ms from a thread, and keeps the samples taken between mark_begin()
    and mark_end() (the timed region).  Read-only queries: no GPU setting is touched."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, uuid: str):
        import pynvml

        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.samples = []  # (t, sm_mhz, reasons bitmask, power W)
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self._thread = None

    def _poll(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((time.perf_counter(), sm, rs, pw))
            except Exception:  # pragma: no cover - a failed query just loses a sample
                pass
            time.sleep(0.002)

    def start(self):
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()

    def mark_begin(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        time.sleep(0.01)
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)
        inside = [x for x in self.samples if self.t0 is not None and self.t1 is not None
                  and self.t0 <= x[0] <= self.t1]
        if not inside and self.samples and self.t0 is not None:
            # a very short timed region: the samples nearest to it
            inside = sorted(self.samples, key=lambda x: abs(x[0] - self.t0))[:3]
        if not inside:
            return None
        mask = 0
        for x in inside:
            mask |= x[2]
        reasons = sorted(name for name, const in self.REASONS
                         if hasattr(self.nv, const) and mask & getattr(self.nv, const))
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside),
                "power_w_median": statistics.median(x[3] for x in inside),
                "window_ms": 1e3 * ((self.t1 or 0) - (self.t0 or 0)), "source": "nvml, 2 ms polling"}


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs
    (fallback when NVML cannot be loaded; 100 ms sampling)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self._thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()
        time.sleep(0.3)

    def mark_begin(self):
        pass

    def mark_end(self):
        pass

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._thread:
            self._thread.join(timeout=2)
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


def dist_setup(n_gpus: int):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def _reduce(x: float, world: int, op) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: the job is done when every rank is."""
    import torch.distributed as dist

    return _reduce(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x: float, world: int) -> float:
    import torch.distributed as dist

    return _reduce(x, world, dist.ReduceOp.SUM if world > 1 else None)


def job_throughput(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank's steps over the slowest rank's device time."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


def ms_per_step_est(per_step_ms) -> float:
    """A step's device time, for sizing a run of a given length."""
    return statistics.median(per_step_ms)


def all_workloads():
    return {**wl.WORKLOADS, **wl.EPILOGUE_WORKLOADS}


def workload_residual(w: wl.Workload, seed: int = 0):
    return wl.make_residual(w.M, w.N, w.out, seed) if w.residual else None


def oracle_rows(w: wl.Workload, A, B, bias, R, rows: int, threads: int):
    """The oracle's result for the first `rows` output rows of the workload."""
    import oracle

    if w.act is not None:
        return oracle.gemm_fused(A[:rows], B, bias=bias, act=w.act,
                                 residual=R[:rows] if R is not None else None, threads=threads)
    return oracle.gemm(A[:rows], B, bias=bias, relu=w.bias_relu, threads=threads)


def cpu_oracle_rate(w: wl.Workload, target_s: float, threads: int, A=None, B=None, bias=None, R=None):
    """Time the oracle on a row sample of the workload sized for about target_s seconds.
    Returns (TFLOP/s, rows timed, seconds)."""
    if A is None:
        A, B, bias = wl.workload_operands(w)
        R = workload_residual(w)
    # grow a row sample until it takes a tenth of the target, then scale to the target
    probe = max(1, min(w.M, threads))
    while True:
        t0 = time.perf_counter()
        oracle_rows(w, A, B, bias, R, probe, threads)
        dt = max(time.perf_counter() - t0, 1e-6)
        if dt >= target_s / 10 or probe >= w.M:
            break
        probe = min(w.M, probe * 4)
    rows = int(min(w.M, max(probe, probe * target_s / dt)))
    rows = max(1, (rows // threads) * threads) if rows >= threads else rows
    t0 = time.perf_counter()
    oracle_rows(w, A, B, bias, R, rows, threads)
    dt = time.perf_counter() - t0
    return 2.0 * rows * w.N * w.K / dt / 1e12, rows, dt


def run_reference(args, w: wl.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle

    threads = oracle.default_threads()
    A, B, bias = wl.workload_operands(w)
    R = workload_residual(w)
    # each step: a row sample sized so that warmup + steps stay within a few minutes
    per_step = max(0.5, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    _, rows, _ = cpu_oracle_rate(w, per_step, threads, A, B, bias, R)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_rows(w, A, B, bias, R, rows, threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    flops = 2.0 * rows * w.N * w.K
    total = sum(times)
    value = flops * len(times) / total / 1e12
    sample = f"{rows} of {w.M} rows of the {w.name} workload per step (all N x K), fp64 oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, None),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: wl.Workload, kcfg):
    epi = "bias_relu" if w.bias_relu else "none"
    if w.act is not None:
        epi = f"bias_{w.act}" + ("_residual (separate fp16 R, read once)" if w.residual else "")
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "out": w.out,
            "epilogue": epi, "accumulate": "f32",
            "inputs": "uniform[-1,1] fp16" if w.dist == "uniform" else "normal(0,1)*0.25 fp16",
            "l2": f"flushed before every step ({FLUSH_BYTES >> 20} MiB write, untimed)",
            "kernel_config": kcfg, "parallelism": "independent problem per GPU"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=wl.WORKLOAD_ORDER + list(wl.EPILOGUE_WORKLOADS))
    ap.add_argument("--impl", default="tlg", choices=["tlg", "reference"])
    ap.add_argument("--config", default=None, help="JSON tlg_config override (tuning sweeps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-library", action="store_true",
                    help="skip the same-box torch/cuBLAS comparison timing")
    ap.add_argument("--layout", default="NN", choices=["NN", "NT", "TN", "TT"],
                    help="op(A), op(B): T = that operand is stored transposed (tlg_gemm_op)")
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="seconds of back-to-back calls (inputs rotated over buffer sets larger than L2) "
                         "timed after the burst steps, with the SM clock sampled; 0 skips it")
    ap.add_argument("--ld-pad", type=int, default=0,
                    help="extra elements in every row stride (odd: strides TMA cannot describe; "
                         "the bench passes the workspace the size query asks for, so the call "
                         "copies such matrices into an aligned layout)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    w = all_workloads()[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch

    world, rank, local = dist_setup(args.gpus)
    import tiled_dense_gemm_tlg_b200 as tlg

    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    A, B, bias = wl.workload_operands(w, seed=rank)
    R = workload_residual(w, seed=rank)
    at, bt = args.layout[0] == "T", args.layout[1] == "T"
    if at:
        A = A.t().contiguous()  # stored K x M; the product uses its transpose
    if bt:
        B = B.t().contiguous()  # stored N x K
    def padded(x: torch.Tensor, pad: int) -> torch.Tensor:
        """x on the device as a view with row stride cols + pad."""
        if pad == 0:
            return x.to(dev)
        buf = torch.empty((x.shape[0], x.shape[1] + pad), dtype=x.dtype, device=dev)
        view = buf[:, :x.shape[1]]
        view.copy_(x)
        return view

    dA, dB = padded(A, args.ld_pad), padded(B, args.ld_pad)
    dbias = bias.to(dev) if bias is not None else None
    dR = padded(R, args.ld_pad) if R is not None else None
    dC = padded(torch.empty((w.M, w.N), dtype=torch.float32 if w.out == "f32" else torch.float16),
                args.ld_pad)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    override = json.loads(args.config) if args.config else None
    kcfg = tlg.tlg_choose_config(w.M, w.N, w.K, w.out, w.has_bias, request=override)
    # The split-K tail and the aligned copies of operands TMA cannot describe need caller
    # scratch; allocated once here, outside the timed region.
    if args.ld_pad or at or bt:
        ws_bytes = tlg.tlg_gemm_workspace_size_op(dA, dB, dC, args.layout[0], args.layout[1], w.out,
                                                  config=override)
    else:
        ws_bytes = tlg.tlg_gemm_workspace_size(w.M, w.N, w.K, w.out, w.has_bias, override)
    ws = tlg.tlg_workspace(ws_bytes, device=dev) if ws_bytes > 0 else None
    fused = w.act is not None
    plain_name = ("tlg_gemm_fused" if fused else "tlg_gemm_bias_relu_f16" if w.bias_relu else
                  ("tlg_gemm_f16f16" if w.out == "f16" else "tlg_gemm_f16f32"))
    use_op = (at or bt or args.ld_pad != 0) and not fused

    def tma_describable(x: torch.Tensor) -> bool:
        """The library's rule for a TMA operand: 16-byte base and row stride."""
        return x.data_ptr() % 16 == 0 and (x.stride(0) * x.element_size()) % 16 == 0

    # Kernels one call launches: the GEMM, plus one kernel copying whichever of A and B TMA
    # cannot describe and one copying such a C out, when the workspace holds the copies (it
    # does: its size comes from the size query that counts them).
    copies = 0
    if ws_bytes > 0 and (args.ld_pad or at or bt):
        copies = int(not (tma_describable(dA) and tma_describable(dB))) + int(not tma_describable(dC))
    launches_per_step = 1 + copies
    use_ex = (ws is not None or override is not None) and not use_op and not fused
    entry = "tlg_gemm_op" if use_op else ("tlg_gemm_ex" if use_ex else plain_name)

    def fused_step(config=None, workspace=None):
        tlg.tlg_gemm_fused(dA, dB, args.layout[0], args.layout[1], bias=dbias, activation=w.act,
                           residual=dR, C=dC, out=w.out, config=config, workspace=workspace,
                           stream=stream)

    def plain_step():
        if fused:
            fused_step()
        elif w.bias_relu:
            tlg.tlg_gemm_bias_relu_f16(dA, dB, dbias, dC, stream=stream)
        elif w.out == "f16":
            tlg.tlg_gemm_f16f16(dA, dB, dC, stream=stream)
        else:
            tlg.tlg_gemm_f16f32(dA, dB, dC, stream=stream)

    def step():
        if fused:
            fused_step(override, ws)
        elif use_op:
            tlg.tlg_gemm_op(dA, dB, args.layout[0], args.layout[1], dbias, dC, out=w.out, config=override,
                            workspace=ws, stream=stream)
        elif use_ex:
            tlg.tlg_gemm_ex(dA, dB, dbias, dC, out=w.out, config=override, workspace=ws, stream=stream)
        else:
            plain_step()

    def gemm_into(a, b, bias_, r_, c, st):
        """The timed call on one set of device buffers, on stream st."""
        if fused:
            tlg.tlg_gemm_fused(a, b, args.layout[0], args.layout[1], bias=bias_, activation=w.act,
                               residual=r_, C=c, out=w.out, config=override, workspace=ws, stream=st)
        elif use_op:
            tlg.tlg_gemm_op(a, b, args.layout[0], args.layout[1], bias_, c, out=w.out, config=override,
                            workspace=ws, stream=st)
        elif use_ex:
            tlg.tlg_gemm_ex(a, b, bias_, c, out=w.out, config=override, workspace=ws, stream=st)
        elif w.bias_relu:
            tlg.tlg_gemm_bias_relu_f16(a, b, bias_, c, stream=st)
        elif w.out == "f16":
            tlg.tlg_gemm_f16f16(a, b, c, stream=st)
        else:
            tlg.tlg_gemm_f16f32(a, b, c, stream=st)

    def new_buffer_set():
        """Another device copy of the step's operands and output, same layout."""
        return (padded(A, args.ld_pad), padded(B, args.ld_pad), bias.to(dev) if bias is not None else None,
                padded(R, args.ld_pad) if R is not None else None,
                padded(torch.empty((w.M, w.N), dtype=dC.dtype), args.ld_pad))

    def timed(fn, n):
        """Per-step device milliseconds of n calls, each after an untimed L2 flush."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        # An untimed ~1 ms spin first, outside every event pair, so the host enqueues the steps
        # ahead of the GPU: no step's interval then holds the host's per-call overhead (that
        # overhead is part of the e2e measurement below).
        torch.cuda._sleep(2_000_000)
        for i in range(n):
            flush.fill_(float(i))  # untimed: evicts A, B and C from L2
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        return [s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)]

    # The clock sampler starts before the warm-up, so the timed steps follow the warm-up
    # directly (no idle gap in which the GPU clocks down).
    try:
        clocks = NvmlClockSampler(nvsmi_id(dev))
    except Exception:
        clocks = ClockSampler(nvsmi_id(dev))
    clocks.start()
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize(dev)
    rc, code = tlg.tlg_device_error(clear=True)
    if rc != 0:
        raise SystemExit(f"device error word {code:#x} during warm-up")

    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.mark_begin()
    per_step_ms = timed(step, args.steps)
    clocks.mark_end()
    barrier(world)
    clk = clocks.stop()
    gemm_ms = sum(per_step_ms)
    rc, code = tlg.tlg_device_error(clear=True)
    if rc != 0:
        raise SystemExit(f"device error word {code:#x} during the timed steps")

    # The same steps through the plain entry point (no workspace), for comparison.
    plain = None
    if use_ex and override is None and not use_op and not fused:
        for _ in range(args.warmup):
            flush.fill_(1.0)
            plain_step()
        barrier(world)
        torch.cuda.synchronize(dev)
        plain_ms = max_over_ranks(sum(timed(plain_step, args.steps)), world)
        barrier(world)
        plain = {"call": plain_name, "value": w.flops * args.steps * world / (plain_ms * 1e-3) / 1e12,
                 "unit": UNIT, "ms_per_step": plain_ms / args.steps}

    # ---- cuBLAS on the same box, for comparison only (never part of `value`): torch.mm of the
    # same fp16 operands into a C of the workload's type, timed the same way (L2 flushed before
    # every call, CUDA events on the same stream); with a bias, also torch's own composition of
    # the workload's epilogue (addmm, the activation, the residual add: separate kernels).
    library = None
    if not args.no_library and world == 1 and not use_op:
        import torch.nn.functional as F

        Cl = torch.empty((w.M, w.N), dtype=torch.float16, device=dev)
        out32 = w.out == "f32"  # fp16 operands into an fp32 C (torch's mm with out_dtype)
        if out32:
            try:
                torch.mm(dA[:8, :8], dB[:8, :8], out_dtype=torch.float32)
            except Exception:
                out32 = False
        act = w.act if fused else ("relu" if dbias is not None else None)
        act_fn = {"relu": F.relu, "gelu": F.gelu, "silu": F.silu,
                  "gelu_tanh": lambda x: F.gelu(x, approximate="tanh"), "none": lambda x: x}

        def lib_mm():
            with torch.cuda.stream(stream):
                if out32:
                    torch.mm(dA, dB, out_dtype=torch.float32)
                else:
                    torch.mm(dA, dB, out=Cl)

        def lib_epi():
            with torch.cuda.stream(stream):
                x = act_fn[act](torch.addmm(dbias, dA, dB))
                if dR is not None:
                    x = x + dR

        def lib_time(fn, call):
            for _ in range(args.warmup):
                flush.fill_(1.0)
                fn()
            torch.cuda.synchronize(dev)
            ms = sum(timed(fn, args.steps))
            return {"call": call, "value": w.flops * args.steps / (ms * 1e-3) / 1e12, "unit": UNIT,
                    "ms_per_step": ms / args.steps}

        library = lib_time(lib_mm, "torch.mm (cuBLAS), " + ("fp32 C (out_dtype)" if out32 else "fp16 C") +
                           ", no epilogue")
        if dbias is not None and dA.dtype == torch.float16:
            library["with_epilogue"] = lib_time(
                lib_epi, f"torch.addmm + {act}" + (" + residual" if dR is not None else "") +
                f", {'fp16' if w.out == 'f16' else 'fp16 (the workload writes fp32)'} C, separate kernels")

    max_ms = max_over_ranks(gemm_ms, world)
    total_flops = w.flops * args.steps * world
    value = job_throughput(w.flops, args.steps, world, max_ms)
    ms_per_step = max_ms / args.steps

    # ---- sustained rate: the same call back to back for a few seconds, with no flush in between;
    # the inputs rotate over enough buffer sets that together they exceed the 126 MB L2, so each
    # call still reads its operands from HBM.  The SM clock is sampled over the window: under the
    # 1000 W cap a long run settles at a lower clock than the short burst above.
    sustained = None
    if args.sustained_s > 0:
        set_bytes = A.numel() * 2 + B.numel() * 2 + dC.numel() * dC.element_size() + (
            R.numel() * R.element_size() if R is not None else 0)
        sets = [(dA, dB, dbias, dR, dC)]
        while len(sets) < 8 and len(sets) * set_bytes < 3 * (126 << 20):
            sets.append(new_buffer_set())
        n = max(len(sets), int(args.sustained_s * 1e3 / max(ms_per_step_est(per_step_ms), 1e-3)))
        for i in range(len(sets)):
            gemm_into(*sets[i], stream)
        torch.cuda.synchronize(dev)
        try:
            sclk = NvmlClockSampler(nvsmi_id(dev))
        except Exception:
            sclk = ClockSampler(nvsmi_id(dev))
        sclk.start()
        barrier(world)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sclk.mark_begin()
        e0.record(stream)
        for i in range(n):
            gemm_into(*sets[i % len(sets)], stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        sclk.mark_end()
        sc = sclk.stop()
        s_ms = max_over_ranks(e0.elapsed_time(e1), world)
        rc, code = tlg.tlg_device_error(clear=True)
        if rc != 0:
            raise SystemExit(f"device error word {code:#x} during the sustained run")
        s_val = w.flops * n * world / (s_ms * 1e-3) / 1e12
        sustained = {"value": s_val, "unit": UNIT, "seconds": s_ms * 1e-3, "calls": n,
                     "buffer_sets": len(sets), "ms_per_call": s_ms / n, "clocks": sc}
        if sc:
            sustained["mcycles_per_call"] = s_ms / n * sc["sm_mhz"] * 1e-3
            sustained["frac_of_clock_peak"] = s_val / world / (148 * 8192 * sc["sm_mhz"] * 1e6 / 1e12)
        del sets

    # ---- end to end through the public API: pinned host inputs -> device -> GEMM -> pinned host output.
    # Every step copies its inputs in and its result out inside the timed region.  The steps are
    # pipelined the way a host-fed job would run them: two device buffer sets, the uploads on one
    # stream, the GEMMs on another and the downloads on a third, so step i's GEMM overlaps step
    # i+1's upload and step i-1's download (the two copy directions use separate copy engines).
    e2e = None
    if not args.no_e2e:
        hA, hB = A.pin_memory(), B.pin_memory()
        hbias = bias.pin_memory() if bias is not None else None
        hR = R.pin_memory() if R is not None else None
        hC = [torch.empty(dC.shape, dtype=dC.dtype).pin_memory() for _ in range(2)]
        h2d = hA.numel() * 2 + hB.numel() * 2 + (hbias.numel() * 2 if hbias is not None else 0)
        h2d += hR.numel() * hR.element_size() if hR is not None else 0
        d2h = hC[0].numel() * hC[0].element_size()
        bufs = [(dA, dB, dbias, dR, dC), new_buffer_set()]
        s_up, s_gemm, s_down = (torch.cuda.Stream(dev) for _ in range(3))
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("up", "gemm", "down")}
        used = [False, False]

        def e2e_step(i):
            k = i % 2
            a, b, bias_, r_, c = bufs[k]
            if used[k]:
                s_up.wait_event(ev["gemm"][k])    # step i-2's GEMM has read these inputs
            with torch.cuda.stream(s_up):
                a.copy_(hA, non_blocking=True)
                b.copy_(hB, non_blocking=True)
                if hbias is not None:
                    bias_.copy_(hbias, non_blocking=True)
                if hR is not None:
                    r_.copy_(hR, non_blocking=True)
            ev["up"][k].record(s_up)
            s_gemm.wait_event(ev["up"][k])
            if used[k]:
                s_gemm.wait_event(ev["down"][k])  # step i-2's result has been read back
            gemm_into(a, b, bias_, r_, c, s_gemm)
            ev["gemm"][k].record(s_gemm)
            s_down.wait_event(ev["gemm"][k])
            with torch.cuda.stream(s_down):
                hC[k].copy_(c, non_blocking=True)
            ev["down"][k].record(s_down)
            used[k] = True

        for i in range(3):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        s_gemm.wait_event(e0)
        s_down.wait_event(e0)
        for i in range(args.steps):
            e2e_step(3 + i)
        s_down.wait_event(ev["gemm"][(3 + args.steps - 1) % 2])
        e1.record(s_down)
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
               "pipeline": "2 buffer sets; upload, GEMM and download on three streams"}

    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))  # fp16 = bf16 rate (same nominal)
    achieved = w.flops / (statistics.mean(per_step_ms) * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                "frac": achieved / peak, "traffic": load_traffic(w.name),
                "peak_source": f"{peak_src} cuBLAS-class bf16 burst x 1.0 (fp16/bf16 nominal ratio)",
                "frac_of_datasheet_fp16": achieved / DATASHEET_FP16_TFLOPS,
                "algorithmic_flops_per_launch": w.flops, "algorithmic_bytes_per_launch": w.algorithmic_bytes}
    if clk:
        roofline["frac_of_clock_peak"] = achieved / (148 * 8192 * clk["sm_mhz"] * 1e6 / 1e12)
    if copies:
        # The step's events bracket the GEMM and its copies: the figure is the whole call's, and
        # the stored per-kernel DRAM traffic does not describe it.
        roofline["covers"] = f"the whole call: the GEMM and {copies} aligned-copy kernel(s)"
        roofline["traffic"] = None

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        import oracle

        threads = oracle.default_threads()
        rate, rows, secs = cpu_oracle_rate(w, 10.0, threads, A, B, bias, R)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} of {w.M} output rows (all N={w.N} columns, K={w.K}) in {secs:.1f} s, fp64"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": dict(workload_config(w, kcfg), entry_point=entry, workspace_bytes=ws_bytes,
                       layout=args.layout, ld_pad=args.ld_pad,
                       operand_path=(("aligned copies in the workspace, then TMA" if ws_bytes > 0
                                      else "plain loads/stores") + " (row strides not 16-byte multiples)"
                                     if (args.ld_pad * 2) % 16 else "TMA")),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "plain_entry_point": plain,
        "library_same_box": library,
        "sustained": sustained,
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clk,
        "per_step_ms": {"min": min(per_step_ms), "median": statistics.median(per_step_ms),
                        "max": max(per_step_ms), "all": [round(x, 5) for x in per_step_ms]},
        "kernel_source_hash": kernel_source_hash(),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

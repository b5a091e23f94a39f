"""The benchmark's multi-rank bookkeeping on CPU: two gloo ranks with
different per-rank times must agree on the max-over-ranks time and the
whole-job throughput (every rank's work over the slowest rank's time)."""

import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, world)
        tot = bench.sum_over_ranks(1.0, world)
        value = bench.job_throughput(2e12, 4, world, mx)
        q.put((rank, mx, tot, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_job_throughput():
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, tot, value in res:
        assert mx == 15.0 and tot == 2.0
        # 2 ranks x 4 steps x 2 TFLOP in 15 ms
        assert value == pytest.approx(2e12 * 4 * 2 / 15e-3 / 1e12)


def test_single_rank_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1e12, 10, 1, 1000.0) == pytest.approx(10.0)  # 1e13 FLOP in 1 s


def test_nvml_sampler_keeps_the_timed_window():
    # The NVML sampler's summary on synthetic samples (no GPU, no NVML calls).
    import types

    import bench

    fake = types.SimpleNamespace(nvmlClocksEventReasonSwPowerCap=0x4, nvmlClocksEventReasonHwSlowdown=0x8,
                                 nvmlClocksEventReasonHwThermalSlowdown=0x40,
                                 nvmlClocksEventReasonSwThermalSlowdown=0x20,
                                 nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80)
    s = bench.NvmlClockSampler.__new__(bench.NvmlClockSampler)
    s.nv, s.max_mhz, s._thread = fake, 1965, None
    s._stop = bench.threading.Event()
    s.samples = [(0.5, 1965, 0x0, 200.0), (1.1, 1500, 0x4, 990.0), (1.2, 1400, 0x4, 1000.0),
                 (1.3, 1600, 0x0, 900.0), (2.5, 1965, 0x0, 150.0)]
    s.t0, s.t1 = 1.0, 1.35
    out = s.stop()
    assert out["samples"] == 3 and out["sm_mhz"] == 1500 and out["reasons"] == ["sw_power_cap"]
    assert out["sm_max_mhz"] == 1965 and out["power_w_median"] == 990.0


def test_kernel_hash_ignores_comments_only():
    import bench

    code = "int f(int x) {\n  return x + 1;  // one more\n}\n/* block\n comment */\n"
    assert bench.strip_comments(code) == bench.strip_comments(code.replace("one more", "plus one"))
    assert bench.strip_comments(code) != bench.strip_comments(code.replace("x + 1", "x + 2"))
    assert "//" not in bench.strip_comments(code) and "block" not in bench.strip_comments(code)

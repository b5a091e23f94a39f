"""bench.py on the GPU: one JSON line with every key the benchmark contract names, on a short
run of the default workload (CUDA events, L2 flushed, clocks sampled, e2e through host buffers)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_default_bench_line_has_the_contract_keys():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
                          "--no-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "gemm_bias_relu_4096_f16"
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] == 2 * (2 * 4096 * 4096) + 2 * 4096
    assert e["d2h_bytes_per_step"] == 2 * 4096 * 4096
    assert d["gpu_launches"] == 3  # one GEMM per timed step
    lib = d["library_same_box"]  # cuBLAS timed the same way on the same box, for comparison
    assert lib["value"] > 0 and "torch.mm" in lib["call"] and lib["with_epilogue"]["value"] > 0
    if d["clocks"] is not None:
        assert d["clocks"]["sm_mhz"] > 0 and isinstance(d["clocks"]["reasons"], list)

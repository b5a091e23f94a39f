"""The C interface from plain C: tests/c_abi_client.c, built with gcc against include/tlg.h
and libtlg.so (no Python, no torch in the client).  The CPU test builds and links it; the
GPU test runs it on seeded inputs and compares both of its results with the oracle."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import tlg_workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "tiled_dense_gemm_tlg_b200")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_client(out_dir):
    lib = os.path.join(PKG, "libtlg.so")
    if not os.path.exists(lib):
        import importlib.util

        spec = importlib.util.spec_from_file_location("tlg_build", os.path.join(PKG, "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    exe = os.path.join(out_dir, "c_abi_client")
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c_abi_client.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
           "-L", PKG, "-ltlg", "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart",
           f"-Wl,-rpath,{PKG}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no gcc")
def test_c_client_builds_and_links(tmp_path):
    exe = build_client(str(tmp_path))
    out = subprocess.run(["ldd", exe], capture_output=True, text=True).stdout
    assert "libtlg.so" in out and "torch" not in out


@pytest.mark.gpu
def test_c_client_matches_oracle(tmp_path):
    M, N, K = 300, 264, 200
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=301)
    R = wl.make_residual(M, N, "f16", seed=301)
    import torch

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    with open(tmp_path / "in.bin", "wb") as f:
        np.array([M, N, K], dtype=np.int64).tofile(f)
        for t in (A, B, bias, R):
            bits(t).tofile(f)
    exe = build_client(str(tmp_path))
    r = subprocess.run([exe, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    out = np.fromfile(tmp_path / "out.bin", dtype=np.uint16)
    assert out.size == 2 * M * N
    c1 = oracle.f16_decode(out[:M * N]).reshape(M, N)
    c2 = oracle.f16_decode(out[M * N:]).reshape(M, N)
    ok, worst, idx = oracle.within_tolerance(c1, oracle.gemm(A, B, bias=bias, relu=True), "f16")
    assert ok, (worst, idx)
    ok, worst, idx = oracle.within_tolerance(c2, oracle.gemm_fused(A, B, bias=bias, act="gelu", residual=R), "f16")
    assert ok, (worst, idx)

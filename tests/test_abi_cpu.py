"""CPU-side checks of the C ABI: the library builds and loads, exports every
function include/tlg.h declares, and rejects bad arguments on the host before
any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib_path():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "tlg_build", os.path.join(ROOT, "tiled_dense_gemm_tlg_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def header_functions():
    src = open(os.path.join(ROOT, "include", "tlg.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tlg_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_three_entry_points():
    names = header_functions()
    for n in ("tlg_gemm_f16f32", "tlg_gemm_f16f16", "tlg_gemm_bias_relu_f16"):
        assert n in names


def test_library_exports_every_declared_function(lib_path):
    lib = ctypes.CDLL(lib_path)
    for name in header_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tlg_[a-z0-9_]+)$", out, flags=re.M))
    assert set(header_functions()) <= exported


def test_library_does_not_link_torch(lib_path):
    out = subprocess.run(["ldd", lib_path], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out


def test_binding_names_match_header(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    for name in header_functions():
        assert hasattr(tlg, name), name
    assert tlg.tlg_version() >= 100


def test_status_strings(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    for s in range(6):
        assert tlg.tlg_status_string(s).startswith("TLG_")
    assert "unknown" in tlg.tlg_status_string(99)


def test_host_side_rejections_need_no_gpu(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    lib = tlg.raw_library()
    f = lib.tlg_gemm_f16f32
    A = 1 << 20  # fake, 16-byte-aligned addresses: these checks never dereference them
    assert f(-1, 8, 8, A, 8, A, 8, A, 8, None) == tlg.TLG_ERR_INVALID_ARG
    assert f(8, 8, 8, None, 8, A, 8, A * 2, 8, None) == tlg.TLG_ERR_INVALID_ARG
    assert f(8, 8, 8, A, 7, A, 8, A * 2, 8, None) == tlg.TLG_ERR_INVALID_ARG
    assert f(8, 8, 8, A + 1, 8, A, 8, A * 2, 8, None) == tlg.TLG_ERR_ALIGNMENT  # odd address for fp16
    assert f(8, 8, 8, A, 8, A, 8, A * 2 + 2, 8, None) == tlg.TLG_ERR_ALIGNMENT  # fp32 C needs 4 bytes
    assert f(8, 8, 8, A, 8, A, 8, A + 64, 8, None) == tlg.TLG_ERR_INVALID_ARG  # C overlaps A
    assert f(0, 8, 8, None, 8, None, 8, None, 8, None) == tlg.TLG_OK  # empty: nothing to do
    assert lib.tlg_gemm_bias_relu_f16(8, 8, 8, A, 8, A, 8, None, A * 2, 8, None) == tlg.TLG_ERR_INVALID_ARG
    assert lib.tlg_gemm_ex(8, 8, 8, A, 8, A, 8, A * 3, A * 2, 8, 0, 1, None, None, 0, None) == tlg.TLG_ERR_UNSUPPORTED
    # workspace must be 256-byte aligned and must not overlap C
    assert lib.tlg_gemm_ex(8, 8, 8, A, 8, A, 8, None, A * 2, 8, 0, 0, None, A * 4 + 16, 4096, None) == tlg.TLG_ERR_ALIGNMENT
    assert lib.tlg_gemm_ex(8, 8, 8, A, 8, A, 8, None, A * 2, 8, 0, 0, None, A * 2, 4096, None) == tlg.TLG_ERR_INVALID_ARG
    assert lib.tlg_selftest_timeout(0, None) == tlg.TLG_ERR_INVALID_ARG


def test_binding_validates_shapes(lib_path):
    import torch

    import tiled_dense_gemm_tlg_b200 as tlg
    A = torch.zeros((4, 8), dtype=torch.float16)
    with pytest.raises(ValueError):
        tlg.tlg_gemm_f16f32(A, torch.zeros((9, 8), dtype=torch.float16))
    with pytest.raises(TypeError):
        tlg.tlg_gemm_f16f32(A.float(), torch.zeros((8, 8), dtype=torch.float16))
    with pytest.raises(ValueError):
        tlg.tlg_gemm_f16f32(torch.zeros((8, 4), dtype=torch.float16).t(), torch.zeros((8, 8), dtype=torch.float16))


def test_fused_epilogue_host_side_rejections(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    lib = tlg.raw_library()
    A = 1 << 20
    C = A * 2

    def call(epi, out=1, c=C, ldc=8):
        return lib.tlg_gemm_fused(8, 8, 8, 0, A, 8, 0, A, 8, ctypes.byref(epi) if epi is not None else None,
                                  c, ldc, out, None, None, 0, None)

    E = tlg.tlg_fused_epilogue
    assert call(E(None, 5, None, 0)) == tlg.TLG_ERR_INVALID_ARG          # no such activation
    assert call(E(None, -1, None, 0)) == tlg.TLG_ERR_INVALID_ARG
    assert call(E(None, 2, C + 64, 8)) == tlg.TLG_ERR_INVALID_ARG        # residual overlaps C, shifted
    assert call(E(None, 2, C, 16)) == tlg.TLG_ERR_INVALID_ARG            # same base, other stride
    assert call(E(None, 0, A * 3, 7)) == tlg.TLG_ERR_INVALID_ARG         # ldr < N
    assert call(E(None, 0, A * 3 + 1, 8)) == tlg.TLG_ERR_ALIGNMENT       # fp16 residual on an odd address
    assert call(E(None, 0, A * 3 + 2, 8), out=0) == tlg.TLG_ERR_ALIGNMENT  # fp32 residual needs 4 bytes
    assert call(E(A + 1, 0, None, 0)) == tlg.TLG_ERR_ALIGNMENT           # bias on an odd address
    assert lib.tlg_gemm_fused(8, 8, 8, 2, A, 8, 0, A, 8, None, C, 8, 1, None, None, 0, None) == tlg.TLG_ERR_INVALID_ARG
    assert lib.tlg_gemm_fused(8, 8, 8, 0, A, 8, 0, A, 8, None, C, 8, 5, None, None, 0, None) == tlg.TLG_ERR_INVALID_ARG
    # residual must not overlap a split-K workspace either
    assert lib.tlg_gemm_fused(8, 8, 8, 0, A, 8, 0, A, 8, ctypes.byref(E(None, 0, A * 4, 8)), C, 8, 1, None,
                              A * 4, 4096, None) == tlg.TLG_ERR_INVALID_ARG
    # empty shapes are fine with any valid descriptor
    assert lib.tlg_gemm_fused(0, 8, 8, 0, None, 8, 0, None, 8, ctypes.byref(E(None, 2, None, 0)), None, 8, 1,
                              None, None, 0, None) == tlg.TLG_OK


def test_extent_overflow_is_rejected_on_the_host(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    lib = tlg.raw_library()
    A = 1 << 20
    # M * ldc * 4 bytes would pass 2^64 with these sizes: refused before any address arithmetic
    assert lib.tlg_gemm_f16f32(2 ** 31 - 300, 8, 8, A, 8, A, 8, A * 4, 2 ** 36, None) == tlg.TLG_ERR_UNSUPPORTED
    assert lib.tlg_gemm_f16f32(2 ** 30, 8, 8, A, 2 ** 36, A, 8, A * 4, 8, None) == tlg.TLG_ERR_UNSUPPORTED


def test_binding_rejects_overlapping_views(lib_path):
    import torch

    import tiled_dense_gemm_tlg_b200 as tlg
    row = torch.ones((1, 8), dtype=torch.float16)
    B = torch.ones((8, 8), dtype=torch.float16)
    with pytest.raises(ValueError):
        tlg.tlg_gemm_f16f32(row.expand(4, 8), B)  # row stride 0: four copies of one row
    with pytest.raises(ValueError):
        tlg.tlg_gemm_f16f32(B, torch.ones((8, 8), dtype=torch.float16).as_strided((8, 8), (4, 1)))


def test_workspace_size_op_host_checks(lib_path):
    import tiled_dense_gemm_tlg_b200 as tlg
    lib = tlg.raw_library()
    A = 1 << 20
    n = ctypes.c_size_t(7)
    assert lib.tlg_gemm_workspace_size_op(8, 8, 8, 0, A, 8, 0, A, 8, A * 2, 8, 1, None, None) == tlg.TLG_ERR_INVALID_ARG
    assert lib.tlg_gemm_workspace_size_op(8, 8, 8, 3, A, 8, 0, A, 8, A * 2, 8, 1, None, ctypes.byref(n)) == tlg.TLG_ERR_INVALID_ARG
    assert n.value == 0
    assert lib.tlg_gemm_workspace_size_op(8, 8, 8, 0, A, 7, 0, A, 8, A * 2, 8, 1, None, ctypes.byref(n)) == tlg.TLG_ERR_INVALID_ARG
    assert lib.tlg_gemm_workspace_size_op(0, 8, 8, 0, None, 8, 0, None, 8, None, 8, 1, None, ctypes.byref(n)) == tlg.TLG_OK
    assert n.value == 0


def test_gelu_tail_coefficients_are_the_fits(lib_path):
    # The kernel's GELU tail polynomials (one per type of C) are the ones the fit script
    # beside the kernel prints, to the last float32 digit, and their degrees match.
    import importlib.util

    import numpy as np

    csrc = os.path.join(ROOT, "tiled_dense_gemm_tlg_b200", "csrc")
    spec = importlib.util.spec_from_file_location("fit_gelu_tail", os.path.join(csrc, "fit_gelu_tail.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    src = open(os.path.join(csrc, "tlg_gemm_kernel.cuh")).read()
    body = src[src.index("gelu_tail_coef(int k)"):src.index("kGeluTailDegree")]
    arrays = re.findall(r"constexpr float c\[(\d+)\] = \{([^}]*)\}", body)
    assert len(arrays) == 2
    for (n, vals), out in zip(arrays, ("f16", "f32")):  # the fp16 fit is written first
        kernel = np.array([float(v.strip().rstrip("f")) for v in vals.split(",")], dtype=np.float32)
        assert int(n) == fit.DEGREE[out] + 1 == kernel.size
        assert np.array_equal(kernel, fit.fit(out)), out
    degrees = re.search(r"kGeluTailDegree = F16 \? (\d+) : (\d+);", src)
    assert (int(degrees.group(1)), int(degrees.group(2))) == (fit.DEGREE["f16"], fit.DEGREE["f32"])


def test_gelu_tail_fits_meet_their_stated_bounds():
    # The accuracy tlg.h states for GELU, checked on the CPU with the kernel's coefficients
    # evaluated in float32 as the kernel does (Horner with fused multiply-adds), against the
    # exact form x Phi(x) from scipy's normal CDF: below 3e-7 for an fp32 C on [-8, 8];
    # within 0.15 fp16 units in the last place for an fp16 C, on every fp16 input in
    # [-16, 16] and on a dense fp32 grid (inputs after a bias add).
    import importlib.util

    import numpy as np
    from scipy.special import ndtr

    spec = importlib.util.spec_from_file_location(
        "fit_gelu_tail", os.path.join(ROOT, "tiled_dense_gemm_tlg_b200", "csrc", "fit_gelu_tail.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    x = np.linspace(-8, 8, 640001).astype(np.float32)
    ref = x.astype(np.float64) * ndtr(x.astype(np.float64))
    assert np.abs(fit.gelu_f32(x, fit.fit("f32")) - ref).max() < 3e-7
    h = np.arange(0, 65536, dtype=np.uint16).view(np.float16)
    h = h[np.isfinite(h) & (np.abs(h) <= 16)].astype(np.float32)
    c16 = fit.fit("f16")
    for pts in (h, np.linspace(-16, 16, 1000001).astype(np.float32)):
        ref = pts.astype(np.float64) * ndtr(pts.astype(np.float64))
        assert (np.abs(fit.gelu_f32(pts, c16) - ref) / fit.ulp_f16(ref)).max() < 0.15

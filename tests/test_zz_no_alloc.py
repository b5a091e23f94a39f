"""tlg_gemm_ex_noalloc: the split-K GEMM for callers that cannot allocate.

A caller that runs inside a framework owning all device memory, that works
within a memory budget fixed at start-up, or that sits on a latency-critical
path where an allocation's device-wide synchronisation is not acceptable has
no workspace to hand to tlg_gemm_ex.  tlg_gemm_ex_noalloc gives such a caller
the same split-K tail with the library's own static 16 MiB scratch array.

These tests call it through the C ABI, twice in a row on different shapes,
outputs and splits, and check each result against the existing entry point
(tlg_gemm_ex with a caller workspace and the same configuration) within the
tolerances the other GPU tests use, and against the CPU oracle.  This file is
named to run last, and it also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

import oracle
import tlg_workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def call_noalloc(tlg, A, B, bias, C, out, cfg):
    """One raw C-ABI call of tlg_gemm_ex_noalloc on device tensors (any row strides); returns
    the status."""
    lib = tlg.raw_library()
    M, K = A.shape
    N = B.shape[1]
    c = tlg.tlg_config(**cfg)
    return lib.tlg_gemm_ex_noalloc(
        M, N, K, A.data_ptr(), A.stride(0), B.data_ptr(), B.stride(0),
        bias.data_ptr() if bias is not None else None, C.data_ptr(), C.stride(0),
        tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16,
        tlg.TLG_EPI_BIAS_RELU if bias is not None else tlg.TLG_EPI_NONE,
        ctypes.byref(c), int(torch.cuda.current_stream().cuda_stream))


# two different problems, run back to back on the same static scratch
CASES = [
    # (M, N, K, out, bias_relu, config)
    (1024, 768, 1000, "f16", True, {"cta_group": 2, "block_n": 256, "split_k": 3}),
    (600, 520, 2000, "f32", False, {"cta_group": 1, "block_n": 128, "split_k": 4}),
]


def test_two_calls_in_a_row_match_the_workspace_entry_point(tlg):
    results = []
    for i, (M, N, K, out, br, cfg) in enumerate(CASES):
        A, B, bias = wl.make_operands(M, N, K, "normal025", bias=br, seed=100 + i)
        dA, dB = A.cuda(), B.cuda()
        dbias = bias.cuda() if bias is not None else None
        odt = torch.float32 if out == "f32" else torch.float16
        C = torch.full((M, N), float("nan"), dtype=odt, device="cuda")
        assert call_noalloc(tlg, dA, dB, dbias, C, out, cfg) == tlg.TLG_OK
        # the existing entry point, same configuration, with a caller workspace
        ws = tlg.tlg_workspace(tlg.tlg_gemm_workspace_size(M, N, K, out, br, cfg))
        ref_gpu = tlg.tlg_gemm_ex(dA, dB, dbias, out=out, config=cfg, workspace=ws)
        torch.cuda.synchronize()
        results.append((C.double().cpu().numpy(), ref_gpu.double().cpu().numpy(), A, B, bias, out, br))
    for got, ref_gpu, A, B, bias, out, br in results:
        ok, worst, idx = oracle.within_tolerance(got, ref_gpu, out)
        assert ok, f"vs tlg_gemm_ex: worst err/bound {worst:.3g} at {idx}"
        ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=br), out)
        assert ok, f"vs oracle: worst err/bound {worst:.3g} at {idx}"
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, hex(code)


def test_scratch_beyond_the_limit_is_rejected(tlg):
    # 4096^3 with its 68 leftover pair-tile slices needs about 17.8 MB of scratch: over 16 MiB
    M = N = K = 4096
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 2}
    assert tlg.tlg_gemm_workspace_size(M, N, K, "f16", False, cfg) > 16 << 20
    A = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    C = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
    assert call_noalloc(tlg, A, A, None, C, "f16", cfg) == tlg.TLG_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (C == 7.0).all()  # nothing was launched


def odd_stride(host: torch.Tensor, pad_value: float) -> torch.Tensor:
    """host on the device as a view whose row stride is one element longer than the row (not a
    multiple of 16 bytes, so TMA cannot describe it); the extra column holds pad_value."""
    rows, cols = host.shape
    buf = torch.full((rows, cols + 1), pad_value, dtype=host.dtype, device="cuda")
    view = buf[:, :cols]
    view.copy_(host.to("cuda"))
    return view


def test_odd_strides_put_aligned_copies_beside_the_split_scratch(tlg):
    # Every row stride odd and a forced split: the call copies A, B and C into aligned layouts
    # in the same static array, after the split partials and counters.  Two calls in a row.
    M, N, K, out = 600, 520, 2000, "f32"
    cfg = {"cta_group": 1, "block_n": 128, "split_k": 4}
    for i in range(2):
        A, B, _ = wl.make_operands(M, N, K, "normal025", bias=False, seed=200 + i)
        dA, dB = odd_stride(A, float("nan")), odd_stride(B, float("nan"))
        C = odd_stride(torch.zeros((M, N), dtype=torch.float32), float("nan"))
        C[:] = float("nan")
        assert dA.stride(0) == K + 1 and dB.stride(0) == N + 1 and C.stride(0) == N + 1
        need = tlg.tlg_gemm_workspace_size_op(dA, dB, C, "N", "N", out, config=cfg)
        assert need <= 16 << 20  # the copies fit in the static array beside the split scratch
        assert call_noalloc(tlg, dA, dB, None, C, out, cfg) == tlg.TLG_OK
        ws = tlg.tlg_workspace(need)
        ref_gpu = odd_stride(torch.zeros((M, N), dtype=torch.float32), float("nan"))
        tlg.tlg_gemm_op(dA, dB, "N", "N", None, ref_gpu, out=out, config=cfg, workspace=ws)
        torch.cuda.synchronize()
        got = C.double().cpu().numpy()
        ok, worst, idx = oracle.within_tolerance(got, ref_gpu.double().cpu().numpy(), out)
        assert ok, f"vs tlg_gemm_op with a workspace: worst err/bound {worst:.3g} at {idx}"
        ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), out)
        assert ok, f"vs oracle: worst err/bound {worst:.3g} at {idx}"
        # the padding column of C (between rows) is untouched
        pad = C.as_strided((M,), (N + 1,), storage_offset=C.storage_offset() + N)
        assert torch.isnan(pad).all()
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, hex(code)


def test_a_call_allocates_nothing(tlg):
    # Everything the calls touch exists before the first one; a warm-up call does the one-time
    # set-up (the array's address, kernel attributes).  A later call must change neither the
    # device's free memory nor torch's allocator.
    M, N, K, out = 1024, 768, 1000, "f16"
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 3}
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=True, seed=300)
    dA, dB, dbias = A.cuda(), B.cuda(), bias.cuda()
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert call_noalloc(tlg, dA, dB, dbias, C, out, cfg) == tlg.TLG_OK
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        assert call_noalloc(tlg, dA, dB, dbias, C, out, cfg) == tlg.TLG_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    ok, worst, idx = oracle.within_tolerance(C.double().cpu().numpy(),
                                             oracle.gemm(A, B, bias=bias, relu=True), out)
    assert ok, f"vs oracle: worst err/bound {worst:.3g} at {idx}"

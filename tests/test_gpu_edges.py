"""GPU edge cases through the C ABI: ragged shapes straddling every tile edge
(with NaN-filled padding and guard bands that must stay untouched), every
tile width the library builds, degenerate sizes, streams, argument errors and
the bounded-wait error path."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from gpu_util import Padded, gemm_padded

pytestmark = pytest.mark.gpu

SIZES = [1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 257]
OUTS = [("f32", False), ("f16", False), ("f16", True)]
WIDTHS = [64, 128, 256]
# every kernel variant the library builds: (CTAs per tile, tile width, ring stages)
TILES = [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)]


def tile_cfg(tile):
    return {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


@pytest.fixture(scope="module")
def lib(tlg):
    return tlg.raw_library()


def edge_cases():
    cases = []
    i = 0
    for M in SIZES:
        for N in (1, 17, 64, 129, 257):
            for K in (1, 16, 63, 65, 129, 300):
                out, br = OUTS[i % 3]
                cases.append((M, N, K, out, br, TILES[(i // 3) % len(TILES)]))
                i += 1
    return cases


@pytest.mark.parametrize("M,N,K,out,bias_relu,tile", edge_cases())
def test_ragged_edges(lib, M, N, K, out, bias_relu, tile):
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=bias_relu, seed=M * 1000003 + N * 1009 + K)
    got, guards = gemm_padded(lib, A, B, bias, out, config=tile_cfg(tile), extra=(8, 8, 4))
    assert guards, f"a write landed outside M x N, or padding was modified: {guards!r}"
    ref = oracle.gemm(A, B, bias=bias, relu=bias_relu, threads=4)
    assert np.isfinite(got).all(), "NaN padding leaked into the product"
    ok, worst, idx = oracle.within_tolerance(got, ref, out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}: got {got[idx]} ref {ref[idx]}"


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_every_tile_on_multi_tile_ragged_shape(lib, tile, out, bias_relu):
    M, N, K = 700, 520, 1000  # several tiles each way, ragged in M, N and K, many k-blocks
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=bias_relu, seed=5)
    got, guards = gemm_padded(lib, A, B, bias, out, config=tile_cfg(tile), extra=(8, 16, 8))
    assert guards, repr(guards)
    ref = oracle.gemm(A, B, bias=bias, relu=bias_relu)
    ok, worst, idx = oracle.within_tolerance(got, ref, out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("tile", [(1, 128, 6), (2, 256, 6), (2, 512, 4)])
@pytest.mark.parametrize("raster_group,max_ctas", [(1, 0), (3, 0), (64, 0), (8, 2), (8, 7)])
def test_scheduler_variants(lib, tile, raster_group, max_ctas):
    # fewer CTAs than tiles makes each CTA loop over many tiles and both TMEM accumulators
    M, N, K = 1100, 900, 333
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=6)
    cfg = dict(tile_cfg(tile), raster_group=raster_group, max_ctas=max_ctas)
    got, guards = gemm_padded(lib, A, B, None, "f32", config=cfg)
    assert guards, repr(guards)
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), "f32")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("tile", [(1, 128, 6), (2, 256, 6), (2, 512, 4)])
def test_dependent_launch_waits_for_the_previous_kernel(tlg, tile):
    # GEMM 2 reads GEMM 1's output and is launched to overlap it.  Integer
    # operands keep every value exact, so GEMM 2's expected result comes from
    # the oracle alone: C1 = A1.B1 exactly (|C1| <= 4*K1 <= 2048, exact in fp16).
    M, K1, N1, N2 = 1000, 256, 520, 392
    A1, B1, _ = wl.integer_operands(M, N1, K1, lo=-2, hi=2, seed=14)
    _, B2, _ = wl.integer_operands(1, N2, N1, lo=-1, hi=1, seed=15)
    C1_ref = oracle.gemm(A1, B1)
    assert np.abs(C1_ref).max() <= 2048
    C2_ref = oracle.gemm(oracle.f16_encode_rne(C1_ref), B2)
    cfg = {"cta_group": tile[0], "block_n": tile[1], "overlap_prev": 1}
    dA1, dB1, dB2 = A1.cuda(), B1.cuda(), B2.cuda()
    for _ in range(3):
        C1 = torch.full((M, N1), float("nan"), dtype=torch.float16, device="cuda")
        tlg.tlg_gemm_ex(dA1, dB1, C=C1, out="f16", config=cfg)
        C2 = tlg.tlg_gemm_ex(C1, dB2, out="f32", config=cfg)
        torch.cuda.synchronize()
        assert np.array_equal(C2.double().cpu().numpy(), C2_ref)


def test_transpose_identity_on_gpu(tlg):
    A, B, _ = wl.make_operands(304, 200, 136, "uniform", seed=8)  # every ld a multiple of 8
    C1 = tlg.tlg_gemm_f16f32(A.cuda(), B.cuda())
    C2 = tlg.tlg_gemm_f16f32(B.t().contiguous().cuda(), A.t().contiguous().cuda())
    torch.cuda.synchronize()
    assert torch.allclose(C1.t(), C2, atol=1e-2, rtol=2e-3)


def test_identity_and_all_ones_exact(tlg):
    B = wl.make_operands(1, 264, 264, "uniform", seed=9)[1]
    I = torch.eye(264, dtype=torch.float16)
    C = tlg.tlg_gemm_f16f32(I.cuda(), B.cuda())
    assert torch.equal(C.cpu(), B.float())
    C16 = tlg.tlg_gemm_f16f16(I.cuda(), B.cuda())
    assert torch.equal(C16.cpu(), B)
    ones = torch.ones((130, 1000), dtype=torch.float16)
    C = tlg.tlg_gemm_f16f32(ones.cuda(), torch.ones((1000, 72), dtype=torch.float16).cuda())
    assert (C == 1000.0).all()


def test_bias_only_and_negative_bias(tlg):
    M, N, K = 140, 136, 72
    bias = (torch.rand(N) - 0.5).half()
    Z = torch.zeros((M, K), dtype=torch.float16).cuda()
    B = wl.make_operands(1, N, K, "uniform", seed=10)[1].cuda()
    C = tlg.tlg_gemm_bias_relu_f16(Z, B, bias.cuda())
    assert torch.equal(C.cpu(), torch.clamp(bias.float(), min=0).half().expand(M, N))
    A = wl.make_operands(M, N, K, "uniform", seed=11)[0].cuda()
    C = tlg.tlg_gemm_bias_relu_f16(A, B, torch.full((N,), -1000.0, dtype=torch.float16).cuda())
    assert (C == 0).all()


@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_k_zero_is_empty_sum(tlg, out, bias_relu):
    M, N = 33, 40
    A = torch.empty((M, 0), dtype=torch.float16, device="cuda")
    B = torch.empty((0, N), dtype=torch.float16, device="cuda")
    bias = (torch.rand(N) - 0.5).half().cuda()
    if bias_relu:
        C = tlg.tlg_gemm_bias_relu_f16(A, B, bias)
        assert torch.equal(C, torch.clamp(bias.float(), min=0).half().expand(M, N))
    else:
        fn = tlg.tlg_gemm_f16f32 if out == "f32" else tlg.tlg_gemm_f16f16
        C = fn(A, B, torch.full((M, N), float("nan"), dtype=torch.float32 if out == "f32" else torch.float16,
                                device="cuda"))
        assert (C == 0).all()


def test_m_or_n_zero_writes_nothing(tlg):
    A = torch.ones((0, 64), dtype=torch.float16, device="cuda")
    B = torch.ones((64, 32), dtype=torch.float16, device="cuda")
    assert tlg.tlg_gemm_f16f32(A, B).shape == (0, 32)
    A = torch.ones((16, 64), dtype=torch.float16, device="cuda")
    B = torch.ones((64, 0), dtype=torch.float16, device="cuda")
    assert tlg.tlg_gemm_f16f16(A, B).shape == (16, 0)


def test_runs_on_a_side_stream(tlg):
    A, B, _ = wl.make_operands(520, 384, 256, "uniform", seed=12)
    dA, dB = A.cuda(), B.cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        C = torch.full((520, 384), float("nan"), device="cuda")
        tlg.tlg_gemm_f16f32(dA, dB, C, stream=s)
    s.synchronize()
    ok, worst, _ = oracle.within_tolerance(C.double().cpu().numpy(), oracle.gemm(A, B), "f32")
    assert ok, worst


# --------------------------------------------------------------------------- argument errors

def _call(lib, M, N, K, pa, lda, pb, ldb, pc, ldc):
    return lib.tlg_gemm_f16f32(M, N, K, pa, lda, pb, ldb, pc, ldc, None)


def test_host_pointer_is_rejected(tlg, lib):
    A = torch.ones((64, 64), dtype=torch.float16)
    B = torch.ones((64, 64), dtype=torch.float16)
    C = torch.zeros((64, 64), dtype=torch.float32)
    assert _call(lib, 64, 64, 64, A.data_ptr(), 64, B.data_ptr(), 64, C.data_ptr(), 64) == tlg.TLG_ERR_INVALID_ARG
    dA, dB = A.cuda(), B.cuda()
    assert _call(lib, 64, 64, 64, dA.data_ptr(), 64, dB.data_ptr(), 64, C.data_ptr(), 64) == tlg.TLG_ERR_INVALID_ARG
    pinned = torch.zeros((64, 64), dtype=torch.float32).pin_memory()
    assert _call(lib, 64, 64, 64, dA.data_ptr(), 64, dB.data_ptr(), 64, pinned.data_ptr(), 64) == tlg.TLG_ERR_INVALID_ARG
    with pytest.raises(tlg.TlgError):
        tlg.tlg_gemm_f16f32(A, B)  # the pitfall: CPU tensors must fail loudly, never return an empty result


def test_argument_errors(tlg, lib):
    A = torch.ones((64, 64), dtype=torch.float16, device="cuda")
    B = torch.ones((64, 64), dtype=torch.float16, device="cuda")
    C = torch.zeros((64, 64), dtype=torch.float32, device="cuda")
    pa, pb, pc = A.data_ptr(), B.data_ptr(), C.data_ptr()
    E = tlg
    assert _call(lib, -1, 64, 64, pa, 64, pb, 64, pc, 64) == E.TLG_ERR_INVALID_ARG
    assert _call(lib, 64, 64, 64, None, 64, pb, 64, pc, 64) == E.TLG_ERR_INVALID_ARG
    assert _call(lib, 64, 64, 64, pa, 63, pb, 64, pc, 64) == E.TLG_ERR_INVALID_ARG
    assert _call(lib, 64, 64, 64, pa, 64, pb, 64, pc, 60) == E.TLG_ERR_INVALID_ARG
    assert _call(lib, 64, 64, 64, pa + 1, 64, pb, 64, pc, 64) == E.TLG_ERR_ALIGNMENT  # odd fp16 address
    assert _call(lib, 64, 64, 64, pa, 64, pb, 64, pc + 2, 64) == E.TLG_ERR_ALIGNMENT  # fp32 C on 2 bytes
    # a row stride TMA cannot describe is served by the plain-load path
    assert _call(lib, 64, 64, 60, pa, 62, pb, 64, pc, 64) == E.TLG_OK
    assert _call(lib, 2 ** 31, 64, 64, pa, 64, pb, 64, pc, 64) == E.TLG_ERR_UNSUPPORTED
    # C overlapping an operand
    big = torch.zeros((256, 64), dtype=torch.float32, device="cuda")
    assert _call(lib, 64, 64, 64, big.data_ptr(), 64, pb, 64, big.data_ptr() + 1024, 64) == E.TLG_ERR_INVALID_ARG
    assert _call(lib, 64, 64, 64, pa, 64, pb, 64, pc, 64) == E.TLG_OK
    with pytest.raises(E.TlgError):
        E.tlg_gemm_ex(A, B, config={"block_n": 96})
    with pytest.raises(E.TlgError):
        E.tlg_gemm_ex(A, B, config={"cta_group": 3})
    with pytest.raises(E.TlgError):
        E.tlg_gemm_ex(A, B, config={"cta_group": 2, "block_n": 64})
    torch.cuda.synchronize()


def test_choose_config_matches_table(tlg):
    props = torch.cuda.get_device_properties(0)
    for name, w in wl.WORKLOADS.items():
        c = tlg.tlg_choose_config(w.M, w.N, w.K, w.out, w.bias_relu)
        assert c["block_n"] in (64, 128, 256, 512) and c["stages"] >= 2
        # the reported CTA count: whole groups, at most one CTA per SM
        assert 0 < c["max_ctas"] <= props.multi_processor_count and c["max_ctas"] % c["cta_group"] == 0
        # asking for exactly that configuration resolves to itself
        assert tlg.tlg_choose_config(w.M, w.N, w.K, w.out, w.bias_relu, request=c) == c


def test_timeout_path_reports_and_recovers(tlg):
    rc, _ = tlg.tlg_device_error(clear=True)
    assert rc == 0
    tlg.tlg_selftest_timeout(2000)  # a wait nothing will satisfy, limited to 2 ms
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == tlg.TLG_ERR_TIMEOUT and (code & 1) and (code & (1 << 11)), hex(code)
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0
    # the context is still usable afterwards
    A, B, _ = wl.make_operands(130, 136, 136, "uniform", seed=13)
    C = tlg.tlg_gemm_f16f32(A.cuda(), B.cuda())
    ok, _, _ = oracle.within_tolerance(C.double().cpu().numpy(), oracle.gemm(A, B), "f32")
    assert ok

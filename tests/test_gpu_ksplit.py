"""The cluster k-split through the C ABI: a cluster of 2 or 4 CTAs shares each tile's K
range and the partial sums are added, in slice order, through distributed shared memory.

Checked against the fp64 oracle on ragged multi-tile shapes with NaN guard bands, for
every output kind and epilogue; bit for bit on integer inputs; for repeatability; with
clusters that loop over several tiles (so the receive buffers are reused); at the
smallest K each split allows; and through the plain entry points, whose automatic
choice takes it for small shapes with no workspace."""

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from gpu_util import gemm_padded
from test_gpu_fused import check, run_fused

pytestmark = pytest.mark.gpu

# (tile width, CTAs per cluster along K) the library builds
KSPLITS = [(128, 2), (256, 2), (256, 4)]
OUTS = [("f32", False), ("f16", False), ("f16", True)]


def ks_cfg(bn, ks, **extra):
    return {"cta_group": 1, "block_n": bn, "k_split": ks, **extra}


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


@pytest.fixture(scope="module")
def lib(tlg):
    return tlg.raw_library()


@pytest.mark.parametrize("bn,ks", KSPLITS, ids=lambda v: str(v))
@pytest.mark.parametrize("out,bias_relu", OUTS)
@pytest.mark.parametrize("M,N,K", [(700, 520, 1000), (129, 300, 257), (256, 256, 256), (1, 1, 130)])
def test_ragged_shapes_against_the_oracle(lib, bn, ks, out, bias_relu, M, N, K):
    if (K + 63) // 64 < ks:
        pytest.skip("fewer k-blocks than CTAs in the cluster")
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=bias_relu, seed=M + 7 * N + 13 * K + ks)
    got, guards = gemm_padded(lib, A, B, bias, out, config=ks_cfg(bn, ks), extra=(8, 16, 8))
    assert guards, repr(guards)
    assert np.isfinite(got).all(), "NaN padding leaked into the product"
    ref = oracle.gemm(A, B, bias=bias, relu=bias_relu)
    ok, worst, idx = oracle.within_tolerance(got, ref, out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}: got {got[idx]} ref {ref[idx]}"


@pytest.mark.parametrize("bn,ks", KSPLITS, ids=lambda v: str(v))
@pytest.mark.parametrize("max_ctas", [0, 8, 4])
def test_integer_inputs_bit_exact_and_repeatable(lib, bn, ks, max_ctas):
    # few clusters for many tiles: each cluster loops over tiles, reusing its receive buffers
    M, N, K = 1100, 900, 333
    A, B, _ = wl.integer_operands(M, N, K, seed=17)
    cfg = ks_cfg(bn, ks, max_ctas=max_ctas) if max_ctas else ks_cfg(bn, ks)
    got1, g1 = gemm_padded(lib, A, B, None, "f32", config=cfg)
    got2, g2 = gemm_padded(lib, A, B, None, "f32", config=cfg)
    assert g1 and g2
    ref = oracle.gemm(A, B)
    assert np.array_equal(got1, ref), "integer inputs must give the exact sums"
    assert np.array_equal(got1, got2)


@pytest.mark.parametrize("bn,ks", KSPLITS, ids=lambda v: str(v))
def test_smallest_k_and_too_small_k(tlg, bn, ks):
    M, N = 300, 504  # rows of B and C stay 16-byte multiples: the TMA path
    K = 64 * ks - 8  # exactly ks k-blocks, the last ragged (rows of A stay 16-byte multiples)
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=3)
    C = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), out="f32", config=ks_cfg(bn, ks))
    torch.cuda.synchronize()
    ok, worst, idx = oracle.within_tolerance(C.double().cpu().numpy(), oracle.gemm(A, B), "f32")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"
    # fewer k-blocks than CTAs: that split is not offered
    small = 64 * (ks - 1)
    with pytest.raises(tlg.TlgError):
        tlg.tlg_gemm_ex(A[:, :small].contiguous().cuda(), B[:small].contiguous().cuda(), out="f32",
                        config=ks_cfg(bn, ks))


@pytest.mark.parametrize("bn,ks", KSPLITS, ids=lambda v: str(v))
@pytest.mark.parametrize("act", ["gelu", "silu"])
@pytest.mark.parametrize("out", ["f16", "f32"])
def test_fused_epilogue(tlg, bn, ks, act, out):
    M, N, K = 333, 520, 700
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=True, seed=29)
    R = wl.make_residual(M, N, out, seed=29)
    got, guards = run_fused(tlg, A, B, bias, act, R, out, cfg=ks_cfg(bn, ks))
    assert not guards, guards
    check(got, A, B, bias, act, R, out)
    got_in, guards = run_fused(tlg, A, B, bias, act, R, out, cfg=ks_cfg(bn, ks), inplace=True)
    assert not guards, guards
    check(got_in, A, B, bias, act, R, out)


def test_split_requests_that_do_not_combine(tlg):
    A = torch.ones((512, 512), dtype=torch.float16, device="cuda")
    # no k-split with a split-K tail, nor for tiles it is not built for
    for cfg in ({"cta_group": 1, "block_n": 256, "k_split": 2, "split_k": 2},
                {"cta_group": 1, "block_n": 64, "k_split": 2},
                {"cta_group": 2, "block_n": 256, "k_split": 2},
                {"cta_group": 1, "block_n": 128, "k_split": 4}):
        with pytest.raises(tlg.TlgError):
            tlg.tlg_gemm_ex(A, A, out="f32", config=cfg)
    with pytest.raises(tlg.TlgError):  # not built for stored transposes
        tlg.tlg_gemm_op(A, A, "T", "N", out="f32", config={"cta_group": 1, "block_n": 256, "k_split": 2})


@pytest.mark.parametrize("M,N,K", [(1024, 1024, 8192), (512, 768, 4096)])
def test_plain_entry_points_use_it_on_long_k_shapes(tlg, M, N, K):
    # the automatic choice for a shape with few tiles and a long K is a k-split, through
    # the workspace-free entry point; every output against the oracle
    cfg = tlg.tlg_choose_config(M, N, K, "f32", False)
    assert cfg["k_split"] >= 2, cfg
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=41)
    C = tlg.tlg_gemm_f16f32(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    ok, worst, idx = oracle.within_tolerance(C.double().cpu().numpy(), oracle.gemm(A, B), "f32")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, hex(code)

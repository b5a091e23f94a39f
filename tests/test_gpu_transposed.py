"""GPU parity of tlg_gemm_op: operands stored transposed (the backward
products grad_A = grad_C . B^T and grad_B = A^T . grad_C of the pages'
autograd wrapper), for every layout, kernel variant and output kind,
against the CPU oracle applied to the same matrices transposed on the host."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from gpu_util import Padded

pytestmark = pytest.mark.gpu

TILES = [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)]
LAYOUTS = [("N", "T"), ("T", "N"), ("T", "T"), ("N", "N")]
OUTS = [("f32", False), ("f16", False), ("f16", True)]


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def stored(x: torch.Tensor, trans: bool) -> torch.Tensor:
    """The matrix as the caller stores it: the operand itself, or its transpose."""
    return x.t().contiguous() if trans else x


def run_padded(tlg, A, B, bias, op_a, op_b, out, cfg, extra=8):
    """Call tlg_gemm_op on padded, NaN-guarded copies of the stored operands."""
    lib = tlg.raw_library()
    at, bt = op_a == "T", op_b == "T"
    M, K = A.shape
    N = B.shape[1]
    sa, sb = stored(A, at), stored(B, bt)
    pa = Padded(sa, sa.shape[0], sa.shape[1], torch.float16, 8, extra)
    pb = Padded(sb, sb.shape[0], sb.shape[1], torch.float16, 8, extra)
    esz = 4 if out == "f32" else 2
    pc = Padded(None, M, N, torch.float32 if out == "f32" else torch.float16, 16 // esz, 4)
    db = bias.cuda() if bias is not None else None
    c = tlg.tlg_config(**cfg)
    rc = lib.tlg_gemm_op(M, N, K, int(at), pa.ptr(), pa.ld, int(bt), pb.ptr(), pb.ld,
                         db.data_ptr() if db is not None else None, pc.ptr(), pc.ld,
                         tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16,
                         tlg.TLG_EPI_BIAS_RELU if bias is not None else tlg.TLG_EPI_NONE,
                         ctypes.byref(c), None, 0, int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    guards = {n: b.guard_changes() for n, b in (("A", pa), ("B", pb), ("C", pc)) if b.guard_changes()}
    return pc.view.double().cpu().numpy(), guards


@pytest.mark.parametrize("layout", LAYOUTS, ids=lambda l: l[0] + l[1])
@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_every_layout_and_tile_matches_oracle(tlg, layout, tile, out, bias_relu):
    M, N, K = 300, 264, 520  # ragged in M and K, several tiles
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=bias_relu, seed=tile[1] + 3 * tile[0])
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}
    got, guards = run_padded(tlg, A, B, bias, layout[0], layout[1], out, cfg)
    assert not guards, guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=bias_relu), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("layout", [("N", "T"), ("T", "N"), ("T", "T")], ids=lambda l: l[0] + l[1])
@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (17, 129, 65), (129, 17, 257), (256, 256, 8)])
def test_ragged_edges_transposed(tlg, layout, M, N, K):
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=M + N + K)
    got, guards = run_padded(tlg, A, B, None, layout[0], layout[1], "f32", {"cta_group": 1, "block_n": 64})
    assert not guards, guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), "f32")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("layout", [("N", "T"), ("T", "N"), ("T", "T")], ids=lambda l: l[0] + l[1])
def test_integer_inputs_bit_exact_transposed(tlg, layout):
    M, N, K = 1536, 1280, 3072
    A, B, _ = wl.integer_operands(M, N, K, seed=21)
    at, bt = layout[0] == "T", layout[1] == "T"
    C = tlg.tlg_gemm_op(stored(A, at).cuda(), stored(B, bt).cuda(), layout[0], layout[1], out="f32")
    torch.cuda.synchronize()
    assert np.array_equal(C.double().cpu().numpy(), oracle.gemm(A, B))


def test_backward_products(tlg):
    # forward C = A.B, then grad_A = grad_C . B^T and grad_B = A^T . grad_C with the operands
    # as the forward pass stored them
    M, N, K = 768, 640, 512
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=31)
    G = (torch.rand((M, N), generator=torch.Generator().manual_seed(33)) * 2 - 1).half()
    dA = tlg.tlg_gemm_op(G.cuda(), B.cuda(), "N", "T", out="f32")   # (M x N) . (N x K)
    dB = tlg.tlg_gemm_op(A.cuda(), G.cuda(), "T", "N", out="f32")   # (K x M) . (M x N)
    torch.cuda.synchronize()
    ok, worst, _ = oracle.within_tolerance(dA.double().cpu().numpy(), oracle.gemm(G, B.t().contiguous()), "f32")
    assert ok, worst
    ok, worst, _ = oracle.within_tolerance(dB.double().cpu().numpy(), oracle.gemm(A.t().contiguous(), G), "f32")
    assert ok, worst


def test_transposed_leading_dimension_checks(tlg):
    lib = tlg.raw_library()
    A = torch.ones((64, 128), dtype=torch.float16, device="cuda")   # stored K x M for op_a = T
    B = torch.ones((64, 64), dtype=torch.float16, device="cuda")
    C = torch.zeros((128, 64), dtype=torch.float32, device="cuda")
    # op(A) is 128 x 64: stored lda must be >= M = 128
    rc = lib.tlg_gemm_op(128, 64, 64, 1, A.data_ptr(), 64, 0, B.data_ptr(), 64, None, C.data_ptr(), 64,
                         0, 0, None, None, 0, None)
    assert rc == tlg.TLG_ERR_INVALID_ARG
    rc = lib.tlg_gemm_op(128, 64, 64, 1, A.data_ptr(), 128, 0, B.data_ptr(), 64, None, C.data_ptr(), 64,
                         0, 0, None, None, 0, None)
    assert rc == tlg.TLG_OK
    rc = lib.tlg_gemm_op(128, 64, 64, 2, A.data_ptr(), 128, 0, B.data_ptr(), 64, None, C.data_ptr(), 64,
                         0, 0, None, None, 0, None)
    assert rc == tlg.TLG_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (C == 64).all()

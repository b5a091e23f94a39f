"""Every output of the timed full-size calls against the oracle.

The benchmark times these calls on seed-0 inputs: tlg_gemm_ex with the workspace
tlg_gemm_workspace_size asks for (the automatic choice, which may cut the tiles of
the partial last wave along K), the workspace-free tlg_gemm_bias_relu_f16 it reports
beside it, tlg_gemm_fused with bias + GELU + residual, and the 8192^3 fp16 product.
Each result is compared element by element with the fp64 oracle over the whole
output, within the tolerance of its output type: the pages check a tiled GEMM
against a reference output element by element ("tilelang operator-compilation
walkthrough", lqnn.cn/news/222844, section 4.3; "TileLang tile-level language
overview", pwwt.cn/news/4964011, section 4.3 FAQ).  The oracle takes a few seconds
at 4096^3 and about half a minute at 8192^3 on the host cores.
"""

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def assert_full(got: torch.Tensor, ref: np.ndarray, out: str, what: str):
    g = got.double().cpu().numpy()
    assert g.shape == ref.shape
    ok, worst, idx = oracle.within_tolerance(g, ref, out)
    assert ok, f"{what}: worst err/bound {worst:.3g} at {idx}"


def test_bias_relu_4096_timed_calls_every_output(tlg):
    w = wl.WORKLOADS["gemm_bias_relu_4096_f16"]
    A, B, bias = wl.workload_operands(w)
    dA, dB, db = A.cuda(), B.cuda(), bias.cuda()
    nbytes = tlg.tlg_gemm_workspace_size(w.M, w.N, w.K, w.out, True)
    ws = tlg.tlg_workspace(nbytes) if nbytes > 0 else None
    timed = tlg.tlg_gemm_ex(dA, dB, db, out=w.out, workspace=ws)
    plain = tlg.tlg_gemm_bias_relu_f16(dA, dB, db)
    torch.cuda.synchronize()
    ref = oracle.gemm(A, B, bias=bias, relu=True)
    assert_full(timed, ref, w.out, f"tlg_gemm_ex, workspace {nbytes} B")
    assert_full(plain, ref, w.out, "tlg_gemm_bias_relu_f16")
    if ws is not None:
        assert int(ws[:4096].count_nonzero()) == 0  # split counters left ready for the next call


@pytest.mark.parametrize("inplace", [False, True])
def test_bias_gelu_residual_4096_timed_call_every_output(tlg, inplace):
    w = wl.EPILOGUE_WORKLOADS["gemm_bias_gelu_residual_4096_f16"]
    A, B, bias = wl.workload_operands(w)
    R = wl.make_residual(w.M, w.N, w.out)
    dR = R.cuda()
    nbytes = tlg.tlg_gemm_workspace_size(w.M, w.N, w.K, w.out, True)
    ws = tlg.tlg_workspace(nbytes) if nbytes > 0 else None
    got = tlg.tlg_gemm_fused(A.cuda(), B.cuda(), bias=bias.cuda(), activation=w.act, residual=dR,
                             C=dR if inplace else None, out=w.out, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.gemm_fused(A, B, bias=bias, act=w.act, residual=R)
    assert_full(got, ref, w.out, f"tlg_gemm_fused, in place {inplace}")


def test_gemm_8192_timed_call_every_output(tlg):
    w = wl.WORKLOADS["gemm_8192_f16"]
    A, B, _ = wl.workload_operands(w)
    got = tlg.tlg_gemm_f16f16(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    assert_full(got, oracle.gemm(A, B), w.out, "tlg_gemm_f16f16 8192^3")

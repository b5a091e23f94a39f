"""Special values and long tile sequences through the epilogue, against the fp64 oracle.

NaN: with A = I, a NaN in B makes its whole output column NaN before the epilogue
(0 * NaN = NaN in every row's sum).  The oracle's ReLU is max(x, 0) taken as
"x > 0 ? x : 0", which maps NaN to 0; GELU, SiLU and tanh-GELU of NaN are NaN.
The kernels must agree: the bias + ReLU build applies ReLU after packing to fp16,
the general epilogue in fp32, and GELU keeps NaN through its clamp of |x|.

Bias across many tiles: a launch limited to one unit walks every tile of the
output in turn, so the tile's bias (kept in shared memory by the epilogue warps
where the plan has room, else spread over the lanes) is replaced once per tile.
Integer operands, bias and residual keep every sum exact, so those results are
compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl

pytestmark = pytest.mark.gpu

TILES = [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)]


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def nan_operands(n: int = 96, col: int = 5, row: int = 3, seed: int = 1):
    A = torch.eye(n, dtype=torch.float16)
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    B = (torch.randn(n, n, generator=g) * 2).half()
    B[row, col] = float("nan")
    bias = ((torch.rand(n, generator=g) - 0.5)).half()
    return A, B, bias, col


def same_nans_and_values(got: np.ndarray, ref: np.ndarray, out: str):
    assert np.array_equal(np.isnan(got), np.isnan(ref)), (
        f"NaN positions differ: kernel {np.argwhere(np.isnan(got))[:4].tolist()}, "
        f"oracle {np.argwhere(np.isnan(ref))[:4].tolist()}")
    keep = ~np.isnan(ref)
    ok, worst, idx = oracle.within_tolerance(got[keep], ref[keep], out)
    assert ok, f"worst err/bound {worst:.3g}"


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("act", ["none", "relu", "gelu", "silu", "gelu_tanh"])
def test_nan_through_every_activation(tlg, act, out):
    A, B, bias, col = nan_operands()
    got = tlg.tlg_gemm_fused(A.cuda(), B.cuda(), bias=bias.cuda(), activation=act, out=out)
    torch.cuda.synchronize()
    g = got.double().cpu().numpy()
    ref = oracle.gemm_fused(A, B, bias=bias, act=act)
    same_nans_and_values(g, ref, out)
    if act == "relu":
        assert np.all(g[:, col] == 0.0)
    else:
        assert np.all(np.isnan(g[:, col]))


@pytest.mark.parametrize("tile", TILES, ids=lambda t: f"{t[0]}x{t[1]}")
def test_nan_through_bias_relu_build(tlg, tile):
    A, B, bias, col = nan_operands()
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}
    got = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), bias.cuda(), out="f16", config=cfg)
    torch.cuda.synchronize()
    g = got.double().cpu().numpy()
    ref = oracle.gemm(A, B, bias=bias, relu=True)
    same_nans_and_values(g, ref, "f16")
    assert np.all(g[:, col] == 0.0)  # ReLU(NaN) = 0, as in the oracle


PLAIN_LOAD_TILES = [(1, 64, 8), (2, 256, 6)]  # the tiles built with plain-load warps too


@pytest.mark.parametrize("tile,N", [(t, 1096) for t in TILES] + [(t, 1100) for t in PLAIN_LOAD_TILES],
                         ids=lambda v: f"{v[0]}x{v[1]}" if isinstance(v, tuple) else f"N{v}")
def test_bias_replaced_every_tile_of_one_unit(tlg, tile, N):
    # One work unit (a CTA or a pair) computes all of a ragged multi-tile output.  N = 1100
    # makes B's row stride 2200 bytes, which TMA cannot describe: with no workspace for an
    # aligned copy, the plain-load warps feed the same epilogue.
    M, K = 700, 200
    A, B, bias = wl.integer_operands(M, N, K, seed=31, bias=True)
    R = wl.integer_operands(M, N, 1, seed=32)[0].float().reshape(M, 1).expand(M, N).half().contiguous()
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2], "max_ctas": tile[0]}
    dA, dB, db = A.cuda(), B.cuda(), bias.cuda()
    relu = tlg.tlg_gemm_ex(dA, dB, db, out="f16", config=cfg)
    fused = tlg.tlg_gemm_fused(dA, dB, bias=db, activation="none", residual=R.cuda(), out="f16",
                               config=cfg)
    torch.cuda.synchronize()
    assert np.array_equal(relu.double().cpu().numpy(), oracle.gemm(A, B, bias=bias, relu=True))
    assert np.array_equal(fused.double().cpu().numpy(),
                          oracle.gemm_fused(A, B, bias=bias, act="none", residual=R))
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, hex(code)

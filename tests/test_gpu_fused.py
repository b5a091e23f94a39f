"""GPU parity of tlg_gemm_fused, the general fused epilogue
C = act(op(A).op(B) + bias[col]) + R[row, col] ("domestic-GPU TileLang
adoption" section 4.1: activation and residual connection fused into the GEMM;
section 4.2: the bias by output column, before the activation), against the
CPU oracle on the same seeded inputs.

Tolerance: the plain GEMM's (fp32 C: 1e-2 + 2e-3 |ref|; fp16 C: 2e-2 +
1e-2 |ref|).  The epilogue adds at most a few fp32 roundings (bias add, the
fp32 erf of GELU within a few ulp, the residual add) and GELU's slope is at
most 1.13, so the accumulation error the bound was derived for still
dominates.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from gpu_util import Padded

pytestmark = pytest.mark.gpu

TILES = [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)]
ACTS = ["none", "relu", "gelu", "silu", "gelu_tanh"]


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def stored(x: torch.Tensor, trans: bool) -> torch.Tensor:
    return x.t().contiguous() if trans else x


def run_fused(tlg, A, B, bias, act, R, out, cfg=None, op_a="N", op_b="N", extra=(8, 8, 4, 4),
              inplace=False, workspace=None, align=None):
    """tlg_gemm_fused on padded, NaN-guarded device copies.  R: host residual
    (C's type) or None; inplace: R is written into C's buffer and passed as C.
    align: row-stride alignment in elements of (A, B, C, R); the default keeps
    every stride 16-byte aligned.  Returns (C as float64 numpy, guard changes)."""
    lib = tlg.raw_library()
    at, bt = op_a == "T", op_b == "T"
    M, K = A.shape
    N = B.shape[1]
    sa, sb = stored(A, at), stored(B, bt)
    cdt = torch.float32 if out == "f32" else torch.float16
    esz = 4 if out == "f32" else 2
    al = align or (8, 8, 16 // esz, 16 // esz)
    pa = Padded(sa, sa.shape[0], sa.shape[1], torch.float16, al[0], extra[0])
    pb = Padded(sb, sb.shape[0], sb.shape[1], torch.float16, al[1], extra[1])
    pc = Padded(R if inplace else None, M, N, cdt, al[2], extra[2])
    pr = None
    if R is not None and not inplace:
        pr = Padded(R, M, N, cdt, al[3], extra[3])
    db = bias.cuda() if bias is not None else None
    epi = tlg.tlg_fused_epilogue(db.data_ptr() if db is not None else None,
                                 {"none": 0, "relu": 1, "gelu": 2, "silu": 3, "gelu_tanh": 4}[act], None, 0)
    if inplace:
        epi.residual, epi.ldr = pc.ptr(), pc.ld
    elif pr is not None:
        epi.residual, epi.ldr = pr.ptr(), pr.ld
    c = tlg.tlg_config(**cfg) if cfg else None
    rc = lib.tlg_gemm_fused(M, N, K, int(at), pa.ptr(), pa.ld, int(bt), pb.ptr(), pb.ld,
                            ctypes.byref(epi), pc.ptr(), pc.ld,
                            tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16,
                            ctypes.byref(c) if c is not None else None,
                            workspace.data_ptr() if workspace is not None else None,
                            workspace.numel() if workspace is not None else 0,
                            int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    bufs = [("A", pa), ("B", pb), ("C", pc)] + ([("R", pr)] if pr is not None else [])
    guards = {n: b.guard_changes() for n, b in bufs if b.guard_changes()}
    if pr is not None:  # the residual is only read
        assert torch.equal(pr.view.cpu(), R), "residual buffer was modified"
    return pc.view.double().cpu().numpy(), guards


def check(got, A, B, bias, act, R, out):
    ref = oracle.gemm_fused(A, B, bias=bias, act=act, residual=R)
    ok, worst, idx = oracle.within_tolerance(got, ref, out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}: got {got[idx]}, ref {ref[idx]}"


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("tile", TILES, ids=lambda t: f"{t[0]}x{t[1]}")
def test_every_tile_and_activation(tlg, tile, act, out):
    M, N, K = 300, 600, 136  # ragged in M, N and K; several tiles of every shape
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=True, seed=tile[1] + tile[0])
    R = wl.make_residual(M, N, out, seed=tile[1])
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}
    got, guards = run_fused(tlg, A, B, bias, act, R, out, cfg)
    assert not guards, guards
    check(got, A, B, bias, act, R, out)


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("residual", ["none", "separate", "inplace"])
@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("with_bias", [False, True], ids=["nobias", "bias"])
def test_every_combination(tlg, with_bias, act, residual, out):
    M, N, K = 257, 333, 200
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=with_bias, seed=7)
    R = wl.make_residual(M, N, out, seed=7) if residual != "none" else None
    got, guards = run_fused(tlg, A, B, bias, act, R, out, inplace=residual == "inplace")
    assert not guards, guards
    check(got, A, B, bias, act, R, out)


@pytest.mark.parametrize("layout", [("N", "T"), ("T", "N"), ("T", "T")], ids=lambda l: l[0] + l[1])
@pytest.mark.parametrize("tile", [(1, 128, 6), (2, 256, 6), (2, 512, 4)], ids=lambda t: f"{t[0]}x{t[1]}")
def test_transposed_operands(tlg, layout, tile):
    M, N, K = 300, 520, 264
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=True, seed=41)
    R = wl.make_residual(M, N, "f16", seed=41)
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}
    got, guards = run_fused(tlg, A, B, bias, "gelu", R, "f16", cfg, op_a=layout[0], op_b=layout[1],
                            inplace=True)
    assert not guards, guards
    check(got, A, B, bias, "gelu", R, "f16")


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("what", ["operands", "residual", "C", "all"])
def test_strides_tma_cannot_describe(tlg, what, out):
    # Odd leading dimensions (and so bases off 16 bytes past the first row):
    # operands go through the plain-load warps, the residual through scalar
    # loads, C through plain stores.
    M, N, K = 200, 300, 150
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=53)
    R = wl.make_residual(M, N, out, seed=53)
    esz = 4 if out == "f32" else 2
    al = [8, 8, 16 // esz, 16 // esz]
    ex = [8, 8, 4, 4]
    if what in ("operands", "all"):
        al[0], al[1], ex[0], ex[1] = 1, 1, 3, 5
    if what in ("residual", "all"):
        al[3], ex[3] = 1, 3
    if what in ("C", "all"):
        al[2], ex[2] = 1, 1
    got, guards = run_fused(tlg, A, B, bias, "gelu", R, out, extra=tuple(ex), align=tuple(al))
    assert not guards, guards
    check(got, A, B, bias, "gelu", R, out)


@pytest.mark.parametrize("inplace", [False, True])
def test_split_k_tail_with_residual(tlg, inplace):
    M, N, K = 1024, 768, 1024  # 12 pair tiles, each cut into 4 k-slices
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=61)
    R = wl.make_residual(M, N, "f16", seed=61)
    cfg = {"cta_group": 2, "block_n": 256, "stages": 6, "split_k": 4}
    nbytes = tlg.tlg_gemm_workspace_size(M, N, K, "f16", True, cfg)
    assert nbytes > 0
    ws = tlg.tlg_workspace(nbytes)
    got, guards = run_fused(tlg, A, B, bias, "gelu", R, "f16", cfg, inplace=inplace, workspace=ws)
    assert not guards, guards
    check(got, A, B, bias, "gelu", R, "f16")
    assert int(ws[:4096].count_nonzero()) == 0  # counters left zero for the next call


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("inplace", [False, True])
def test_empty_sum(tlg, inplace, out):
    # K == 0: C = act(bias) + R
    M, N = 70, 90
    A = torch.empty((M, 0), dtype=torch.float16)
    B = torch.empty((0, N), dtype=torch.float16)
    _, _, bias = wl.make_operands(1, N, 1, bias=True, seed=3)
    R = wl.make_residual(M, N, out, seed=3)
    got, guards = run_fused(tlg, A, B, bias, "gelu", R, out, inplace=inplace)
    assert not guards, guards
    check(got, A, B, bias, "gelu", R, out)


def test_bias_relu_descriptor_matches_bias_relu_entry_point_bit_for_bit(tlg):
    M, N, K = 640, 768, 512
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=71)
    dA, dB, db = A.cuda(), B.cuda(), bias.cuda()
    c1 = tlg.tlg_gemm_bias_relu_f16(dA, dB, db)
    c2 = tlg.tlg_gemm_fused(dA, dB, bias=db, activation="relu", out="f16")
    c3 = tlg.tlg_gemm_f16f16(dA, dB)
    c4 = tlg.tlg_gemm_fused(dA, dB, out="f16")  # empty epilogue: the plain product
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    assert torch.equal(c3, c4)


def test_binding_in_place_residual(tlg):
    # the Python binding with residual=C: a residual connection updated in place
    M, N, K = 512, 384, 256
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=81)
    R = wl.make_residual(M, N, "f16", seed=81)
    C = R.cuda().clone()
    out = tlg.tlg_gemm_fused(A.cuda(), B.cuda(), bias=bias.cuda(), activation="gelu", residual=C, C=C)
    torch.cuda.synchronize()
    assert out.data_ptr() == C.data_ptr()
    check(C.double().cpu().numpy(), A, B, bias, "gelu", R, "f16")


@pytest.mark.parametrize("inplace", [False, True])
def test_full_size_sampled(tlg, inplace):
    # the bias + GELU + residual workload at 4096^3 in the launch configuration
    # the benchmark times (automatic), checked at sampled positions
    w = wl.EPILOGUE_WORKLOADS["gemm_bias_gelu_residual_4096_f16"]
    A, B, bias = wl.workload_operands(w)
    R = wl.make_residual(w.M, w.N, w.out)
    dR = R.cuda()
    C = dR if inplace else None
    got = tlg.tlg_gemm_fused(A.cuda(), B.cuda(), bias=bias.cuda(), activation=w.act, residual=dR, C=C,
                             out=w.out)
    torch.cuda.synchronize()
    rows, cols = wl.sample_positions(w.M, w.N, w.sample)
    ref = oracle.gemm_at_fused(A, B, rows.numpy(), cols.numpy(), bias=bias, act=w.act, residual=R)
    g = got.double().cpu().numpy()[rows.numpy(), cols.numpy()]
    ok, worst, idx = oracle.within_tolerance(g, ref, w.out)
    assert ok, f"worst err/bound {worst:.3g} at sample {idx}"
    assert np.isfinite(got.float().cpu().numpy()).all()


def test_gelu_matches_exact_form_pointwise(tlg):
    # A = I: C = gelu(B + bias) exactly at fp16 points in [-6, 6]; the kernel's
    # fp32 GELU must stay within a few fp32 ulp of the fp64 oracle (before the
    # fp32 store), far inside the GEMM tolerance.
    N = 1024
    x = torch.linspace(-6, 6, 64 * N).reshape(64, N).half()
    A = torch.eye(64, dtype=torch.float16)
    got = tlg.tlg_gemm_fused(A.cuda(), x.cuda(), activation="gelu", out="f32")
    torch.cuda.synchronize()
    ref = oracle.gemm_fused(A, x, act="gelu")
    err = np.abs(got.double().cpu().numpy() - ref)
    assert err.max() <= 1e-6 * (1 + np.abs(ref).max()), err.max()


def _ulp_f16(v: np.ndarray) -> np.ndarray:
    """The fp16 unit in the last place at |v| (the subnormal spacing below 2^-14)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -14)))
    return 2.0 ** (e - 10)


def test_gelu_fp16_output_within_a_fraction_of_an_ulp(tlg):
    # A = I: C = gelu(B) rounded to fp16, for every fp16 value B in [-16, 16] (fp16
    # subnormals included).  Before the rounding the kernel's GELU is within 0.15 fp16
    # units in the last place of the exact form, so each stored result lies within
    # 0.65 units of the fp64 oracle (a correct rounding alone allows 0.5).
    h = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.float16)
    h = h[torch.isfinite(h) & (h.abs() <= 16)]
    N = 640
    assert h.numel() <= 64 * N
    x = torch.zeros(64 * N, dtype=torch.float16)
    x[: h.numel()] = h
    x = x.reshape(64, N)
    A = torch.eye(64, dtype=torch.float16)
    got = tlg.tlg_gemm_fused(A.cuda(), x.cuda(), activation="gelu", out="f16")
    torch.cuda.synchronize()
    ref = oracle.gemm_fused(A, x, act="gelu")
    err_ulp = np.abs(got.double().cpu().numpy() - ref) / _ulp_f16(ref)
    worst = np.unravel_index(int(np.argmax(err_ulp)), err_ulp.shape)
    assert err_ulp.max() <= 0.65, (err_ulp.max(), float(x[worst]))
    # With a bias the activation's input x + bias is an fp32 value between the fp16 points;
    # the bound is the same (the fit holds on every fp32 input, not only fp16 ones).
    bias = (torch.arange(N, dtype=torch.float32) % 7 - 3).mul(0.1).half()
    got = tlg.tlg_gemm_fused(A.cuda(), x.cuda(), bias=bias.cuda(), activation="gelu", out="f16")
    torch.cuda.synchronize()
    ref = oracle.gemm_fused(A, x, bias=bias, act="gelu")
    err_ulp = np.abs(got.double().cpu().numpy() - ref) / _ulp_f16(ref)
    worst = np.unravel_index(int(np.argmax(err_ulp)), err_ulp.shape)
    assert err_ulp.max() <= 0.65, (err_ulp.max(), float(x[worst]), float(bias[worst[1]]))


def test_argument_errors_on_device(tlg):
    lib = tlg.raw_library()
    A = torch.ones((64, 64), dtype=torch.float16, device="cuda")
    C = torch.zeros((64, 64), dtype=torch.float16, device="cuda")
    host_r = torch.zeros((64, 64), dtype=torch.float16)
    E = tlg.tlg_fused_epilogue
    st = int(torch.cuda.current_stream().cuda_stream)

    def call(epi):
        return lib.tlg_gemm_fused(64, 64, 64, 0, A.data_ptr(), 64, 0, A.data_ptr(), 64, ctypes.byref(epi),
                                  C.data_ptr(), 64, 1, None, None, 0, st)

    assert call(E(None, 0, host_r.data_ptr(), 64)) == tlg.TLG_ERR_INVALID_ARG  # host residual
    assert call(E(None, 0, C.data_ptr() + 2 * 64, 64)) == tlg.TLG_ERR_INVALID_ARG  # shifted overlap with C
    assert call(E(None, 7, None, 0)) == tlg.TLG_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        tlg.tlg_gemm_fused(A, A, residual=torch.zeros((64, 64), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        tlg.tlg_gemm_fused(A, A, activation="tanh")
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
def test_sigmoid_form_activations_pointwise(tlg, act):
    # A = I: C = act(B) at fp16 points in [-12, 12]; fp32 results within a few fp32 ulp-scale
    # errors of the fp64 definitions
    N = 1024
    x = torch.linspace(-12, 12, 64 * N).reshape(64, N).half()
    A = torch.eye(64, dtype=torch.float16)
    got = tlg.tlg_gemm_fused(A.cuda(), x.cuda(), activation=act, out="f32")
    torch.cuda.synchronize()
    ref = oracle.gemm_fused(A, x, act=act)
    err = np.abs(got.double().cpu().numpy() - ref)
    assert err.max() <= 2e-6 * (1 + np.abs(ref).max()), err.max()

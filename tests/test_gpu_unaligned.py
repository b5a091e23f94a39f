"""GPU parity of the paths for operands the TMA unit cannot describe: row
strides that are not multiples of 16 bytes, and base addresses that are only
element-aligned.  A and B then go through the plain-load loader warps, C
through predicated plain stores, and the bias through scalar loads; the
tensor-core pipeline is the same.  Every case is checked against the CPU
oracle, with guard bands around each stored matrix that must stay untouched."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl

pytestmark = pytest.mark.gpu

PLAIN_TILES = [(1, 64, 8), (2, 256, 6)]
OUTS = [("f32", False), ("f16", False), ("f16", True)]
POISON = {torch.float16: 0x7E01, torch.float32: 0x7FC00001}  # NaN bit patterns


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


class Raw:
    """rows x cols stored with row stride ld, starting `offset` elements into a NaN-filled buffer."""

    def __init__(self, host, rows, cols, ld, dtype, offset=0):
        self.rows, self.cols, self.ld, self.dtype, self.offset = rows, cols, ld, dtype, offset
        ityp = torch.int16 if dtype == torch.float16 else torch.int32
        total = offset + rows * ld + 64
        self.bits = torch.full((total,), POISON[dtype], dtype=ityp, device="cuda")
        self.buf = self.bits.view(dtype)
        if host is not None:
            view = self.buf[offset:offset + rows * ld].view(rows, ld)[:, :cols]
            view.copy_(host.to("cuda"))

    def ptr(self):
        return self.buf.data_ptr() + self.offset * self.buf.element_size()

    def matrix(self):
        return self.buf[self.offset:self.offset + self.rows * self.ld].view(self.rows, self.ld)[:, :self.cols]

    def guard_ok(self):
        mask = torch.ones_like(self.bits, dtype=torch.bool)
        mask[self.offset:self.offset + self.rows * self.ld].view(self.rows, self.ld)[:, :self.cols] = False
        return bool((self.bits[mask] == POISON[self.dtype]).all().item())


def run(tlg, A, B, bias, out, cfg=None, ld_extra=(1, 1, 1), offsets=(0, 0, 0), bias_offset=0,
        op=("N", "N")):
    lib = tlg.raw_library()
    at, bt = op[0] == "T", op[1] == "T"
    M, K = A.shape
    N = B.shape[1]
    sa = A.t().contiguous() if at else A
    sb = B.t().contiguous() if bt else B
    ra = Raw(sa, sa.shape[0], sa.shape[1], sa.shape[1] + ld_extra[0], torch.float16, offsets[0])
    rb = Raw(sb, sb.shape[0], sb.shape[1], sb.shape[1] + ld_extra[1], torch.float16, offsets[1])
    odt = torch.float32 if out == "f32" else torch.float16
    rc_ = Raw(None, M, N, N + ld_extra[2], odt, offsets[2])
    rbias = Raw(bias.view(1, -1), 1, N, N, torch.float16, bias_offset) if bias is not None else None
    c = tlg.tlg_config(**(cfg or {}))
    rc = lib.tlg_gemm_op(M, N, K, int(at), ra.ptr(), ra.ld, int(bt), rb.ptr(), rb.ld,
                         rbias.ptr() if rbias is not None else None, rc_.ptr(), rc_.ld,
                         tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16,
                         tlg.TLG_EPI_BIAS_RELU if bias is not None else tlg.TLG_EPI_NONE,
                         ctypes.byref(c), None, 0, int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    guards = all(r.guard_ok() for r in (ra, rb, rc_) + ((rbias,) if rbias is not None else ()))
    return rc_.matrix().double().cpu().numpy(), guards


@pytest.mark.parametrize("tile", PLAIN_TILES)
@pytest.mark.parametrize("out,bias_relu", OUTS)
@pytest.mark.parametrize("op", [("N", "N"), ("N", "T"), ("T", "N"), ("T", "T")], ids=lambda o: o[0] + o[1])
def test_odd_strides_every_path(tlg, tile, out, bias_relu, op):
    # lda, ldb, ldc odd: no stride is a multiple of 16 bytes
    M, N, K = 333, 277, 299
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=bias_relu, seed=tile[1] + M)
    cfg = {"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]}
    got, guards = run(tlg, A, B, bias, out, cfg, op=op)
    assert guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=bias_relu), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_element_aligned_bases(tlg, out, bias_relu):
    # every base one element past a 16-byte boundary, strides aligned
    M, N, K = 260, 192, 256
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=bias_relu, seed=41)
    got, guards = run(tlg, A, B, bias, out, ld_extra=(0, 0, 0), offsets=(1, 3, 1), bias_offset=1)
    assert guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=bias_relu), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("out", ["f32", "f16"])
def test_only_c_unaligned_keeps_tma_loads(tlg, out):
    M, N, K = 520, 301, 512
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=42)
    got, guards = run(tlg, A, B, None, out, ld_extra=(0, 3, 1))  # ldb = 304 (aligned), ldc = N + 1
    assert guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


def test_only_bias_unaligned(tlg):
    M, N, K = 256, 512, 128
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=43)
    got, guards = run(tlg, A, B, bias, "f16", ld_extra=(0, 0, 0), bias_offset=3)
    assert guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=True), "f16")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (129, 65, 63), (255, 17, 1001)])
def test_unaligned_ragged_edges(tlg, M, N, K):
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=M * N + K)
    got, guards = run(tlg, A, B, None, "f32", ld_extra=(1, 3, 1), offsets=(1, 1, 1))
    assert guards
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), "f32")
    assert ok, f"worst err/bound {worst:.3g} at {idx}"


def test_unaligned_integer_inputs_bit_exact(tlg):
    M, N, K = 1001, 999, 2047
    A, B, _ = wl.integer_operands(M, N, K, seed=44)
    got, guards = run(tlg, A, B, None, "f32")
    assert guards
    assert np.array_equal(got, oracle.gemm(A, B))

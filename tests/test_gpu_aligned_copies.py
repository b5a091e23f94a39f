"""Operands the TMA unit cannot describe, with a workspace large enough for aligned copies
(tlg_gemm_workspace_size_op): the call copies such an A or B into the workspace, runs the TMA
path on the copies, and produces such a C in the workspace and copies it out.  Every case is
checked against the CPU oracle, with NaN guard bands around each caller matrix, and the
workspace's split-K counters must be left zero."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from test_gpu_unaligned import Raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def call(tlg, A, B, bias, out, ld_extra, offsets=(0, 0, 0), op=("N", "N"), cfg=None, ws_mode="full",
         act=None, residual=None, inplace=False):
    """One call on raw buffers; ws_mode: "full" (the size query's bytes), "split" (only the
    split scratch: copies do not fit) or "none"."""
    lib = tlg.raw_library()
    at, bt = op[0] == "T", op[1] == "T"
    M, K = A.shape
    N = B.shape[1]
    sa = A.t().contiguous() if at else A
    sb = B.t().contiguous() if bt else B
    ra = Raw(sa, sa.shape[0], sa.shape[1], sa.shape[1] + ld_extra[0], torch.float16, offsets[0])
    rb = Raw(sb, sb.shape[0], sb.shape[1], sb.shape[1] + ld_extra[1], torch.float16, offsets[1])
    odt = torch.float32 if out == "f32" else torch.float16
    rc_ = Raw(residual if inplace else None, M, N, N + ld_extra[2], odt, offsets[2])
    dbias = bias.cuda() if bias is not None else None
    c = tlg.tlg_config(**cfg) if cfg else None
    o = tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16
    full = ctypes.c_size_t(0)
    rcq = lib.tlg_gemm_workspace_size_op(M, N, K, int(at), ra.ptr(), ra.ld, int(bt), rb.ptr(), rb.ld, rc_.ptr(),
                                         rc_.ld, o, ctypes.byref(c) if c else None, ctypes.byref(full))
    assert rcq == 0, tlg.tlg_status_string(rcq)
    split_only = tlg.tlg_gemm_workspace_size(M, N, K, out, bias is not None, cfg)
    nbytes = {"full": full.value, "split": split_only, "none": 0}[ws_mode]
    ws = tlg.tlg_workspace(nbytes) if nbytes else None
    epi = tlg.tlg_fused_epilogue(dbias.data_ptr() if dbias is not None else None,
                                 {None: 0, "relu": 1, "gelu": 2}[act], None, 0)
    if inplace:
        epi.residual, epi.ldr = rc_.ptr(), rc_.ld
    rc = lib.tlg_gemm_fused(M, N, K, int(at), ra.ptr(), ra.ld, int(bt), rb.ptr(), rb.ld, ctypes.byref(epi),
                            rc_.ptr(), rc_.ld, o, ctypes.byref(c) if c else None,
                            ws.data_ptr() if ws is not None else None, nbytes,
                            int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    assert all(r.guard_ok() for r in (ra, rb, rc_)), "guard band changed"
    if ws is not None:
        assert int(ws[:4096].count_nonzero()) == 0, "split-K counters left non-zero"
    return rc_.matrix().double().cpu().numpy(), full.value


@pytest.mark.parametrize("out", ["f16", "f32"])
@pytest.mark.parametrize("which", ["A", "B", "C", "AB", "ABC"])
@pytest.mark.parametrize("ws_mode", ["full", "split", "none"])
def test_copies_or_plain_loads(tlg, which, out, ws_mode):
    M, N, K = 300, 264, 200
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=401)
    ex = (1 if "A" in which else 8, 1 if "B" in which else 8, 1 if "C" in which else 16 // (4 if out == "f32" else 2))
    offs = (1 if "A" in which else 0, 3 if "B" in which else 0, 1 if "C" in which else 0)
    got, full = call(tlg, A, B, bias, out, ex, offs, ws_mode=ws_mode, act="relu")
    assert full > 0
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=True), out)
    assert ok, (worst, idx)


@pytest.mark.parametrize("op", [("T", "N"), ("N", "T"), ("T", "T")], ids=lambda o: o[0] + o[1])
def test_copies_of_transposed_operands(tlg, op):
    M, N, K = 260, 300, 136
    A, B, _ = wl.make_operands(M, N, K, "normal025", seed=402)
    got, _ = call(tlg, A, B, None, "f32", (3, 5, 1), (1, 1, 1), op=op)
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B), "f32")
    assert ok, (worst, idx)


def test_copy_of_c_with_in_place_residual(tlg):
    # R == C, both unaligned: the kernel reads R from the caller's C and writes the aligned copy,
    # which is then copied over C
    M, N, K = 300, 264, 200
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=403)
    R = wl.make_residual(M, N, "f16", seed=403)
    got, _ = call(tlg, A, B, bias, "f16", (1, 1, 1), (1, 1, 1), act="gelu", residual=R, inplace=True)
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm_fused(A, B, bias=bias, act="gelu", residual=R), "f16")
    assert ok, (worst, idx)


def test_copies_with_a_forced_split(tlg):
    M, N, K = 1024, 768, 1024
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=404)
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 4}
    got, full = call(tlg, A, B, bias, "f16", (1, 1, 1), (1, 1, 1), cfg=cfg, act="relu")
    assert full > tlg.tlg_gemm_workspace_size(M, N, K, "f16", True, cfg)
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=True), "f16")
    assert ok, (worst, idx)


def test_integer_inputs_bit_exact_through_copies(tlg):
    M, N, K = 700, 520, 1000
    A, B, _ = wl.integer_operands(M, N, K, seed=405)
    got, _ = call(tlg, A, B, None, "f32", (1, 1, 1), (1, 1, 1))
    assert np.array_equal(got, oracle.gemm(A, B))


def test_size_query_for_aligned_operands_is_the_split_scratch(tlg):
    M = N = K = 4096
    A = torch.empty((M, K), dtype=torch.float16, device="cuda")
    B = torch.empty((K, N), dtype=torch.float16, device="cuda")
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert tlg.tlg_gemm_workspace_size_op(A, B, C) == tlg.tlg_gemm_workspace_size(M, N, K, "f16", False)
    Ao = torch.empty((M, K + 1), dtype=torch.float16, device="cuda")[:, :K]
    more = tlg.tlg_gemm_workspace_size_op(Ao, B, C)
    assert more >= tlg.tlg_gemm_workspace_size(M, N, K, "f16", False) + M * K * 2


def test_size_query_bytes_hold_the_split_and_the_copy(tlg):
    # 108 pair tiles (3072 x 2304): one whole wave, then a tail the automatic choice cuts in two
    # along K when the workspace holds the slices' partial sums (K = 2048: 32 k-blocks, long
    # enough that the model keeps the split).  Only A needs a copy.  With exactly the size
    # query's bytes the call must take the same schedule as the query: the split scratch
    # first, then A's aligned copy, ending at the workspace's last byte.
    M, N, K = 3072, 2304, 2048
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=406)
    lib = tlg.raw_library()
    ra = Raw(A, M, K, K + 1, torch.float16, 0)
    Bd, C = B.cuda(), torch.empty((M, N), dtype=torch.float16, device="cuda")
    full = ctypes.c_size_t(0)
    rcq = lib.tlg_gemm_workspace_size_op(M, N, K, 0, ra.ptr(), ra.ld, 0, Bd.data_ptr(), N, C.data_ptr(), N,
                                         tlg.TLG_OUT_F16, None, ctypes.byref(full))
    assert rcq == 0, tlg.tlg_status_string(rcq)
    a_copy = M * K * 2  # rows of 4096 bytes: already 16- and 256-byte multiples
    split_ws = tlg.tlg_gemm_workspace_size(M, N, K, "f16", True)
    assert split_ws > 4096, "the automatic choice no longer splits this shape"
    assert full.value == (split_ws + 255) // 256 * 256 + a_copy
    ws = tlg.tlg_workspace(full.value)
    ws[4096:] = 0xFF
    dbias = bias.cuda()
    epi = tlg.tlg_fused_epilogue(dbias.data_ptr(), 1, None, 0)
    rc = lib.tlg_gemm_fused(M, N, K, 0, ra.ptr(), ra.ld, 0, Bd.data_ptr(), N, ctypes.byref(epi), C.data_ptr(), N,
                            tlg.TLG_OUT_F16, None, ws.data_ptr(), full.value,
                            int(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    assert ra.guard_ok()
    assert int(ws[:4096].count_nonzero()) == 0, "split-K counters left non-zero"
    tail = ws[full.value - a_copy:].view(torch.float16).view(M, K).cpu()
    assert torch.equal(tail.view(torch.int16), A.view(torch.int16)), "A's copy is not where the query put it"
    assert int((ws[4096:4096 + 1024] != 0xFF).sum()) > 0, "no partial sums: the split tail was not taken"
    rows = np.arange(0, M, 97)
    got = C[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    ref = oracle.gemm(A[torch.from_numpy(rows)], B, bias=bias, relu=True)
    ok, worst, idx = oracle.within_tolerance(got, ref, "f16")
    assert ok, (worst, idx)


def test_copy_chain_back_to_back(tlg):
    # Calls whose A, B and C all need copies, issued back to back on one stream with two input
    # sets alternating: the copy of A and B, the GEMM (a programmatic dependent of it) and the
    # copy of C (a dependent of the GEMM) must each see the kernel before it complete.  A result
    # that mixed in the other set's data would differ from that set's first result, which the
    # oracle checks; the kernels are deterministic, so every repeat must match it bit for bit.
    lib = tlg.raw_library()
    M, N, K = 520, 264, 1000
    sets = [wl.make_operands(M, N, K, "uniform", bias=True, seed=407 + i) for i in range(2)]
    raws = []
    for A, B, bias in sets:
        ra = Raw(A, M, K, K + 1, torch.float16, 1)
        rb = Raw(B, K, N, N + 3, torch.float16, 3)
        raws.append((ra, rb, bias.cuda()))
    rc_ = Raw(None, M, N, N + 1, torch.float16, 1)
    full = ctypes.c_size_t(0)
    ra0, rb0, _ = raws[0]
    assert lib.tlg_gemm_workspace_size_op(M, N, K, 0, ra0.ptr(), ra0.ld, 0, rb0.ptr(), rb0.ld, rc_.ptr(), rc_.ld,
                                          tlg.TLG_OUT_F16, None, ctypes.byref(full)) == 0
    ws = tlg.tlg_workspace(full.value)
    stream = int(torch.cuda.current_stream().cuda_stream)
    outs = []
    for it in range(12):
        ra, rb, dbias = raws[it % 2]
        rc = lib.tlg_gemm_op(M, N, K, 0, ra.ptr(), ra.ld, 0, rb.ptr(), rb.ld, dbias.data_ptr(), rc_.ptr(), rc_.ld,
                             tlg.TLG_OUT_F16, tlg.TLG_EPI_BIAS_RELU, None, ws.data_ptr(), full.value, stream)
        assert rc == 0, tlg.tlg_status_string(rc)
        outs.append(rc_.matrix().clone())  # stream-ordered copy of this call's C
    torch.cuda.synchronize()
    assert rc_.guard_ok()
    for i, (A, B, bias) in enumerate(sets):
        got = outs[i].double().cpu().numpy()
        ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=True), "f16")
        assert ok, (i, worst, idx)
    for it in range(2, 12):
        assert torch.equal(outs[it].view(torch.int16), outs[it % 2].view(torch.int16)), it


@pytest.mark.parametrize("out", ["f16", "f32"])
def test_large_copies_match_the_aligned_call_bit_for_bit(tlg, out):
    # 4096 rows of 8 KB (fp16) or 16 KB (fp32): every warp of the copy kernels walks many row
    # pieces.  The same GEMM configuration runs on aligned operands and on odd-stride ones
    # (copied in, C copied out); the copies are exact, so the two Cs must agree bit for bit.
    lib = tlg.raw_library()
    M, N, K = 4096, 4096, 256
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=408)
    odt = torch.float32 if out == "f32" else torch.float16
    o = tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16
    cfg = tlg.tlg_config(cta_group=2, block_n=256, split_k=1)
    stream = int(torch.cuda.current_stream().cuda_stream)
    dA, dB = A.cuda(), B.cuda()
    ref = torch.empty((M, N), dtype=odt, device="cuda")
    rc = lib.tlg_gemm_op(M, N, K, 0, dA.data_ptr(), K, 0, dB.data_ptr(), N, None, ref.data_ptr(), N, o,
                         tlg.TLG_EPI_NONE, ctypes.byref(cfg), None, 0, stream)
    assert rc == 0, tlg.tlg_status_string(rc)
    ra = Raw(A, M, K, K + 1, torch.float16, 1)
    rb = Raw(B, K, N, N + 3, torch.float16, 5)
    rc_ = Raw(None, M, N, N + 1, odt, 1)
    full = ctypes.c_size_t(0)
    assert lib.tlg_gemm_workspace_size_op(M, N, K, 0, ra.ptr(), ra.ld, 0, rb.ptr(), rb.ld, rc_.ptr(), rc_.ld, o,
                                          ctypes.byref(cfg), ctypes.byref(full)) == 0
    ws = tlg.tlg_workspace(full.value)
    rc = lib.tlg_gemm_op(M, N, K, 0, ra.ptr(), ra.ld, 0, rb.ptr(), rb.ld, None, rc_.ptr(), rc_.ld, o,
                         tlg.TLG_EPI_NONE, ctypes.byref(cfg), ws.data_ptr(), full.value, stream)
    assert rc == 0, tlg.tlg_status_string(rc)
    torch.cuda.synchronize()
    assert all(r.guard_ok() for r in (ra, rb, rc_)), "guard band changed"
    ityp = torch.int32 if out == "f32" else torch.int16
    assert torch.equal(rc_.matrix().contiguous().view(ityp), ref.view(ityp))
    rows = np.arange(0, M, 127)
    got = ref[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A[torch.from_numpy(rows)], B), out)
    assert ok, (worst, idx)

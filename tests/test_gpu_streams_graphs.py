"""Concurrency and CUDA-graph capture of the C ABI calls, on the GPU, against the oracle.

- Two GEMMs of different shapes and epilogues in flight at once on two streams: the
  library's only shared device state is its error words, so both results must match.
- A call captured into a CUDA graph after one eager call (which prepares the kernel's launch
  attributes) and replayed: every replay recomputes C from the current inputs.
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


def test_two_streams_at_once(tlg):
    A1, B1, b1 = wl.make_operands(1024, 768, 2048, "uniform", bias=True, seed=201)
    A2, B2, _ = wl.make_operands(600, 1300, 520, "normal025", seed=202)
    R2 = wl.make_residual(600, 1300, "f32", seed=202)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    d1 = (A1.cuda(), B1.cuda(), b1.cuda())
    d2 = (A2.cuda(), B2.cuda(), R2.cuda())
    torch.cuda.synchronize()
    outs = []
    for _ in range(4):  # several rounds so the kernels overlap in time
        c1 = tlg.tlg_gemm_bias_relu_f16(*d1, stream=s1)
        c2 = tlg.tlg_gemm_fused(d2[0], d2[1], activation="gelu", residual=d2[2], out="f32", stream=s2)
        outs.append((c1, c2))
    torch.cuda.synchronize()
    ref1 = oracle.gemm(A1, B1, bias=b1, relu=True)
    ref2 = oracle.gemm_fused(A2, B2, act="gelu", residual=R2)
    for c1, c2 in outs:
        ok, worst, idx = oracle.within_tolerance(c1.double().cpu().numpy(), ref1, "f16")
        assert ok, (worst, idx)
        ok, worst, idx = oracle.within_tolerance(c2.double().cpu().numpy(), ref2, "f32")
        assert ok, (worst, idx)
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0


@pytest.mark.parametrize("entry", ["bias_relu", "ex_split", "fused"])
def test_graph_capture_and_replay(tlg, entry):
    M, N, K = 2560, 2048, 512  # 80 pair tiles: one whole wave, then 6 tiles a split can cut
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=211)
    dA, dB, db = A.cuda(), B.cuda(), bias.cuda()
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = None
    if entry == "ex_split":
        cfg = {"cta_group": 2, "block_n": 256, "split_k": 2}
        ws = tlg.tlg_workspace(tlg.tlg_gemm_workspace_size(M, N, K, "f16", True, cfg))

    def call(stream=None):
        if entry == "bias_relu":
            tlg.tlg_gemm_bias_relu_f16(dA, dB, db, C, stream=stream)
        elif entry == "ex_split":
            tlg.tlg_gemm_ex(dA, dB, db, C, out="f16", config=cfg, workspace=ws, stream=stream)
        else:
            tlg.tlg_gemm_fused(dA, dB, bias=db, activation="gelu", C=C, out="f16", stream=stream)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        call(s)  # eager first call: sets the kernel's launch attributes
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(s)
    act = "gelu" if entry == "fused" else "relu"
    for seed in (212, 213):
        # new inputs in the same buffers; the replay must use them
        A2, B2, b2 = wl.make_operands(M, N, K, "uniform", bias=True, seed=seed)
        dA.copy_(A2)
        dB.copy_(B2)
        db.copy_(b2)
        C.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.gemm_fused(A2, B2, bias=b2, act=act)
        ok, worst, idx = oracle.within_tolerance(C.double().cpu().numpy(), ref, "f16")
        assert ok, (entry, seed, worst, idx)
    if ws is not None:
        assert int(ws[:4096].count_nonzero()) == 0
    del g
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0

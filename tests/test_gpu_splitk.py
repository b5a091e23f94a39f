"""GPU tests of the split-K tail (tlg_gemm_ex with a workspace): forced and
automatic splits against the CPU oracle, determinism, and the workspace
counters returning to zero after every call."""

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from gpu_util import gemm_padded

pytestmark = pytest.mark.gpu

TILES = [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)]
OUTS = [("f32", False), ("f16", False), ("f16", True)]


@pytest.fixture(scope="module")
def tlg():
    import tiled_dense_gemm_tlg_b200 as t
    return t


def counters_zero(ws):
    return bool((ws[:4096] == 0).all().item())


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("split", [2, 3, 5])
@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_forced_split_matches_oracle(tlg, tile, split, out, bias_relu):
    # few tiles (all in the tail), ragged M/N/K, K-blocks not divisible by the split
    M, N, K = 300, 200, 1000
    A, B, bias = wl.make_operands(M, N, K, "normal025", bias=bias_relu, seed=split * 10 + tile[1])
    cfg = {"cta_group": tile[0], "block_n": tile[1], "split_k": split}
    nbytes = tlg.tlg_gemm_workspace_size(M, N, K, out, bias_relu, cfg)
    assert nbytes > 4096
    ws = tlg.tlg_workspace(nbytes)
    C = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), bias.cuda() if bias is not None else None, out=out,
                        config=cfg, workspace=ws)
    torch.cuda.synchronize()
    ok, worst, idx = oracle.within_tolerance(C.double().cpu().numpy(), oracle.gemm(A, B, bias=bias, relu=bias_relu), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"
    assert counters_zero(ws)


@pytest.mark.parametrize("out,bias_relu", OUTS)
def test_split_tail_with_whole_waves_and_guards(tlg, out, bias_relu):
    # more tiles than resident units: whole-tile waves plus a split tail, on padded operands
    import ctypes
    lib = tlg.raw_library()
    M, N, K = 2200, 2100, 777
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=bias_relu, seed=4)
    cfg = {"cta_group": 1, "block_n": 128, "split_k": 2, "max_ctas": 100}
    nbytes = tlg.tlg_gemm_workspace_size(M, N, K, out, bias_relu, cfg)
    ws = tlg.tlg_workspace(nbytes)
    got, guards = gemm_padded(lib, A, B, bias, out, config=cfg, extra=(8, 8, 8), workspace=ws)
    assert guards, repr(guards)
    ok, worst, idx = oracle.within_tolerance(got, oracle.gemm(A, B, bias=bias, relu=bias_relu), out)
    assert ok, f"worst err/bound {worst:.3g} at {idx}"
    assert counters_zero(ws)


def test_split_is_deterministic(tlg):
    M, N, K = 1024, 768, 2048
    A, B, _ = wl.make_operands(M, N, K, "uniform", seed=5)
    dA, dB = A.cuda(), B.cuda()
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 4}
    ws = tlg.tlg_workspace(tlg.tlg_gemm_workspace_size(M, N, K, "f32", False, cfg))
    C1 = tlg.tlg_gemm_ex(dA, dB, out="f32", config=cfg, workspace=ws)
    C2 = tlg.tlg_gemm_ex(dA, dB, out="f32", config=cfg, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)
    ok, _, _ = oracle.within_tolerance(C1.double().cpu().numpy(), oracle.gemm(A, B), "f32")
    assert ok


def test_split_integer_inputs_bit_exact(tlg):
    # with exact partial sums the split result equals the oracle bit for bit
    M, N, K = 640, 512, 4096
    A, B, _ = wl.integer_operands(M, N, K, seed=6)
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 3}
    ws = tlg.tlg_workspace(tlg.tlg_gemm_workspace_size(M, N, K, "f32", False, cfg))
    C = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), out="f32", config=cfg, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(C.double().cpu().numpy(), oracle.gemm(A, B))


def test_forced_split_on_the_bias_relu_workload(tlg):
    # the full-size bias+ReLU workload with its leftover tiles split in two
    w = wl.WORKLOADS["gemm_bias_relu_4096_f16"]
    cfg = {"cta_group": 2, "block_n": 256, "split_k": 2}
    nbytes = tlg.tlg_gemm_workspace_size(w.M, w.N, w.K, "f16", True, cfg)
    assert nbytes > 4096
    # automatic: whole tiles, or (given the scratch) this same split of the partial last wave
    assert tlg.tlg_gemm_workspace_size(w.M, w.N, w.K, "f16", True) in (0, nbytes)
    A, B, bias = wl.workload_operands(w)
    ws = tlg.tlg_workspace(nbytes)
    C = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), bias.cuda(), out="f16", config=cfg, workspace=ws)
    torch.cuda.synchronize()
    rows, cols = wl.sample_positions(w.M, w.N, 4096, seed=1)
    # include rows of every row block of the tail tiles: the last rows of the matrix
    r = np.concatenate([rows.numpy(), np.arange(w.M - 512, w.M)])
    c = np.concatenate([cols.numpy(), np.random.default_rng(0).integers(0, w.N, 512)])
    ref = oracle.gemm_at(A, B, r, c, bias=bias, relu=True)
    got = C[torch.as_tensor(r).cuda(), torch.as_tensor(c).cuda()].double().cpu().numpy()
    ok, worst, idx = oracle.within_tolerance(got, ref, "f16")
    assert ok, f"worst err/bound {worst:.3g} at ({r[idx]}, {c[idx]})"
    assert counters_zero(ws)


def test_split_without_workspace_is_rejected_or_skipped(tlg):
    A = torch.ones((512, 512), dtype=torch.float16, device="cuda")
    with pytest.raises(tlg.TlgError):
        tlg.tlg_gemm_ex(A, A, out="f32", config={"split_k": 2, "cta_group": 2, "block_n": 256})
    # automatic choice: whole tiles, no workspace needed
    C = tlg.tlg_gemm_ex(A, A, out="f32")
    assert (C == 512).all()


def test_no_device_error_after_split_runs(tlg):
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, hex(code)


def test_automatic_split_with_a_workspace(tlg):
    # 256 pair tiles on 74 pairs leave a partial last wave; with a workspace the automatic
    # choice splits that tail (and only then); the result is the forced split's, bit for bit.
    M, N, K = 4096, 4096, 512
    A, B, bias = wl.make_operands(M, N, K, "uniform", bias=True, seed=91)
    auto = tlg.tlg_choose_config(M, N, K, "f16", True)
    nbytes = tlg.tlg_gemm_workspace_size(M, N, K, "f16", True)
    dA, dB, db = A.cuda(), B.cuda(), bias.cuda()
    plain = tlg.tlg_gemm_bias_relu_f16(dA, dB, db)
    if auto["split_k"] < 2:
        assert nbytes == 0
        pytest.skip(f"no split chosen on this device: {auto}")
    assert nbytes > 0
    ws = tlg.tlg_workspace(nbytes)
    C = tlg.tlg_gemm_ex(dA, dB, db, out="f16", workspace=ws)
    forced = tlg.tlg_gemm_ex(dA, dB, db, out="f16", config=auto, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(C, forced)
    assert int(ws[:4096].count_nonzero()) == 0
    rows, cols = wl.sample_positions(M, N, 4096, seed=92)
    ref = oracle.gemm_at(A, B, rows.numpy(), cols.numpy(), bias=bias, relu=True)
    for got in (C, plain):
        ok, worst, idx = oracle.within_tolerance(got.double().cpu().numpy()[rows.numpy(), cols.numpy()], ref, "f16")
        assert ok, f"worst err/bound {worst:.3g} at sample {idx}"
    # without a workspace the same automatic call does not split (and still runs)
    C2 = tlg.tlg_gemm_ex(dA, dB, db, out="f16")
    torch.cuda.synchronize()
    assert torch.equal(C2, plain)

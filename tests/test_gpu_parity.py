"""GPU parity against the CPU oracle on the five workloads, through the C ABI.

Small shapes are compared element by element over the whole output; the full
-size shapes run in the launch configuration the benchmark times (the
automatic choice) and are compared on sampled outputs plus their first and
last rows and columns, which cross every ragged tile edge.
Tolerances: fp32 output |gpu - ref| <= 1e-2 + 2e-3 |ref|; fp16 output
|gpu - ref| <= 2e-2 + 1e-2 |ref|.
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


def run_workload(tlg, w, A, B, bias):
    dA, dB = A.cuda(), B.cuda()
    if w.bias_relu:
        C = tlg.tlg_gemm_bias_relu_f16(dA, dB, bias.cuda())
    elif w.out == "f16":
        C = tlg.tlg_gemm_f16f16(dA, dB)
    else:
        C = tlg.tlg_gemm_f16f32(dA, dB)
    torch.cuda.synchronize()
    return C


def check_positions(C, A, B, bias, w, rows, cols):
    ref = oracle.gemm_at(A, B, rows, cols, bias=bias, relu=w.bias_relu)
    got = C[torch.as_tensor(rows, device=C.device), torch.as_tensor(cols, device=C.device)].double().cpu().numpy()
    ok, worst, idx = oracle.within_tolerance(got, ref, w.out)
    assert ok, f"{w.name}: worst err/bound {worst:.3g} at sample {idx} ({rows[idx]}, {cols[idx]}) got {got[idx]} ref {ref[idx]}"
    return worst


def edge_positions(M, N, count=2048, seed=3):
    rng = np.random.default_rng(seed)
    r = np.concatenate([np.zeros(count // 4, np.int64), np.full(count // 4, M - 1),
                        rng.integers(0, M, count // 4), rng.integers(0, M, count // 4)])
    c = np.concatenate([rng.integers(0, N, count // 4), rng.integers(0, N, count // 4),
                        np.zeros(count // 4, np.int64), np.full(count // 4, N - 1)])
    return r, c


@pytest.mark.parametrize("name", ["gemm_256_f32", "gemm_1024_f32", "gemm_ragged_4000x3000x1000_f32"])
def test_full_output_matches_oracle(tlg, name):
    w = wl.WORKLOADS[name]
    A, B, bias = wl.workload_operands(w)
    C = run_workload(tlg, w, A, B, bias)
    ref = oracle.gemm(A, B, bias=bias, relu=w.bias_relu)
    got = C.double().cpu().numpy()
    ok, worst, idx = oracle.within_tolerance(got, ref, w.out)
    assert ok, f"{name}: worst err/bound {worst:.3g} at {idx}: got {got[idx]} ref {ref[idx]}"
    assert np.isfinite(got).all()


@pytest.mark.parametrize("name", ["gemm_bias_relu_4096_f16", "gemm_8192_f16"])
def test_full_size_sampled_matches_oracle(tlg, name):
    w = wl.WORKLOADS[name]
    A, B, bias = wl.workload_operands(w)
    C = run_workload(tlg, w, A, B, bias)
    rows, cols = wl.sample_positions(w.M, w.N, w.sample or 4096, seed=1)
    check_positions(C, A, B, bias, w, rows.numpy(), cols.numpy())
    er, ec = edge_positions(w.M, w.N)
    check_positions(C, A, B, bias, w, er, ec)
    assert torch.isfinite(C).all()
    if w.bias_relu:
        assert (C >= 0).all()


@pytest.mark.parametrize("name", wl.WORKLOAD_ORDER)
def test_integer_inputs_are_bit_exact(tlg, name):
    # Entries in {-2..2}: every partial sum is an integer of magnitude <= 4K < 2^24,
    # so the fp32 accumulation is exact in any order and the fp32 result must equal
    # the oracle bit for bit; fp16 results must equal the oracle's RNE rounding.
    w = wl.WORKLOADS[name]
    A, B, bias = wl.integer_operands(w.M, w.N, w.K, seed=11, bias=w.bias_relu)
    C = run_workload(tlg, w, A, B, bias)
    if w.sample:
        rows, cols = wl.sample_positions(w.M, w.N, w.sample, seed=12)
        rows, cols = rows.numpy(), cols.numpy()
        ref = oracle.gemm_at(A, B, rows, cols, bias=bias, relu=w.bias_relu)
        got = C[torch.as_tensor(rows).cuda(), torch.as_tensor(cols).cuda()].cpu()
    else:
        ref = oracle.gemm(A, B, bias=bias, relu=w.bias_relu)
        got = C.cpu()
    if w.out == "f32":
        assert np.array_equal(got.double().numpy(), ref)
    else:
        want = oracle.f16_encode_rne(ref)
        assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), want)


@pytest.mark.parametrize("tile", [(1, 64, 8), (1, 128, 6), (1, 256, 4), (2, 128, 8), (2, 256, 6), (2, 512, 4)])
def test_every_tile_on_the_bias_relu_workload(tlg, tile):
    # the full-size bias+ReLU workload under each kernel variant the library builds
    w = wl.WORKLOADS["gemm_bias_relu_4096_f16"]
    A, B, bias = wl.workload_operands(w)
    C = tlg.tlg_gemm_ex(A.cuda(), B.cuda(), bias.cuda(), out="f16",
                        config={"cta_group": tile[0], "block_n": tile[1], "stages": tile[2]})
    torch.cuda.synchronize()
    er, ec = edge_positions(w.M, w.N, count=1024, seed=sum(tile))
    check_positions(C, A, B, bias, w, er, ec)


def test_matches_cublas_secondary(tlg):
    # secondary cross-check only (not the oracle): torch.matmul on the same fp16 inputs
    A, B, _ = wl.make_operands(1024, 768, 2048, "uniform", seed=21)
    dA, dB = A.cuda(), B.cuda()
    C = tlg.tlg_gemm_f16f32(dA, dB)
    ref = torch.matmul(dA.float(), dB.float())
    assert torch.allclose(C, ref, atol=1e-2, rtol=2e-3)


def test_repeatable_bit_for_bit(tlg):
    w = wl.WORKLOADS["gemm_ragged_4000x3000x1000_f32"]
    A, B, _ = wl.workload_operands(w)
    dA, dB = A.cuda(), B.cuda()
    C1 = tlg.tlg_gemm_f16f32(dA, dB)
    C2 = tlg.tlg_gemm_f16f32(dA, dB)
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)


def test_no_device_error_reported(tlg):
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0, f"device error word {code:#x}"

"""Extreme shapes through the automatic configuration: a K of 2^20 (16384 k-blocks), a
300000-row and a 500000-column output (thousands of ragged tiles), and 8192 x 8192 with
K = 8 (a single ragged k-block per tile).  Integer-valued inputs keep every partial sum
exact in fp32, so fp32 results must equal the oracle bit for bit."""

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


@pytest.mark.parametrize("M,N,K,lo,hi", [
    (64, 64, 1 << 20, -1, 1),      # K * max|a| * max|b| = 2^20 < 2^24: exact in fp32
    (300000, 8, 24, -2, 2),        # tall and skinny: 2344 row tiles, N = 8 of 64
    (8, 500000, 16, -2, 2),        # short and wide
    (8192, 8192, 8, -2, 2),        # many tiles, one ragged k-block each
], ids=["k2^20", "tall", "wide", "k8"])
def test_extreme_shapes_bit_exact(tlg, M, N, K, lo, hi):
    A, B, _ = wl.integer_operands(M, N, K, lo=lo, hi=hi, seed=M + N + K)
    C = tlg.tlg_gemm_f16f32(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    got = C.double().cpu().numpy()
    if M * N <= 4_000_000:
        assert np.array_equal(got, oracle.gemm(A, B))
    else:  # the full oracle would be large to hold; exact values at sampled positions
        rows, cols = wl.sample_positions(M, N, 20000, seed=7)
        ref = oracle.gemm_at(A, B, rows.numpy(), cols.numpy())
        assert np.array_equal(got[rows.numpy(), cols.numpy()], ref)
        assert np.isfinite(got).all()
    rc, code = tlg.tlg_device_error(clear=True)
    assert rc == 0 and code == 0

"""Pins for the CPU oracle, against things other than the oracle itself.

Each check is written as a function of a GEMM callable so that the same
checks can be run against deliberately broken copies of the oracle (the
"planted mistakes" at the bottom): every plausible mistake must fail at least
one pin.  All of this runs on the CPU.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import tlg_workloads as wl
from conftest import read_golden_blocks, read_golden_pairs


def f16(x):
    return np.asarray(x, dtype=np.float16)


def dec(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64)


# ----------------------------------------------------------------------------- codec

def test_decode_exhaustive_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_decode(bits)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_decode_golden_values():
    for h, v in read_golden_pairs("f16_values.txt"):
        got = oracle.f16_decode(np.array([int(h, 16)], dtype=np.uint16))[0]
        want = float(v)
        assert got == want, (h, got, want)
        assert math.copysign(1.0, got) == math.copysign(1.0, want), h


def test_encode_golden_rounding():
    for x, h in read_golden_pairs("f16_rounding.txt"):
        got = int(oracle.f16_encode_rne(np.array([float(x)]))[0])
        assert got == int(h, 16), (x, hex(got), h)


def test_encode_roundtrips_every_finite_fp16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(vals)
    back = oracle.f16_encode_rne(vals[finite])
    assert np.array_equal(back, bits[finite])


def test_encode_matches_numpy_on_random_doubles():
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
        rng.uniform(-70000, 70000, 50000),
        # exact midpoints between neighbouring fp16 values
        (np.arange(0, 31743, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
         + np.arange(1, 31744, 7, dtype=np.uint16).view(np.float16).astype(np.float64)) / 2,
    ])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = oracle.f16_encode_rne(x)
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------- pins as functions of a GEMM

def pin_golden(gemm):
    for ex in read_golden_blocks("gemm_worked_examples.txt"):
        M, N, K = ex["shape"]
        A = f16(ex["A"]).reshape(M, K)
        B = f16(ex["B"]).reshape(K, N)
        C = np.array(ex["C"]).reshape(M, N)
        assert np.array_equal(gemm(A, B, None, False), C), ex["name"]


def pin_golden_bias_relu(gemm):
    for ex in read_golden_blocks("bias_relu_worked_examples.txt"):
        M, N, K = ex["shape"]
        A = f16(ex["A"]).reshape(M, K)
        B = f16(ex["B"]).reshape(K, N)
        bias = f16(ex["bias"])
        C = np.array(ex["C"]).reshape(M, N)
        assert np.array_equal(gemm(A, B, bias, True), C), ex["name"]


def pin_identity(gemm):
    rng = np.random.default_rng(1)
    B = f16(rng.uniform(-1, 1, (37, 23)))
    I = np.eye(37, dtype=np.float16)
    assert np.array_equal(gemm(I, B, None, False), dec(B))
    A = f16(rng.uniform(-1, 1, (19, 23)))
    I2 = np.eye(23, dtype=np.float16)
    assert np.array_equal(gemm(A, I2, None, False), dec(A))


def pin_all_ones(gemm):
    for M, N, K in [(3, 5, 1), (4, 7, 17), (2, 3, 256), (5, 2, 1000)]:
        C = gemm(np.ones((M, K), np.float16), np.ones((K, N), np.float16), None, False)
        assert np.array_equal(C, np.full((M, N), float(K)))


def pin_numpy_matmul(gemm):
    rng = np.random.default_rng(2)
    for M, N, K in [(67, 45, 129), (1, 130, 257), (33, 1, 64)]:
        A = f16(rng.uniform(-1, 1, (M, K)))
        B = f16(rng.standard_normal((K, N)))
        want = dec(A) @ dec(B)
        scale = np.abs(dec(A)) @ np.abs(dec(B))
        got = gemm(A, B, None, False)
        assert np.all(np.abs(got - want) <= 1e-12 * (scale + 1e-300)), (M, N, K)


def pin_fsum_dots(gemm):
    rng = np.random.default_rng(3)
    for K in [1, 2, 63, 64, 65, 1000]:
        a = f16(rng.uniform(-1, 1, (1, K)))
        b = f16(rng.uniform(-1, 1, (K, 1)))
        exact = math.fsum(float(x) * float(y) for x, y in zip(dec(a)[0], dec(b)[:, 0]))
        got = gemm(a, b, None, False)[0, 0]
        bound = 1e-13 * math.fsum(abs(float(x) * float(y)) for x, y in zip(dec(a)[0], dec(b)[:, 0]))
        assert abs(got - exact) <= bound, K


def pin_transpose(gemm):
    rng = np.random.default_rng(4)
    A = f16(rng.uniform(-1, 1, (9, 13)))
    B = f16(rng.uniform(-1, 1, (13, 6)))
    assert np.array_equal(gemm(A, B, None, False).T, gemm(B.T.copy(), A.T.copy(), None, False))


def pin_bias_column_broadcast(gemm):
    rng = np.random.default_rng(5)
    M, N, K = 6, 11, 4
    bias = f16(rng.uniform(-0.5, 0.5, N))
    zero = gemm(np.zeros((M, K), np.float16), f16(rng.uniform(-1, 1, (K, N))), bias, True)
    assert np.array_equal(zero, np.tile(np.maximum(dec(bias), 0.0), (M, 1)))
    neg = gemm(f16(rng.uniform(-1, 1, (M, K))), f16(rng.uniform(-1, 1, (K, N))),
               np.full(N, -1000, np.float16), True)
    assert np.array_equal(neg, np.zeros((M, N)))
    A = f16(rng.uniform(-1, 1, (M, K)))
    B = f16(rng.uniform(-1, 1, (K, N)))
    r = gemm(A, B, bias, True)
    assert np.all(r >= 0)
    plain = gemm(A, B, None, False)
    assert np.array_equal(r, np.maximum(plain + dec(bias)[None, :], 0.0))


PINS = [pin_golden, pin_golden_bias_relu, pin_identity, pin_all_ones, pin_numpy_matmul,
        pin_fsum_dots, pin_transpose, pin_bias_column_broadcast]


def oracle_gemm(A, B, bias, relu):
    return oracle.gemm(A, B, bias=bias, relu=relu, threads=2)


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pins(pin):
    pin(oracle_gemm)


# ----------------------------------------------------------------------------- other invariants

def test_sampled_equals_full_bit_for_bit():
    A, B, bias = wl.make_operands(70, 90, 300, "uniform", bias=True, seed=7)
    full = oracle.gemm(A, B, bias=bias, relu=True)
    rows, cols = wl.sample_positions(70, 90, 500, seed=8)
    at = oracle.gemm_at(A, B, rows.numpy(), cols.numpy(), bias=bias, relu=True)
    assert np.array_equal(at, full[rows.numpy(), cols.numpy()])


def test_thread_count_does_not_change_result():
    A, B, _ = wl.make_operands(64, 48, 200, "normal025", seed=9)
    r1 = oracle.gemm(A, B, threads=1)
    r8 = oracle.gemm(A, B, threads=8)
    assert np.array_equal(r1, r8)


def test_pure_python_loop_agrees_on_tiny_input():
    A, B, bias = wl.make_operands(3, 4, 5, "uniform", bias=True, seed=10)
    a, b, bb = dec(A.numpy()), dec(B.numpy()), dec(bias.numpy())
    want = np.zeros((3, 4))
    for i in range(3):
        for j in range(4):
            s = 0.0
            for k in range(5):
                s += a[i, k] * b[k, j]
            want[i, j] = max(s + bb[j], 0.0)
    assert np.array_equal(oracle.gemm(A, B, bias=bias, relu=True), want)


def test_empty_and_degenerate_shapes():
    A = np.zeros((0, 5), np.float16)
    B = np.ones((5, 3), np.float16)
    assert oracle.gemm(A, B).shape == (0, 3)
    A = np.zeros((4, 0), np.float16)
    B = np.zeros((0, 3), np.float16)
    assert np.array_equal(oracle.gemm(A, B), np.zeros((4, 3)))  # empty sum is 0
    bias = f16([-1, 0.5, 2])
    assert np.array_equal(oracle.gemm(A, B, bias=bias, relu=True), np.tile([0.0, 0.5, 2.0], (4, 1)))


def test_uniform_generator_statistics():
    # U[-1,1] entries: each product has variance 1/9, so an output has variance K/9 and mean 0.
    w = wl.WORKLOADS["gemm_256_f32"]
    A, B, _ = wl.workload_operands(w)
    C = oracle.gemm(A, B)
    K = w.K
    assert abs(C.mean()) < 0.05 * math.sqrt(K / 9)
    assert abs(C.var() / (K / 9) - 1.0) < 0.05
    a = dec(A.numpy())
    assert a.min() >= -1 and a.max() <= 1 and abs(a.var() - 1 / 3) < 0.01


def test_inputs_are_seeded_and_ordered():
    A1, B1, b1 = wl.make_operands(8, 9, 10, "uniform", bias=True, seed=0)
    A2, B2, b2 = wl.make_operands(8, 9, 10, "uniform", bias=True, seed=0)
    assert torch.equal(A1, A2) and torch.equal(B1, B2) and torch.equal(b1, b2)
    g = torch.Generator().manual_seed(0)
    assert torch.equal(A1, (torch.rand((8, 10), generator=g) * 2 - 1).half())
    A3, _, _ = wl.make_operands(8, 9, 10, "uniform", seed=1)
    assert not torch.equal(A1, A3)


def test_tolerance_helper():
    ref = np.array([0.0, 1.0, 100.0])
    ok, worst, _ = oracle.within_tolerance(ref + np.array([0.009, 0.011, 0.2]), ref, "f32")
    assert ok and worst < 1.0
    ok, _, idx = oracle.within_tolerance(ref + np.array([0.0, 0.0, 0.3]), ref, "f32")
    assert not ok and idx == (2,)
    ok, _, _ = oracle.within_tolerance(np.array([np.nan, 1.0, 100.0]), ref, "f32")
    assert not ok


# ----------------------------------------------------------------------------- planted mistakes
# Broken copies of the oracle's arithmetic (numpy, on the CPU).  Each must fail
# at least one of the pins above, which shows the pins can see that mistake.

def _ref(A, B, bias, relu):
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if relu:
        C = np.maximum(C, 0.0)
    return C


def mutant_dropped_last_k(A, B, bias, relu):
    return _ref(np.ascontiguousarray(A[:, :-1]), np.ascontiguousarray(B[:-1, :]), bias, relu)


def mutant_transposed_B(A, B, bias, relu):
    K, N = B.shape
    if K == N:
        return _ref(A, np.ascontiguousarray(B.T), bias, relu)
    return _ref(A, np.ascontiguousarray(B.reshape(N, K).T), bias, relu)


def mutant_row_bias(A, B, bias, relu):
    C = dec(A) @ dec(B)
    if bias is not None:
        M = C.shape[0]
        bb = dec(bias)
        C = C + np.resize(bb, M)[:, None]
    return np.maximum(C, 0.0) if relu else C


def mutant_bias_sign(A, B, bias, relu):
    return _ref(A, B, None if bias is None else (-dec(bias)).astype(np.float16), relu)


def mutant_relu_before_bias(A, B, bias, relu):
    C = dec(A) @ dec(B)
    if relu:
        C = np.maximum(C, 0.0)
    if bias is not None:
        C = C + dec(bias)[None, :]
    return C


def mutant_fp16_accumulator(A, B, bias, relu):
    a, b = dec(A), dec(B)
    M, K = a.shape
    N = b.shape[1]
    C = np.zeros((M, N), np.float16)
    for k in range(K):
        C = (C + (a[:, k:k + 1] * b[k:k + 1, :]).astype(np.float16)).astype(np.float16)
    C = C.astype(np.float64)
    if bias is not None:
        C = C + dec(bias)[None, :]
    return np.maximum(C, 0.0) if relu else C


def mutant_off_by_one_row(A, B, bias, relu):
    C = _ref(A, B, bias, relu)
    return np.roll(C, 1, axis=0) if C.shape[0] > 1 else C


def mutant_f32_products(A, B, bias, relu):
    C = (dec(A).astype(np.float32) @ dec(B).astype(np.float32)).astype(np.float64)
    if bias is not None:
        C = C + dec(bias)[None, :]
    return np.maximum(C, 0.0) if relu else C


MUTANTS = [mutant_dropped_last_k, mutant_transposed_B, mutant_row_bias, mutant_bias_sign,
           mutant_relu_before_bias, mutant_fp16_accumulator, mutant_off_by_one_row, mutant_f32_products]


def test_reference_numpy_copy_passes_pins():
    for pin in PINS:
        pin(_ref)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_planted_mistake_is_caught(mutant):
    failed = []
    for pin in PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"{mutant.__name__} passed every pin"


# ----------------------------------------------------------------------------- the general fused epilogue
# ref = act(A.B + bias[col]) + R[row, col], act in {none, relu, gelu}
# ("domestic-GPU TileLang adoption" section 4.1: activation and residual fused
# into the GEMM; section 4.2: bias by output column, before the activation).
# GELU is x * Phi(x), Phi the standard normal CDF, checked against scipy's
# normal CDF and against the symmetry gelu(x) - gelu(-x) = x.

from scipy.special import ndtr  # noqa: E402

PHI_1 = 0.841344746068542948  # the standard normal CDF at 1 (table value)


def _gelu_scipy(x):
    x = np.asarray(x, dtype=np.float64)
    return x * ndtr(x)


def fpin_golden(g):
    for ex in read_golden_blocks("fused_epilogue_worked_examples.txt"):
        M, N, K = ex["shape"]
        A = f16(ex["A"]).reshape(M, K)
        B = f16(ex["B"]).reshape(K, N)
        bias = None if ex["bias"] is None else f16(ex["bias"])
        R = None if ex["R"] is None else f16(ex["R"]).reshape(M, N)
        C = np.array(ex["C"]).reshape(M, N)
        got = g(A, B, bias, ex["act"], R)
        assert np.all(np.abs(got - C) <= 1e-15), (ex["name"], got, C)


def fpin_gelu_library(g):
    # A = I (K = N), B = x as fp16: the output row is act(x) exactly at the input points.
    x = np.concatenate([np.linspace(-6, 6, 61), [-1.0, 1.0, 0.0, 1e-4, -1e-4, 0.5, -0.5]])
    xb = f16(x)
    n = xb.size
    out = g(np.ones((1, 1), np.float16), xb.reshape(1, n), None, "gelu", None)[0]
    want = _gelu_scipy(dec(xb))
    assert np.all(np.abs(out - want) <= 4e-15 * (1 + np.abs(dec(xb)))), np.max(np.abs(out - want))


def fpin_gelu_symmetry_and_limits(g):
    xb = f16(np.linspace(0, 8, 33))
    pos = g(np.ones((1, 1), np.float16), xb.reshape(1, -1), None, "gelu", None)[0]
    neg = g(-np.ones((1, 1), np.float16), xb.reshape(1, -1), None, "gelu", None)[0]
    x = dec(xb)
    assert np.all(np.abs((pos - neg) - x) <= 1e-14 * (1 + x))
    assert pos[0] == 0.0 and neg[0] == 0.0
    assert abs(pos[-1] - 8.0) < 1e-13 and abs(neg[-1]) < 1e-13
    one = g(np.ones((1, 1), np.float16), np.ones((1, 1), np.float16), None, "gelu", None)[0, 0]
    assert abs(one - PHI_1) <= 1e-15


def fpin_residual_is_added_after_activation(g):
    rng = np.random.default_rng(6)
    M, N, K = 5, 7, 3
    A = f16(rng.uniform(-1, 1, (M, K)))
    B = f16(rng.uniform(-1, 1, (K, N)))
    bias = f16(rng.uniform(-0.5, 0.5, N))
    R = f16(rng.uniform(-2, 2, (M, N)))
    for act in ("none", "relu", "gelu"):
        with_r = g(A, B, bias, act, R)
        without = g(A, B, bias, act, None)
        assert np.array_equal(with_r, without + dec(R)), act
    # a zero product leaves act(bias) + R: the residual keeps its row and column
    zero = g(np.zeros((M, K), np.float16), B, bias, "relu", R)
    assert np.array_equal(zero, np.maximum(dec(bias), 0.0)[None, :] + dec(R))


def fpin_fused_reduces_to_bias_relu(g):
    rng = np.random.default_rng(7)
    M, N, K = 9, 12, 70
    A = f16(rng.uniform(-1, 1, (M, K)))
    B = f16(rng.uniform(-1, 1, (K, N)))
    bias = f16(rng.uniform(-0.5, 0.5, N))
    want = dec(A) @ dec(B) + dec(bias)[None, :]
    scale = np.abs(dec(A)) @ np.abs(dec(B)) + np.abs(dec(bias))[None, :]
    got = g(A, B, bias, "relu", None)
    assert np.all(np.abs(got - np.maximum(want, 0.0)) <= 1e-12 * scale)
    got = g(A, B, None, "none", None)
    assert np.all(np.abs(got - dec(A) @ dec(B)) <= 1e-12 * scale)


FPINS = [fpin_golden, fpin_gelu_library, fpin_gelu_symmetry_and_limits,
         fpin_residual_is_added_after_activation, fpin_fused_reduces_to_bias_relu]


def oracle_fused(A, B, bias, act, R):
    return oracle.gemm_fused(A, B, bias=bias, act=act, residual=R, threads=2)


@pytest.mark.parametrize("pin", FPINS, ids=lambda p: p.__name__)
def test_oracle_fused_pins(pin):
    pin(oracle_fused)


def test_fused_sampled_equals_full_bit_for_bit():
    rng = np.random.default_rng(8)
    M, N, K = 40, 33, 129
    A = f16(rng.uniform(-1, 1, (M, K)))
    B = f16(rng.uniform(-1, 1, (K, N)))
    bias = f16(rng.uniform(-0.5, 0.5, N))
    R = f16(rng.uniform(-1, 1, (M, N)))
    rows = rng.integers(0, M, 200)
    cols = rng.integers(0, N, 200)
    for act in ("none", "relu", "gelu"):
        full = oracle.gemm_fused(A, B, bias=bias, act=act, residual=R, threads=3)
        at = oracle.gemm_at_fused(A, B, rows, cols, bias=bias, act=act, residual=R, threads=2)
        assert np.array_equal(at, full[rows, cols]), act
    assert np.array_equal(oracle.gemm_fused(A, B, bias=bias, act="relu", threads=2),
                          oracle.gemm(A, B, bias=bias, relu=True, threads=2))


def test_oracle_activation_points():
    assert oracle.activation(-2.0, "relu") == 0.0 and oracle.activation(3.0, "relu") == 3.0
    assert oracle.activation(-2.5, "none") == -2.5
    assert abs(oracle.activation(1.0, "gelu") - PHI_1) <= 1e-15


def _fref(A, B, bias, act, R):
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if act == "relu":
        C = np.maximum(C, 0.0)
    elif act == "gelu":
        C = _gelu_scipy(C)
    if R is not None:
        C = C + dec(R)
    return C


def fmutant_residual_inside_activation(A, B, bias, act, R):
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if R is not None:
        C = C + dec(R)
    return _fref(np.ones((C.shape[0], 1), np.float16), np.zeros((1, C.shape[1]), np.float16),
                 None, "none", None) + (np.maximum(C, 0.0) if act == "relu" else
                                        _gelu_scipy(C) if act == "gelu" else C)


def fmutant_gelu_tanh_form(A, B, bias, act, R):
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if act == "relu":
        C = np.maximum(C, 0.0)
    elif act == "gelu":
        C = 0.5 * C * (1 + np.tanh(math.sqrt(2 / math.pi) * (C + 0.044715 * C ** 3)))
    return C + (dec(R) if R is not None else 0.0)


def fmutant_gelu_sign(A, B, bias, act, R):
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if act == "relu":
        C = np.maximum(C, 0.0)
    elif act == "gelu":
        C = C * ndtr(-C)
    return C + (dec(R) if R is not None else 0.0)


def fmutant_residual_transposed(A, B, bias, act, R):
    C = _fref(A, B, bias, act, None)
    if R is not None:
        M, N = C.shape
        C = C + dec(R).reshape(N, M).T
    return C


def fmutant_residual_dropped(A, B, bias, act, R):
    return _fref(A, B, bias, act, None)


def fmutant_residual_shifted_row(A, B, bias, act, R):
    C = _fref(A, B, bias, act, None)
    if R is not None:
        C = C + np.roll(dec(R), 1, axis=0)
    return C


FMUTANTS = [fmutant_residual_inside_activation, fmutant_gelu_tanh_form, fmutant_gelu_sign,
            fmutant_residual_transposed, fmutant_residual_dropped, fmutant_residual_shifted_row]


def test_fused_numpy_copy_passes_pins():
    for pin in FPINS:
        pin(_fref)


@pytest.mark.parametrize("mutant", FMUTANTS, ids=lambda m: m.__name__)
def test_fused_planted_mistake_is_caught(mutant):
    failed = []
    for pin in FPINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"{mutant.__name__} passed every pin"


def test_fused_residual_in_fp32():
    # An fp32 residual enters at its exact value: R = 2^-20 * odd integers,
    # which fp16 cannot hold, is added exactly after the activation.
    rng = np.random.default_rng(9)
    M, N, K = 4, 6, 5
    A = f16(rng.uniform(-1, 1, (M, K)))
    B = f16(rng.uniform(-1, 1, (K, N)))
    R = (rng.integers(-2 ** 19, 2 ** 19, (M, N)) * 2 + 1).astype(np.float32) * np.float32(2.0 ** -20)
    base = oracle.gemm_fused(A, B, act="gelu", threads=1)
    got = oracle.gemm_fused(A, B, act="gelu", residual=R, threads=1)
    assert np.array_equal(got, base + R.astype(np.float64))
    assert not np.array_equal(got, base + dec(R.astype(np.float16)))


# ----------------------------------------------------------------------------- SiLU and the tanh form of GELU
# Standard definitions (the adoption page names activation fusion without formulas): SiLU is
# x * sigmoid(x), checked against scipy's expit; the tanh form of GELU is checked against
# torch's own implementation (gelu(approximate="tanh")) in float64.

from scipy.special import expit  # noqa: E402


def _points():
    return f16(np.concatenate([np.linspace(-12, 12, 97), [-1.0, 1.0, 0.0, 1e-3, -1e-3, 30.0, -30.0]]))


def _act_row(g, act):
    xb = _points()
    return dec(xb), g(np.ones((1, 1), np.float16), xb.reshape(1, -1), None, act, None)[0]


def apin_silu_library(g):
    x, out = _act_row(g, "silu")
    assert np.all(np.abs(out - x * expit(x)) <= 4e-16 * (1 + np.abs(x))), np.max(np.abs(out - x * expit(x)))


def apin_gelu_tanh_library(g):
    import torch
    x, out = _act_row(g, "gelu_tanh")
    want = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.all(np.abs(out - want) <= 1e-15 * (1 + np.abs(x))), np.max(np.abs(out - want))


def apin_sigmoid_forms_limits(g):
    for act in ("silu", "gelu_tanh"):
        x, out = _act_row(g, act)
        assert out[np.argmin(np.abs(x))] == 0.0                      # act(0) = 0
        big = x >= 12
        assert np.all(np.abs(out[big] - x[big]) <= 1e-4 * x[big])     # act(x) -> x
        assert np.all(np.abs(out[x <= -12]) <= 1e-4)                  # act(x) -> 0
    # SiLU(x) - SiLU(-x) = x, and the tanh-GELU obeys the same symmetry
    xb = f16(np.linspace(0, 6, 25))
    for act in ("silu", "gelu_tanh"):
        pos = g(np.ones((1, 1), np.float16), xb.reshape(1, -1), None, act, None)[0]
        neg = g(-np.ones((1, 1), np.float16), xb.reshape(1, -1), None, act, None)[0]
        assert np.all(np.abs((pos - neg) - dec(xb)) <= 1e-14 * (1 + dec(xb))), act


APINS = [apin_silu_library, apin_gelu_tanh_library, apin_sigmoid_forms_limits]


@pytest.mark.parametrize("pin", APINS, ids=lambda p: p.__name__)
def test_oracle_activation_pins(pin):
    pin(oracle_fused)


def _aref(A, B, bias, act, R):
    import torch
    C = dec(A) @ dec(B)
    if bias is not None:
        C = C + dec(bias)[None, :]
    if act == "silu":
        C = C * expit(C)
    elif act == "gelu_tanh":
        C = torch.nn.functional.gelu(torch.from_numpy(C), approximate="tanh").numpy()
    elif act == "gelu":
        C = _gelu_scipy(C)
    elif act == "relu":
        C = np.maximum(C, 0.0)
    return C + (dec(R) if R is not None else 0.0)


def amutant_silu_sign(A, B, bias, act, R):
    if act == "silu":
        C = dec(A) @ dec(B) + (dec(bias)[None, :] if bias is not None else 0.0)
        return C * expit(-C)
    return _aref(A, B, bias, act, R)


def amutant_gelu_tanh_without_cubic(A, B, bias, act, R):
    if act == "gelu_tanh":
        C = dec(A) @ dec(B) + (dec(bias)[None, :] if bias is not None else 0.0)
        return 0.5 * C * (1 + np.tanh(math.sqrt(2 / math.pi) * C))
    return _aref(A, B, bias, act, R)


def amutant_silu_is_exact_gelu(A, B, bias, act, R):
    return _aref(A, B, bias, "gelu" if act == "silu" else act, R)


def test_activation_numpy_copy_passes_pins():
    for pin in APINS:
        pin(_aref)


@pytest.mark.parametrize("mutant", [amutant_silu_sign, amutant_gelu_tanh_without_cubic, amutant_silu_is_exact_gelu],
                         ids=lambda m: m.__name__)
def test_activation_planted_mistake_is_caught(mutant):
    failed = []
    for pin in APINS:
        try:
            pin(mutant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"{mutant.__name__} passed every pin"

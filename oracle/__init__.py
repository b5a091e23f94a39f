"""CPU oracle for the fp16 GEMM (+bias+ReLU) path -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  The CUDA library never does: the two share no code,
no headers and no helpers.  The arithmetic lives in ``gemm_oracle.c`` (plain C,
fp64 accumulation); this module only marshals numpy/torch buffers into it.

Functions and the passages they follow:

* ``f16_decode`` / ``f16_encode_rne`` -- IEEE 754 binary16 codec (the pages
  use fp16 operands throughout, "tilelang operator-compilation walkthrough"
  (lqnn.cn/news/222844) section 4.2).
* ``gemm`` -- ref = A.B summed in fp64 ("tilelang operator-compilation
  walkthrough" sections 2.1 and 4.2; "TileLang Python DSL practice"
  (codechina.net/.../126997) section 3.2), optionally followed by
  ``max(ref + bias[col], 0)`` ("domestic-GPU TileLang adoption"
  (xdnf.cn/news/333523) section 4.2).
* ``gemm_at`` -- the same value at selected (row, col) positions.
* ``gemm_fused`` / ``gemm_at_fused`` -- act(A.B + bias[col]) + R[row, col] with
  act in {none, relu, gelu, silu, gelu_tanh} ("domestic-GPU TileLang adoption"
  section 4.1: activation and residual fused into the operator; the pages give
  no formulas, so each activation is its standard definition: GELU in its exact
  erf form, SiLU x*sigmoid(x), and the tanh form of GELU).

Every function is pinned by tests/test_oracle_pins.py; none is parity unpinned.
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from . import build as _build

_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            lib = ctypes.CDLL(path)
            lib.oracle_f16_decode.restype = ctypes.c_double
            lib.oracle_f16_decode.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_encode_rne.restype = ctypes.c_uint16
            lib.oracle_f16_encode_rne.argtypes = [ctypes.c_double]
            lib.oracle_f16_decode_array.argtypes = [_p, _p, _i64]
            lib.oracle_f16_encode_array.argtypes = [_p, _p, _i64]
            lib.oracle_gemm.restype = ctypes.c_int
            lib.oracle_gemm.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, ctypes.c_int,
                                        _p, _i64, ctypes.c_int]
            lib.oracle_gemm_at.argtypes = [_i64, _p, _i64, _p, _i64, _p, ctypes.c_int,
                                           _p, _p, _i64, _p, ctypes.c_int]
            lib.oracle_openmp_enabled.restype = ctypes.c_int
            lib.oracle_activation.restype = ctypes.c_double
            lib.oracle_activation.argtypes = [ctypes.c_double, ctypes.c_int]
            lib.oracle_gemm_fused.restype = ctypes.c_int
            lib.oracle_gemm_fused.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, ctypes.c_int,
                                              _p, _i64, _p, _i64, ctypes.c_int]
            lib.oracle_gemm_at_fused.argtypes = [_i64, _p, _i64, _p, _i64, _p, ctypes.c_int, _p, _i64,
                                                 _p, _p, _i64, _p, ctypes.c_int]
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _bits(x) -> np.ndarray:
    """fp16 data (torch tensor, numpy float16 or uint16 array) -> C-contiguous uint16 numpy array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            if x.dtype != torch.float16:
                raise TypeError(f"expected fp16 tensor, got {x.dtype}")
            x = x.detach().cpu().contiguous().view(torch.int16).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    elif x.dtype == np.int16:
        x = x.view(np.uint16)
    if x.dtype != np.uint16:
        raise TypeError(f"expected fp16 bits, got {x.dtype}")
    return np.ascontiguousarray(x)


def f16_decode(bits) -> np.ndarray:
    b = _bits(bits)
    out = np.empty(b.shape, dtype=np.float64)
    _load().oracle_f16_decode_array(b.ctypes.data, out.ctypes.data, b.size)
    return out


def _values(x) -> np.ndarray:
    """A residual in the output's type as exact float64 values: fp16 through the
    oracle's own decoder, fp32 (and fp64) by numpy's exact widening."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            if x.dtype == torch.float16:
                return f16_decode(x)
            if x.dtype not in (torch.float32, torch.float64):
                raise TypeError(f"residual must be fp16 or fp32, got {x.dtype}")
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype in (np.float16, np.uint16, np.int16):
        return f16_decode(x)
    if x.dtype not in (np.float32, np.float64):
        raise TypeError(f"residual must be fp16 or fp32, got {x.dtype}")
    return np.ascontiguousarray(x.astype(np.float64))


def f16_encode_rne(x) -> np.ndarray:
    """Round float64 values to binary16 (ties to even); returns the uint16 bit patterns."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f16_encode_array(x.ctypes.data, out.ctypes.data, x.size)
    return out


def gemm(A, B, bias=None, relu: bool = False, threads: int | None = None) -> np.ndarray:
    """ref[M,N] (float64) for fp16 A[M,K], B[K,N] and an optional fp16 bias[N]."""
    a, b = _bits(A), _bits(B)
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[0]:
        raise ValueError(f"shape mismatch {a.shape} x {b.shape}")
    M, K = a.shape
    N = b.shape[1]
    bb = None
    if bias is not None:
        bb = _bits(bias)
        if bb.shape != (N,):
            raise ValueError(f"bias must have shape ({N},), got {bb.shape}")
    out = np.empty((M, N), dtype=np.float64)
    rc = _load().oracle_gemm(M, N, K, a.ctypes.data, K, b.ctypes.data, N,
                             bb.ctypes.data if bb is not None else None, int(bool(relu)),
                             out.ctypes.data, N, int(threads or default_threads()))
    if rc != 0:
        raise MemoryError("oracle_gemm could not allocate its decoded copy of B")
    return out


def gemm_at(A, B, rows, cols, bias=None, relu: bool = False, threads: int | None = None) -> np.ndarray:
    """ref[rows[s], cols[s]] for each s, as float64."""
    a, b = _bits(A), _bits(B)
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[0]:
        raise ValueError(f"shape mismatch {a.shape} x {b.shape}")
    M, K = a.shape
    N = b.shape[1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    c = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    if r.shape != c.shape or r.ndim != 1:
        raise ValueError("rows and cols must be 1-D and of equal length")
    if r.size and (r.min() < 0 or r.max() >= M or c.min() < 0 or c.max() >= N):
        raise IndexError("sample position out of range")
    bb = None
    if bias is not None:
        bb = _bits(bias)
        if bb.shape != (N,):
            raise ValueError(f"bias must have shape ({N},), got {bb.shape}")
    out = np.empty(r.shape, dtype=np.float64)
    _load().oracle_gemm_at(K, a.ctypes.data, K, b.ctypes.data, N,
                           bb.ctypes.data if bb is not None else None, int(bool(relu)),
                           r.ctypes.data, c.ctypes.data, r.size, out.ctypes.data,
                           int(threads or default_threads()))
    return out


ACT = {"none": 0, "relu": 1, "gelu": 2, "silu": 3, "gelu_tanh": 4}


def activation(x: float, act: str) -> float:
    """The oracle's activation at one point (none, relu, gelu)."""
    return float(_load().oracle_activation(float(x), ACT[act]))


def gemm_fused(A, B, bias=None, act: str = "none", residual=None, threads: int | None = None) -> np.ndarray:
    """ref = act(A.B + bias[col]) + residual[row, col], float64 (the general fused epilogue).
    The residual has the output's type: fp16 (decoded here) or fp32."""
    a, b = _bits(A), _bits(B)
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[0]:
        raise ValueError(f"shape mismatch {a.shape} x {b.shape}")
    M, K = a.shape
    N = b.shape[1]
    bb = _bits(bias) if bias is not None else None
    if bb is not None and bb.shape != (N,):
        raise ValueError(f"bias must have shape ({N},)")
    rr = _values(residual) if residual is not None else None
    if rr is not None and rr.shape != (M, N):
        raise ValueError(f"residual must have shape ({M}, {N})")
    out = np.empty((M, N), dtype=np.float64)
    rc = _load().oracle_gemm_fused(M, N, K, a.ctypes.data, K, b.ctypes.data, N,
                                   bb.ctypes.data if bb is not None else None, ACT[act],
                                   rr.ctypes.data if rr is not None else None, N,
                                   out.ctypes.data, N, int(threads or default_threads()))
    if rc != 0:
        raise MemoryError("oracle_gemm_fused could not allocate its decoded copy of B")
    return out


def gemm_at_fused(A, B, rows, cols, bias=None, act: str = "none", residual=None,
                  threads: int | None = None) -> np.ndarray:
    a, b = _bits(A), _bits(B)
    M, K = a.shape
    N = b.shape[1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    c = np.ascontiguousarray(np.asarray(cols, dtype=np.int64))
    if r.size and (r.min() < 0 or r.max() >= M or c.min() < 0 or c.max() >= N):
        raise IndexError("sample position out of range")
    bb = _bits(bias) if bias is not None else None
    rr = _values(residual) if residual is not None else None
    if rr is not None and rr.shape != (M, N):
        raise ValueError(f"residual must have shape ({M}, {N})")
    out = np.empty(r.shape, dtype=np.float64)
    _load().oracle_gemm_at_fused(K, a.ctypes.data, K, b.ctypes.data, N,
                                 bb.ctypes.data if bb is not None else None, ACT[act],
                                 rr.ctypes.data if rr is not None else None, N,
                                 r.ctypes.data, c.ctypes.data, r.size, out.ctypes.data,
                                 int(threads or default_threads()))
    return out


def openmp_enabled() -> bool:
    return bool(_load().oracle_openmp_enabled())


# Output tolerances for comparing the GPU path with this oracle.
# fp32 outputs: |gpu - ref| <= 1e-2 + 2e-3 |ref|;  fp16 outputs: <= 2e-2 + 1e-2 |ref|.
TOL = {"f32": (1e-2, 2e-3), "f16": (2e-2, 1e-2)}


def within_tolerance(gpu: np.ndarray, ref: np.ndarray, out: str):
    """(ok, worst ratio |err| / bound, index of the worst element)."""
    atol, rtol = TOL[out]
    g = np.asarray(gpu, dtype=np.float64)
    err = np.abs(g - ref)
    bound = atol + rtol * np.abs(ref)
    ratio = np.where(np.isfinite(g), err / bound, np.inf)
    if ratio.size == 0:
        return True, 0.0, None
    idx = int(np.argmax(ratio))
    worst = float(ratio.flat[idx])
    return worst <= 1.0, worst, np.unravel_index(idx, ratio.shape)

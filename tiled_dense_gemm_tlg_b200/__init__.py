"""Python binding of libtlg, the B200 (sm_100a) fp16 GEMM library.

Argument marshalling only: every step of the GEMM runs in the CUDA kernels of
``libtlg.so`` behind the C interface in ``include/tlg.h``.  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: importing
this package fails when the library has not been built, and a call with CPU
tensors is rejected by the library (TLG_ERR_INVALID_ARG) rather than returning
an empty result.

Functions (same names as the C entry points):

* ``tlg_gemm_f16f32(A, B, C=None)``        C fp32 = A.B
* ``tlg_gemm_f16f16(A, B, C=None)``        C fp16 = A.B
* ``tlg_gemm_bias_relu_f16(A, B, bias, C=None)``  C fp16 = max(A.B + bias, 0)
* ``tlg_gemm_ex(...)``                     any of the above with an explicit configuration
* ``tlg_gemm_op(...)``                     operands stored transposed
* ``tlg_gemm_fused(...)``                  C = act(op(A).op(B) + bias) + residual
* ``tlg_choose_config``, ``tlg_device_error``, ``tlg_selftest_timeout``,
  ``tlg_status_string``, ``tlg_version``

A and B are 2-D fp16 tensors with unit stride along their last dimension
(row-major); their row strides become lda / ldb.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtlg.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libtlg.so not found at {LIB_PATH}: build it with `python tiled_dense_gemm_tlg_b200/build.py` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

TLG_OK, TLG_ERR_INVALID_ARG, TLG_ERR_ALIGNMENT, TLG_ERR_UNSUPPORTED, TLG_ERR_CUDA, TLG_ERR_TIMEOUT = range(6)
TLG_OUT_F32, TLG_OUT_F16 = 0, 1
TLG_EPI_NONE, TLG_EPI_BIAS_RELU = 0, 1
TLG_OP_N, TLG_OP_T = 0, 1
TLG_ACT_NONE, TLG_ACT_RELU, TLG_ACT_GELU, TLG_ACT_SILU, TLG_ACT_GELU_TANH = 0, 1, 2, 3, 4
_ACT = {"none": TLG_ACT_NONE, "relu": TLG_ACT_RELU, "gelu": TLG_ACT_GELU, "silu": TLG_ACT_SILU,
        "gelu_tanh": TLG_ACT_GELU_TANH}

EXPORTED = ("tlg_gemm_f16f32", "tlg_gemm_f16f16", "tlg_gemm_bias_relu_f16", "tlg_gemm_ex",
            "tlg_gemm_op", "tlg_gemm_fused", "tlg_gemm_ex_noalloc", "tlg_gemm_workspace_size",
            "tlg_gemm_workspace_size_op", "tlg_choose_config", "tlg_device_error",
            "tlg_selftest_timeout", "tlg_status_string", "tlg_version")


class tlg_config(ctypes.Structure):
    _fields_ = [("block_n", ctypes.c_int32), ("stages", ctypes.c_int32), ("cta_group", ctypes.c_int32),
                ("raster_group", ctypes.c_int32), ("max_ctas", ctypes.c_int32),
                ("split_k", ctypes.c_int32), ("overlap_prev", ctypes.c_int32), ("k_split", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class tlg_fused_epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("activation", ctypes.c_int32),
                ("residual", ctypes.c_void_p), ("ldr", ctypes.c_int64)]


_i64, _p, _i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
_lib.tlg_gemm_f16f32.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _i64, _p]
_lib.tlg_gemm_f16f16.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _i64, _p]
_lib.tlg_gemm_bias_relu_f16.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p, _i64, _p]
_sz = ctypes.c_size_t
_lib.tlg_gemm_ex.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p, _i64, _i32, _i32,
                             ctypes.POINTER(tlg_config), _p, _sz, _p]
_lib.tlg_gemm_op.argtypes = [_i64, _i64, _i64, _i32, _p, _i64, _i32, _p, _i64, _p, _p, _i64, _i32, _i32,
                             ctypes.POINTER(tlg_config), _p, _sz, _p]
_lib.tlg_gemm_fused.argtypes = [_i64, _i64, _i64, _i32, _p, _i64, _i32, _p, _i64,
                                ctypes.POINTER(tlg_fused_epilogue), _p, _i64, _i32,
                                ctypes.POINTER(tlg_config), _p, _sz, _p]
_lib.tlg_gemm_ex_noalloc.argtypes = [_i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p, _i64, _i32, _i32,
                                     ctypes.POINTER(tlg_config), _p]
_lib.tlg_gemm_workspace_size.argtypes = [_i64, _i64, _i64, _i32, _i32, ctypes.POINTER(tlg_config),
                                         ctypes.POINTER(_sz)]
_lib.tlg_gemm_workspace_size_op.argtypes = [_i64, _i64, _i64, _i32, _p, _i64, _i32, _p, _i64, _p, _i64, _i32,
                                            ctypes.POINTER(tlg_config), ctypes.POINTER(_sz)]
_lib.tlg_choose_config.argtypes = [_i64, _i64, _i64, _i32, _i32, ctypes.POINTER(tlg_config)]
_lib.tlg_device_error.argtypes = [_i32, ctypes.POINTER(ctypes.c_uint32)]
_lib.tlg_selftest_timeout.argtypes = [ctypes.c_uint32, _p]
_lib.tlg_status_string.argtypes = [_i32]
_lib.tlg_status_string.restype = ctypes.c_char_p
_lib.tlg_version.restype = ctypes.c_int32
for _name in ("tlg_gemm_f16f32", "tlg_gemm_f16f16", "tlg_gemm_bias_relu_f16", "tlg_gemm_ex",
              "tlg_gemm_op", "tlg_gemm_fused", "tlg_gemm_ex_noalloc", "tlg_gemm_workspace_size", "tlg_gemm_workspace_size_op", "tlg_choose_config", "tlg_device_error", "tlg_selftest_timeout"):
    getattr(_lib, _name).restype = _i32


class TlgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tlg_status_string(status)}")


def tlg_status_string(status: int) -> str:
    return _lib.tlg_status_string(int(status)).decode()


def tlg_version() -> int:
    return int(_lib.tlg_version())


def _check(rc: int, where: str):
    if rc != TLG_OK:
        raise TlgError(rc, where)


def _stream_handle(stream, *tensors) -> int:
    if stream is not None:
        return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)
    for t in tensors:
        if t is not None and t.is_cuda:
            return int(torch.cuda.current_stream(t.device).cuda_stream)
    return 0


def _mat(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor")
    if t.size(1) > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must be row-major (unit stride along its last dimension)")
    if t.size(0) > 1 and t.stride(0) < t.size(1):
        # a broadcast or overlapping view: its rows are not `stride(0)` elements apart in a
        # buffer of rows x stride(0) elements, which is what the library would read
        raise ValueError(f"{name} has overlapping rows (row stride {t.stride(0)} < {t.size(1)} columns)")
    return t.data_ptr(), max(t.stride(0), t.size(1))


def _shapes(A, B):
    if A.dtype != torch.float16 or B.dtype != torch.float16:
        raise TypeError("A and B must be fp16")
    M, K = A.shape
    K2, N = B.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: A is {tuple(A.shape)}, B is {tuple(B.shape)}")
    return M, N, K


def _out(C, M, N, dtype, like):
    if C is None:
        return torch.empty((M, N), dtype=dtype, device=like.device)
    if C.dtype != dtype or tuple(C.shape) != (M, N):
        raise ValueError(f"C must be {dtype} of shape ({M}, {N})")
    return C


def tlg_gemm_f16f32(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor | None = None, stream=None):
    M, N, K = _shapes(A, B)
    C = _out(C, M, N, torch.float32, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    _check(_lib.tlg_gemm_f16f32(M, N, K, pa, lda, pb, ldb, pc, ldc, _stream_handle(stream, A, B, C)),
           "tlg_gemm_f16f32")
    return C


def tlg_gemm_f16f16(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor | None = None, stream=None):
    M, N, K = _shapes(A, B)
    C = _out(C, M, N, torch.float16, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    _check(_lib.tlg_gemm_f16f16(M, N, K, pa, lda, pb, ldb, pc, ldc, _stream_handle(stream, A, B, C)),
           "tlg_gemm_f16f16")
    return C


def tlg_gemm_bias_relu_f16(A: torch.Tensor, B: torch.Tensor, bias: torch.Tensor,
                           C: torch.Tensor | None = None, stream=None):
    M, N, K = _shapes(A, B)
    if bias.dtype != torch.float16 or bias.dim() != 1 or bias.numel() != N or (N > 1 and bias.stride(0) != 1):
        raise ValueError(f"bias must be a contiguous fp16 vector of length {N}")
    C = _out(C, M, N, torch.float16, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    _check(_lib.tlg_gemm_bias_relu_f16(M, N, K, pa, lda, pb, ldb, bias.data_ptr(), pc, ldc,
                                       _stream_handle(stream, A, B, C)), "tlg_gemm_bias_relu_f16")
    return C


def tlg_gemm_ex(A: torch.Tensor, B: torch.Tensor, bias: torch.Tensor | None = None,
                C: torch.Tensor | None = None, out: str = "f32", config: dict | None = None,
                workspace: torch.Tensor | None = None, stream=None):
    """Explicit-configuration form; ``out`` is "f32" or "f16"; a bias selects the bias+ReLU epilogue.
    ``workspace``: optional device buffer (see ``tlg_workspace``) enabling the split-K tail."""
    M, N, K = _shapes(A, B)
    o = TLG_OUT_F32 if out == "f32" else TLG_OUT_F16
    C = _out(C, M, N, torch.float32 if o == TLG_OUT_F32 else torch.float16, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    cfg = None
    if config is not None:
        cfg = tlg_config(**{k: int(v) for k, v in config.items()})
    epi = TLG_EPI_BIAS_RELU if bias is not None else TLG_EPI_NONE
    ws_ptr, ws_bytes = (None, 0)
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check(_lib.tlg_gemm_ex(M, N, K, pa, lda, pb, ldb, bias.data_ptr() if bias is not None else None,
                            pc, ldc, o, epi, ctypes.byref(cfg) if cfg is not None else None,
                            ws_ptr, ws_bytes, _stream_handle(stream, A, B, C)), "tlg_gemm_ex")
    return C


def tlg_gemm_op(A: torch.Tensor, B: torch.Tensor, op_a: str = "N", op_b: str = "N",
                bias: torch.Tensor | None = None, C: torch.Tensor | None = None, out: str = "f32",
                config: dict | None = None, workspace: torch.Tensor | None = None, stream=None):
    """C = op(A).op(B): ``op_a == "T"`` means A is stored K x M and its transpose is used;
    ``op_b == "T"`` means B is stored N x K.  Stored matrices are row-major."""
    at, bt = op_a.upper() == "T", op_b.upper() == "T"
    if A.dtype != torch.float16 or B.dtype != torch.float16:
        raise TypeError("A and B must be fp16")
    M, K = (A.shape[1], A.shape[0]) if at else tuple(A.shape)
    K2, N = (B.shape[1], B.shape[0]) if bt else tuple(B.shape)
    if K != K2:
        raise ValueError(f"inner dimensions differ: op(A) is {M}x{K}, op(B) is {K2}x{N}")
    o = TLG_OUT_F32 if out == "f32" else TLG_OUT_F16
    C = _out(C, M, N, torch.float32 if o == TLG_OUT_F32 else torch.float16, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    cfg = tlg_config(**{k: int(v) for k, v in config.items()}) if config is not None else None
    epi = TLG_EPI_BIAS_RELU if bias is not None else TLG_EPI_NONE
    ws_ptr, ws_bytes = (None, 0)
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check(_lib.tlg_gemm_op(M, N, K, TLG_OP_T if at else TLG_OP_N, pa, lda, TLG_OP_T if bt else TLG_OP_N,
                            pb, ldb, bias.data_ptr() if bias is not None else None, pc, ldc, o, epi,
                            ctypes.byref(cfg) if cfg is not None else None, ws_ptr, ws_bytes,
                            _stream_handle(stream, A, B, C)), "tlg_gemm_op")
    return C


def tlg_gemm_fused(A: torch.Tensor, B: torch.Tensor, op_a: str = "N", op_b: str = "N",
                   bias: torch.Tensor | None = None, activation: str = "none",
                   residual: torch.Tensor | None = None, C: torch.Tensor | None = None,
                   out: str = "f16", config: dict | None = None,
                   workspace: torch.Tensor | None = None, stream=None):
    """C = act(op(A).op(B) + bias[col]) + residual[row, col].

    ``activation``: "none", "relu", "gelu" (exact erf form), "silu" or "gelu_tanh".  ``residual``:
    an M x N row-major tensor of C's type (fp16 for out="f16", fp32 for
    out="f32"); it may be ``C`` itself for an in-place residual connection.
    Operands and ``op_a`` / ``op_b`` as ``tlg_gemm_op``."""
    at, bt = op_a.upper() == "T", op_b.upper() == "T"
    if A.dtype != torch.float16 or B.dtype != torch.float16:
        raise TypeError("A and B must be fp16")
    M, K = (A.shape[1], A.shape[0]) if at else tuple(A.shape)
    K2, N = (B.shape[1], B.shape[0]) if bt else tuple(B.shape)
    if K != K2:
        raise ValueError(f"inner dimensions differ: op(A) is {M}x{K}, op(B) is {K2}x{N}")
    if activation not in _ACT:
        raise ValueError(f"activation must be one of {sorted(_ACT)}")
    o = TLG_OUT_F32 if out == "f32" else TLG_OUT_F16
    cdt = torch.float32 if o == TLG_OUT_F32 else torch.float16
    C = _out(C, M, N, cdt, A)
    if bias is not None and (bias.dtype != torch.float16 or bias.dim() != 1 or bias.numel() != N
                             or (N > 1 and bias.stride(0) != 1)):
        raise ValueError(f"bias must be a contiguous fp16 vector of length {N}")
    epi = tlg_fused_epilogue(bias.data_ptr() if bias is not None else None, _ACT[activation], None, 0)
    if residual is not None:
        if residual.dtype != cdt or tuple(residual.shape) != (M, N):
            raise ValueError(f"residual must be {cdt} of shape ({M}, {N})")
        epi.residual, epi.ldr = _mat(residual, "residual")
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    cfg = tlg_config(**{k: int(v) for k, v in config.items()}) if config is not None else None
    ws_ptr, ws_bytes = (None, 0)
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check(_lib.tlg_gemm_fused(M, N, K, TLG_OP_T if at else TLG_OP_N, pa, lda, TLG_OP_T if bt else TLG_OP_N,
                               pb, ldb, ctypes.byref(epi), pc, ldc, o,
                               ctypes.byref(cfg) if cfg is not None else None, ws_ptr, ws_bytes,
                               _stream_handle(stream, A, B, C)), "tlg_gemm_fused")
    return C


def tlg_gemm_ex_noalloc(A: torch.Tensor, B: torch.Tensor, bias: torch.Tensor | None = None,
                        C: torch.Tensor | None = None, out: str = "f32", config: dict | None = None,
                        stream=None):
    """tlg_gemm_ex with the library's static scratch instead of a workspace (see tlg.h).
    Allocates nothing in the library; C is allocated here only when not given."""
    M, N, K = _shapes(A, B)
    o = TLG_OUT_F32 if out == "f32" else TLG_OUT_F16
    C = _out(C, M, N, torch.float32 if o == TLG_OUT_F32 else torch.float16, A)
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    pc, ldc = _mat(C, "C")
    cfg = tlg_config(**{k: int(v) for k, v in config.items()}) if config is not None else None
    epi = TLG_EPI_BIAS_RELU if bias is not None else TLG_EPI_NONE
    _check(_lib.tlg_gemm_ex_noalloc(M, N, K, pa, lda, pb, ldb, bias.data_ptr() if bias is not None else None,
                                    pc, ldc, o, epi, ctypes.byref(cfg) if cfg is not None else None,
                                    _stream_handle(stream, A, B, C)), "tlg_gemm_ex_noalloc")
    return C


def tlg_gemm_workspace_size(M: int, N: int, K: int, out: str = "f32", bias_relu: bool = False,
                            config: dict | None = None) -> int:
    cfg = tlg_config(**{k: int(v) for k, v in config.items()}) if config else None
    n = ctypes.c_size_t(0)
    _check(_lib.tlg_gemm_workspace_size(M, N, K, TLG_OUT_F32 if out == "f32" else TLG_OUT_F16,
                                        TLG_EPI_BIAS_RELU if bias_relu else TLG_EPI_NONE,
                                        ctypes.byref(cfg) if cfg is not None else None, ctypes.byref(n)),
           "tlg_gemm_workspace_size")
    return int(n.value)


def tlg_gemm_workspace_size_op(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor | None = None,
                               op_a: str = "N", op_b: str = "N", out: str = "f16",
                               config: dict | None = None) -> int:
    """Workspace bytes for a call on these operands: the split-K scratch plus aligned copies of
    the matrices TMA cannot describe (see tlg.h).  C = None assumes an aligned C."""
    at, bt = op_a.upper() == "T", op_b.upper() == "T"
    M, K = (A.shape[1], A.shape[0]) if at else tuple(A.shape)
    N = B.shape[0] if bt else B.shape[1]
    pa, lda = _mat(A, "A")
    pb, ldb = _mat(B, "B")
    esz = 4 if out == "f32" else 2
    if C is None:
        pc, ldc = 1 << 20, ((N * esz + 15) // 16 * 16) // esz  # a stand-in aligned C
    else:
        pc, ldc = _mat(C, "C")
    cfg = tlg_config(**{k: int(v) for k, v in config.items()}) if config else None
    n = ctypes.c_size_t(0)
    _check(_lib.tlg_gemm_workspace_size_op(M, N, K, TLG_OP_T if at else TLG_OP_N, pa, lda,
                                           TLG_OP_T if bt else TLG_OP_N, pb, ldb, pc, ldc,
                                           TLG_OUT_F32 if out == "f32" else TLG_OUT_F16,
                                           ctypes.byref(cfg) if cfg is not None else None, ctypes.byref(n)),
           "tlg_gemm_workspace_size_op")
    return int(n.value)


def tlg_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled device workspace of at least ``nbytes`` (torch's allocator; 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")


def tlg_choose_config(M: int, N: int, K: int, out: str = "f32", bias_relu: bool = False,
                      request: dict | None = None) -> dict:
    """The configuration tlg_gemm_ex would run for this shape (request fields of 0 = automatic)."""
    cfg = tlg_config(**{k: int(v) for k, v in (request or {}).items()})
    _check(_lib.tlg_choose_config(M, N, K, TLG_OUT_F32 if out == "f32" else TLG_OUT_F16,
                                  TLG_EPI_BIAS_RELU if bias_relu else TLG_EPI_NONE, ctypes.byref(cfg)),
           "tlg_choose_config")
    return cfg.as_dict()


def tlg_device_error(clear: bool = True):
    """(status, raw word) of the device error word of the current device; synchronizes."""
    code = ctypes.c_uint32(0)
    rc = _lib.tlg_device_error(int(bool(clear)), ctypes.byref(code))
    return rc, int(code.value)


def tlg_selftest_timeout(limit_us: int, stream=None):
    _check(_lib.tlg_selftest_timeout(int(limit_us), _stream_handle(stream)), "tlg_selftest_timeout")


def raw_library():
    """The ctypes handle of libtlg.so, for callers that marshal their own pointers."""
    return _lib

"""Helpers for the GPU tests: padded device operands with NaN guard bands, and
calls into libtlg through the Python binding (which marshals to the C ABI)."""

from __future__ import annotations

import numpy as np
import torch

POISON_F16 = 0x7E01      # a quiet NaN pattern
POISON_F32 = 0x7FC00001


def round_up(x, m):
    return (x + m - 1) // m * m


class Padded:
    """A rows x cols matrix inside a larger device buffer: one guard row above,
    two below, and `extra` padding columns, all filled with a NaN pattern."""

    def __init__(self, host: torch.Tensor | None, rows, cols, dtype, align_elems, extra=0, device="cuda"):
        self.rows, self.cols, self.dtype = rows, cols, dtype
        self.ld = max(round_up(cols + extra, align_elems), align_elems)
        int_dtype = torch.int16 if dtype == torch.float16 else torch.int32
        poison = POISON_F16 if dtype == torch.float16 else POISON_F32
        if poison >= 2 ** (8 * (2 if dtype == torch.float16 else 4) - 1):
            poison -= 2 ** (8 * (2 if dtype == torch.float16 else 4))
        self.poison = poison
        self.buf = torch.full((rows + 3, self.ld), poison, dtype=int_dtype, device=device).view(dtype)
        self.view = self.buf[1:1 + rows, :cols]
        if host is not None:
            self.view.copy_(host.to(device))

    def ptr(self):
        return self.buf.data_ptr() + self.ld * self.buf.element_size()

    def guard_changes(self):
        """Buffer positions (row, col) outside the matrix whose poison was overwritten."""
        bits = self.buf.view(torch.int16 if self.dtype == torch.float16 else torch.int32)
        mask = torch.ones_like(bits, dtype=torch.bool)
        mask[1:1 + self.rows, :self.cols] = False
        bad = mask & (bits != self.poison)
        return [tuple(x) for x in bad.nonzero().tolist()[:8]]

    def guard_intact(self) -> bool:
        return not self.guard_changes()


def gemm_padded(lib, A: torch.Tensor, B: torch.Tensor, bias: torch.Tensor | None, out: str,
                config: dict | None = None, extra=(0, 0, 0), stream=None, workspace=None):
    """Run one GEMM through tlg_gemm_ex on padded operands; returns (C as float64 numpy, guards ok)."""
    import ctypes

    import tiled_dense_gemm_tlg_b200 as tlg

    M, K = A.shape
    N = B.shape[1]
    esz_out = 4 if out == "f32" else 2
    pa = Padded(A, M, K, torch.float16, 8, extra[0])
    pb = Padded(B, K, N, torch.float16, 8, extra[1])
    pc = Padded(None, M, N, torch.float32 if out == "f32" else torch.float16, 16 // esz_out, extra[2])
    pbias = None
    if bias is not None:
        pbias = bias.to("cuda").contiguous()
    cfg = None
    if config is not None:
        cfg = tlg.tlg_config(**{k: int(v) for k, v in config.items()})
    st = int(stream.cuda_stream) if stream is not None else int(torch.cuda.current_stream().cuda_stream)
    rc = lib.tlg_gemm_ex(M, N, K, pa.ptr(), pa.ld, pb.ptr(), pb.ld,
                         pbias.data_ptr() if pbias is not None else None, pc.ptr(), pc.ld,
                         tlg.TLG_OUT_F32 if out == "f32" else tlg.TLG_OUT_F16,
                         tlg.TLG_EPI_BIAS_RELU if bias is not None else tlg.TLG_EPI_NONE,
                         ctypes.byref(cfg) if cfg is not None else None,
                         workspace.data_ptr() if workspace is not None else None,
                         workspace.numel() if workspace is not None else 0, st)
    if rc != 0:
        raise tlg.TlgError(rc, "tlg_gemm_ex")
    torch.cuda.synchronize()
    changes = {name: b.guard_changes() for name, b in (("A", pa), ("B", pb), ("C", pc))}
    return pc.view.double().cpu().numpy(), GuardReport(changes)


class GuardReport:
    """Truthy when no guard element changed; its repr names the changed positions."""

    def __init__(self, changes):
        self.changes = {k: v for k, v in changes.items() if v}

    def __bool__(self):
        return not self.changes

    def __repr__(self):
        return f"guard changes (buffer row, col) {self.changes}"

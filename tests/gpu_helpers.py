"""Shared helpers for the GPU parity tests: canary-guarded output buffers,
C-ABI calls on torch tensors, and the tolerance comparison against the
oracle.  Expected values come only from oracle/ (or, for the exact-integer
cases, from torch rounding the oracle's exact value)."""
import os

import numpy as np
import torch

import dense_gemm_16_b200 as dg
import oracle

THREADS = max(1, min(32, os.cpu_count() or 1))

# |got - ref| <= atol + rtol*|ref|: 1e-2 for fp16/bf16 outputs, 1e-3 for fp32
TOL = {2: (1e-2, 1e-2), 4: (1e-3, 1e-3)}

_SENT16 = 0x7E5A          # a NaN pattern no finite result can produce
_SENT32 = 0x7FC0DEAD


def torch_dtype(code):
    return {dg.GEMM_F16: torch.float16, dg.GEMM_BF16: torch.bfloat16,
            dg.GEMM_F16_OUT_F32: torch.float32, dg.GEMM_BF16_OUT_F32: torch.float32}[code]


def in_name(t: torch.Tensor) -> str:
    return "bf16" if t.dtype == torch.bfloat16 else "f16"


class Guarded:
    """An M x N output with leading dimension ldc inside a sentinel-filled
    buffer: pad elements before and after, and ldc - N pad columns per row."""

    def __init__(self, M, N, ldc, dtype, pad=128):
        self.M, self.N, self.ldc, self.pad = M, N, ldc, pad
        self.buf = torch.empty(pad + M * ldc + pad, dtype=dtype, device="cuda")
        self.ibuf = self.buf.view(torch.int32 if dtype == torch.float32 else torch.int16)
        self.sent = _SENT32 if dtype == torch.float32 else _SENT16
        self.ibuf.fill_(self.sent)
        self.ptr = self.buf.data_ptr() + pad * self.buf.element_size()

    def matrix(self) -> torch.Tensor:
        return self.buf[self.pad:self.pad + self.M * self.ldc].view(self.M, self.ldc)[:, :self.N]

    def check_canaries(self):
        raw = self.ibuf.cpu()
        assert bool((raw[:self.pad] == self.sent).all()), "write before C"
        assert bool((raw[self.pad + self.M * self.ldc:] == self.sent).all()), "write after C"
        if self.ldc > self.N and self.M > 0:
            body = raw[self.pad:self.pad + self.M * self.ldc].view(self.M, self.ldc)
            assert bool((body[:, self.N:] == self.sent).all()), "write into ldc padding"


def run_gemm(A, B, bias, M, N, K, *, b_col=False, relu=False, out_f32=False, ldc=None,
             stream=None, expect_rc=0):
    """Launch gemm() through the C ABI on device tensors; returns the guard."""
    code = dg.dtype_code(A.dtype, out_f32)
    ldc = ldc or ((N + 7) // 8 * 8)
    g = Guarded(M, N, ldc, torch.float32 if out_f32 else A.dtype)
    epi = (dg.GEMM_EPI_BIAS if bias is not None else 0) | (dg.GEMM_EPI_RELU if relu else 0) | \
        (dg.GEMM_B_COL_MAJOR if b_col else 0)
    rc = dg.gemm(M, N, K, A if K else None, A.stride(0) if K else 0, B if K else None,
                 B.stride(0) if K else 0, g.ptr, ldc, bias, epi, code, stream)
    assert rc == expect_rc, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status(stream) == 0
    return g


def compare(got: np.ndarray, ref: np.ndarray, out_bytes: int, what=""):
    atol, rtol = TOL[out_bytes]
    ok, max_abs, max_rel, worst = oracle.within_tolerance(got, ref, atol, rtol)
    assert ok, (f"{what}: max|err|={max_abs:.3e} max rel={max_rel:.3e} worst flat index "
                f"{worst}: got {got.ravel()[worst]!r} ref {ref.ravel()[worst]!r}")
    return max_abs


def pad_cols(x: torch.Tensor, ld: int) -> torch.Tensor:
    """A copy of 2-D x stored with leading dimension ld (>= x.shape[1])."""
    r, c = x.shape
    buf = torch.full((r, ld), float("nan"), dtype=x.dtype, device=x.device)
    buf[:, :c] = x
    return buf[:, :c]

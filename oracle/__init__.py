"""CPU oracle for the dense GEMM path -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``dense_gemm_16_b200``) never imports, links or calls it, and the two share
no code: the oracle is plain C (``gemm_oracle.c``) compiled with gcc, with its
own IEEE binary16 / bfloat16 decoders, and this module only marshals numpy
arrays into it.

What it computes (plain definition, fp64 accumulation, k ascending):

    C[i, j] = act( sum_k A[i, k] * B[k, j] + bias[j] ),   act in {identity, ReLU}

following "用Triton跨芯片优化GEMM" sections 2.1 (the tiled kernel's result) and
3.4 (bias + ReLU fused after the GEMM), and "Triton 学习笔记" section 2.1
(accumulate wider than the inputs).  The grouped variant applies the same
definition per group of rows ("用Triton跨芯片优化GEMM" section 2.3, the MoE
layer's many GEMMs).

Every function here is pinned by ``tests/test_oracle.py`` against things
other than itself: torch's own fp16/bf16 conversions over all 65536 bit
patterns, pure-Python brute force on tiny integer inputs, identity and
permutation matrices, all-ones closed forms, linearity, and hand-worked
golden cases under ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gemm_oracle.c")
_LIB = os.path.join(_HERE, "_gemm_oracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16 = 0, 1
_DTYPES = {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-Wall",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point the wrapper at a deliberately broken build of
            # the oracle (tests/test_oracle_mutations.py) to show the pins fail.
            override = os.environ.get("GEMM_ORACLE_LIB")
            if override:
                lib = ctypes.CDLL(override)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            u16p = ctypes.POINTER(ctypes.c_uint16)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            i32p = ctypes.POINTER(ctypes.c_int32)
            I, L = ctypes.c_int, ctypes.c_int64
            lib.oracle_decode_f16.restype = ctypes.c_double
            lib.oracle_decode_f16.argtypes = [ctypes.c_uint16]
            lib.oracle_decode_bf16.restype = ctypes.c_double
            lib.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
            lib.oracle_decode_array.argtypes = [u16p, L, I, f64p]
            lib.oracle_gemm_f64.argtypes = [I, I, I, f64p, L, f64p, L, I, f64p, I, f64p, L, I]
            lib.oracle_gemm.argtypes = [I, I, I, u16p, L, u16p, L, I, u16p, I, I, f64p, L, I]
            f32p = ctypes.POINTER(ctypes.c_float)
            lib.oracle_gemm_f32.argtypes = [I, I, I, f32p, L, f32p, L, I, f32p, I, f64p, L, I]
            lib.oracle_gemm_at.argtypes = [I, I, I, u16p, L, u16p, L, I, u16p, I, I,
                                           L, i64p, i64p, f64p, I]
            lib.oracle_grouped_gemm.argtypes = [I, i32p, I, I, u16p, L, u16p, L, L, I,
                                                u16p, I, I, f64p, L, I]
            lib.oracle_grouped_gemm_at.argtypes = [I, i32p, I, I, u16p, L, u16p, L, L, I,
                                                   u16p, I, I, L, i64p, i64p, f64p, I]
            lib.oracle_threads_used.argtypes = [I]
            lib.oracle_conv2d_nhwc.argtypes = [I] * 13 + [u16p, u16p, u16p, I, I, f64p, I]
            _lib = lib
    return _lib


def _dt(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    key = str(dtype).replace("torch.", "")
    if key not in _DTYPES:
        raise ValueError(f"oracle: unsupported dtype {dtype!r}")
    return _DTYPES[key]


def _bits(x) -> np.ndarray:
    """Raw 16-bit patterns of a numpy uint16/float16 array or a torch fp16/bf16 tensor."""
    if hasattr(x, "detach"):  # torch tensor -> its bit patterns, no value conversion
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype in (torch.float16, torch.bfloat16):
            x = x.view(torch.int16)
        x = x.numpy()
    x = np.ascontiguousarray(x)
    if x.dtype.itemsize != 2:
        raise TypeError("oracle: expected a 16-bit array")
    return x.view(np.uint16).reshape(-1)


def _p(arr, ctype):
    if arr is None:
        return None
    return arr.ctypes.data_as(ctypes.POINTER(ctype))


def _rc(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle: {what} rejected its arguments (rc={rc})")


def threads_used(nthreads: int) -> int:
    return int(_load().oracle_threads_used(int(nthreads)))


def decode(bits, dtype) -> np.ndarray:
    """fp16 / bf16 bit patterns -> float64, by the oracle's own decoders."""
    b = _bits(bits)
    out = np.empty(b.size, dtype=np.float64)
    _rc(_load().oracle_decode_array(_p(b, ctypes.c_uint16), b.size, _dt(dtype),
                                    _p(out, ctypes.c_double)), "decode")
    return out


def decode_scalar(h: int, dtype) -> float:
    lib = _load()
    return lib.oracle_decode_bf16(h) if _dt(dtype) == BF16 else lib.oracle_decode_f16(h)


def gemm_f64(A: np.ndarray, B: np.ndarray, bias=None, relu=False, b_colmajor=False,
             threads: int = 1) -> np.ndarray:
    """The definition on float64 operands.  A is (M, K); B is (K, N), or
    (N, K) when ``b_colmajor``."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0] if b_colmajor else B.shape[1]
    if (B.shape[1] if b_colmajor else B.shape[0]) != K:
        raise ValueError("oracle: inner dimensions differ")
    bs = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    out = np.zeros((M, N), dtype=np.float64)
    _rc(_load().oracle_gemm_f64(M, N, K, _p(A, ctypes.c_double), K, _p(B, ctypes.c_double),
                                B.shape[1], int(bool(b_colmajor)), _p(bs, ctypes.c_double),
                                int(bool(relu)), _p(out, ctypes.c_double), N, threads),
        "gemm_f64")
    return out


def gemm(M, N, K, A, lda, B, ldb, *, b_colmajor=False, bias=None, relu=False,
         dtype="f16", threads: int = 1) -> np.ndarray:
    """Full (M, N) float64 result from 16-bit buffers addressed through lda/ldb."""
    a = None if A is None else _bits(A)
    b = None if B is None else _bits(B)
    bs = None if bias is None else _bits(bias)
    out = np.zeros((M, N), dtype=np.float64)
    _rc(_load().oracle_gemm(M, N, K, _p(a, ctypes.c_uint16), lda, _p(b, ctypes.c_uint16), ldb,
                            int(bool(b_colmajor)), _p(bs, ctypes.c_uint16), int(bool(relu)),
                            _dt(dtype), _p(out, ctypes.c_double), max(N, 1), threads), "gemm")
    return out


def _f32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    x = np.ascontiguousarray(x)
    if x.dtype != np.float32:
        raise TypeError("oracle: expected float32 data")
    return x.reshape(-1)


def gemm_f32(M, N, K, A, lda, B, ldb, *, b_colmajor=False, bias=None, relu=False,
             threads: int = 1) -> np.ndarray:
    """Full (M, N) float64 result from fp32 buffers addressed through lda/ldb
    (the exact product of the fp32 values, before any tf32 rounding)."""
    a, b, bs = _f32(A), _f32(B), _f32(bias)
    out = np.zeros((M, N), dtype=np.float64)
    _rc(_load().oracle_gemm_f32(M, N, K, _p(a, ctypes.c_float), lda, _p(b, ctypes.c_float), ldb,
                                int(bool(b_colmajor)), _p(bs, ctypes.c_float), int(bool(relu)),
                                _p(out, ctypes.c_double), max(N, 1), threads), "gemm_f32")
    return out


def gemm_at(M, N, K, A, lda, B, ldb, rows, cols, *, b_colmajor=False, bias=None,
            relu=False, dtype="f16", threads: int = 1) -> np.ndarray:
    """C[rows[t], cols[t]] for each t, computed element by element."""
    a = None if A is None else _bits(A)
    b = None if B is None else _bits(B)
    bs = None if bias is None else _bits(bias)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.zeros(r.size, dtype=np.float64)
    _rc(_load().oracle_gemm_at(M, N, K, _p(a, ctypes.c_uint16), lda, _p(b, ctypes.c_uint16),
                               ldb, int(bool(b_colmajor)), _p(bs, ctypes.c_uint16),
                               int(bool(relu)), _dt(dtype), r.size, _p(r, ctypes.c_int64),
                               _p(c, ctypes.c_int64), _p(out, ctypes.c_double), threads),
        "gemm_at")
    return out


def grouped_gemm(group_rows, N, K, A, lda, B, ldb, strideB, *, b_colmajor=False, bias=None,
                 relu=False, dtype="bf16", threads: int = 1) -> np.ndarray:
    """Full (sum(group_rows), N) float64 result of the grouped GEMM."""
    g = np.ascontiguousarray(group_rows, dtype=np.int32)
    total = int(g.astype(np.int64).sum())
    a = None if A is None else _bits(A)
    b = None if B is None else _bits(B)
    bs = None if bias is None else _bits(bias)
    out = np.zeros((total, N), dtype=np.float64)
    _rc(_load().oracle_grouped_gemm(g.size, _p(g, ctypes.c_int32), N, K, _p(a, ctypes.c_uint16),
                                    lda, _p(b, ctypes.c_uint16), ldb, strideB,
                                    int(bool(b_colmajor)), _p(bs, ctypes.c_uint16),
                                    int(bool(relu)), _dt(dtype), _p(out, ctypes.c_double),
                                    max(N, 1), threads), "grouped_gemm")
    return out


def grouped_gemm_at(group_rows, N, K, A, lda, B, ldb, strideB, rows, cols, *, b_colmajor=False,
                    bias=None, relu=False, dtype="bf16", threads: int = 1) -> np.ndarray:
    """Sampled grouped GEMM; rows are global row indices."""
    g = np.ascontiguousarray(group_rows, dtype=np.int32)
    a = None if A is None else _bits(A)
    b = None if B is None else _bits(B)
    bs = None if bias is None else _bits(bias)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.zeros(r.size, dtype=np.float64)
    _rc(_load().oracle_grouped_gemm_at(g.size, _p(g, ctypes.c_int32), N, K,
                                       _p(a, ctypes.c_uint16), lda, _p(b, ctypes.c_uint16), ldb,
                                       strideB, int(bool(b_colmajor)), _p(bs, ctypes.c_uint16),
                                       int(bool(relu)), _dt(dtype), r.size,
                                       _p(r, ctypes.c_int64), _p(c, ctypes.c_int64),
                                       _p(out, ctypes.c_double), threads), "grouped_gemm_at")
    return out


def within_tolerance(got: np.ndarray, ref: np.ndarray, atol: float, rtol: float):
    """|got - ref| <= atol + rtol*|ref| elementwise ("Triton 学习笔记" 2.1); any
    NaN/Inf in got fails.  Returns (ok, max_abs_err, max_rel_err, worst_index)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    finite = np.isfinite(got)
    ok_mask = finite & (err <= bound)
    ok = bool(ok_mask.all())
    if err.size == 0:
        return True, 0.0, 0.0, -1
    excess = np.where(finite, err - bound, np.inf)
    worst = int(np.argmax(excess))
    rel = err / np.maximum(np.abs(ref), 1e-30)
    return ok, float(np.nanmax(err)), float(np.nanmax(np.where(np.abs(ref) > 0, rel, 0.0))), worst


def conv_out_size(H, W, KH, KW, stride=(1, 1), pad=(0, 0), dil=(1, 1)):
    OH = (H + 2 * pad[0] - dil[0] * (KH - 1) - 1) // stride[0] + 1
    OW = (W + 2 * pad[1] - dil[1] * (KW - 1) - 1) // stride[1] + 1
    return OH, OW


def conv2d_nhwc(x, w, *, stride=(1, 1), pad=(0, 0), dil=(1, 1), bias=None, relu=False,
                dtype="f16", threads: int = 1) -> np.ndarray:
    """Direct NHWC convolution: x (batch, H, W, cin), w (KH, KW, cin, cout)
    -> (batch, OH, OW, cout) float64."""
    batch, H, W, cin = x.shape
    KH, KW, cin2, cout = w.shape
    if cin2 != cin:
        raise ValueError("oracle: channel counts differ")
    OH, OW = conv_out_size(H, W, KH, KW, stride, pad, dil)
    xb, wb = _bits(x), _bits(w)
    bs = None if bias is None else _bits(bias)
    out = np.zeros((batch, OH, OW, cout), dtype=np.float64)
    _rc(_load().oracle_conv2d_nhwc(batch, H, W, cin, cout, KH, KW, stride[0], stride[1], pad[0],
                                   pad[1], dil[0], dil[1], _p(xb, ctypes.c_uint16),
                                   _p(wb, ctypes.c_uint16), _p(bs, ctypes.c_uint16),
                                   int(bool(relu)), _dt(dtype), _p(out, ctypes.c_double),
                                   threads), "conv2d_nhwc")
    return out

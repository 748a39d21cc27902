"""dense_gemm_16_b200 -- Python binding of the B200 tiled GEMM library.

This module only marshals arguments into the C ABI declared in
``include/dense_gemm.h`` (``libdense_gemm.so``, built in-tree by
``python -m dense_gemm_16_b200.build``).  Every step of the computation runs
in the library's CUDA kernels; there is no Python, PyTorch or CPU fallback.
If the library is missing, importing works but every call raises.

The names mirror the C ABI: ``gemm``, ``grouped_gemm``, ``gemm_status_string``,
``gemm_device_status``, ...  Tensor arguments may be torch tensors (their
``data_ptr()`` is passed) or raw integer addresses.  ``matmul`` and
``grouped_matmul`` are conveniences that allocate the output with torch and
call the same entry points.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdense_gemm.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "dense_gemm.h")

GEMM_OK = 0
GEMM_ERR_INVALID_ARG = -1
GEMM_ERR_UNSUPPORTED = -2
GEMM_ERR_MISALIGNED = -3
GEMM_ERR_CUDA = -4
GEMM_ERR_DEVICE_TIMEOUT = -5

GEMM_F16, GEMM_BF16, GEMM_F16_OUT_F32, GEMM_BF16_OUT_F32, GEMM_F32_TF32 = 0, 1, 2, 3, 4
GEMM_EPI_BIAS = 0x1
GEMM_EPI_RELU = 0x2
GEMM_B_COL_MAJOR = 0x100

# trace events (gemm_set_trace): column of a block's row in the trace buffer
(GEMM_TRACE_ENTRY, GEMM_TRACE_SETUP, GEMM_TRACE_FIRST_LOAD, GEMM_TRACE_FIRST_DATA,
 GEMM_TRACE_LAST_MMA, GEMM_TRACE_FIRST_EPI, GEMM_TRACE_EPI_DONE, GEMM_TRACE_EXIT) = range(8)
GEMM_TRACE_EVENTS = 8

_lib = None
_lock = threading.Lock()


class GemmError(RuntimeError):
    def __init__(self, status: int, what: str = "gemm"):
        self.status = status
        super().__init__(f"{what}: {gemm_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with `python -m dense_gemm_16_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            I, U, L64, P = ctypes.c_int, ctypes.c_uint, ctypes.c_int64, ctypes.c_void_p
            L.gemm.argtypes = [I, I, I, P, L64, P, L64, P, L64, P, U, I, P]
            L.gemm.restype = I
            L.grouped_gemm.argtypes = [I, P, I, I, I, P, L64, P, L64, L64, P, L64, P, U, I, P]
            L.grouped_gemm.restype = I
            L.gemm_status_string.argtypes = [I]
            L.gemm_status_string.restype = ctypes.c_char_p
            L.gemm_version.restype = ctypes.c_char_p
            L.gemm_device_status.argtypes = [P, I]
            L.gemm_set_timeout_ns.argtypes = [ctypes.c_uint64]
            L.gemm_set_timeout_ns.restype = ctypes.c_uint64
            L.gemm_watchdog_selftest.argtypes = [ctypes.c_uint64, P]
            L.gemm_config_name.argtypes = [I, ctypes.c_char_p, I]
            L.gemm_select_config.argtypes = [I, I, I, I, U]
            L.gemm_force_config.argtypes = [I]
            L.gemm_smem_ring_bytes.argtypes = [I, I, I, I, I]
            L.gemm_smem_ring_bytes.restype = ctypes.c_int64
            L.gemm_k_iterations.argtypes = [I, I]
            L.gemm_tile_coord.argtypes = [ctypes.c_int64, I, I, I, ctypes.POINTER(I),
                                          ctypes.POINTER(I)]
            L.gemm_strided_batched.argtypes = [I, I, I, I, P, L64, L64, P, L64, L64, P, L64, L64,
                                               P, L64, U, I, P]
            L.gemm_strided_batched.restype = I
            L.conv2d_im2col.argtypes = [I] * 13 + [P, P, P, P, U, I, P]
            L.conv2d_im2col.restype = I
            L.gemm_splitk_noalloc.argtypes = [I, I, I, P, L64, P, L64, P, L64, P, U, I, I, P]
            L.gemm_splitk_noalloc.restype = I
            L.gemm_set_trace.argtypes = [P, L64]
            L.gemm_set_trace.restype = I
            L.gemm_free_scratch.argtypes = [P, I]
            L.gemm_free_scratch.restype = I
            _lib = L
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------- raw C ABI

def gemm(M, N, K, A, lda, B, ldb, C, ldc, bias, epilogue, dtype, stream=None) -> int:
    """C-ABI ``gemm``; returns the gemm_status."""
    return lib().gemm(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(C), ldc, _ptr(bias),
                      epilogue, dtype, _stream(stream))


def gemm_strided_batched(batch, M, N, K, A, lda, stride_a, B, ldb, stride_b, C, ldc, stride_c,
                         bias, stride_bias, epilogue, dtype, stream=None) -> int:
    """C-ABI ``gemm_strided_batched``; returns the gemm_status."""
    return lib().gemm_strided_batched(batch, M, N, K, _ptr(A), lda, stride_a, _ptr(B), ldb,
                                      stride_b, _ptr(C), ldc, stride_c, _ptr(bias), stride_bias,
                                      epilogue, dtype, _stream(stream))


def grouped_gemm(num_groups, group_rows, total_rows, N, K, A, lda, B, ldb, stride_b, C, ldc,
                 bias, epilogue, dtype, stream=None) -> int:
    """C-ABI ``grouped_gemm``; returns the gemm_status."""
    return lib().grouped_gemm(num_groups, _ptr(group_rows), total_rows, N, K, _ptr(A), lda,
                              _ptr(B), ldb, stride_b, _ptr(C), ldc, _ptr(bias), epilogue, dtype,
                              _stream(stream))


def gemm_splitk_noalloc(M, N, K, A, lda, B, ldb, C, ldc, bias, epilogue, dtype, splits,
                        stream=None) -> int:
    """C-ABI ``gemm_splitk_noalloc`` (split-K with the library's fixed
    scratch, no device allocation); returns the gemm_status."""
    return lib().gemm_splitk_noalloc(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(C), ldc,
                                     _ptr(bias), epilogue, dtype, splits, _stream(stream))


def conv2d_im2col(batch, H, W, cin, cout, KH, KW, stride_h, stride_w, pad_h, pad_w, dil_h,
                  dil_w, x, w, y, bias, epilogue, dtype, stream=None) -> int:
    """C-ABI ``conv2d_im2col``; returns the gemm_status."""
    return lib().conv2d_im2col(batch, H, W, cin, cout, KH, KW, stride_h, stride_w, pad_h, pad_w,
                               dil_h, dil_w, _ptr(x), _ptr(w), _ptr(y), _ptr(bias), epilogue,
                               dtype, _stream(stream))


def gemm_status_string(status: int) -> str:
    try:
        return lib().gemm_status_string(status).decode()
    except ImportError:
        return f"status {status}"


def gemm_version() -> str:
    return lib().gemm_version().decode()


def gemm_device_status(stream=None, clear: bool = True) -> int:
    return lib().gemm_device_status(_stream(stream), int(clear))


def gemm_free_scratch(stream=None, all_streams: bool = False) -> int:
    """C-ABI ``gemm_free_scratch``: free the library's scratch for ``stream``
    (the current stream by default), or for every stream with all_streams."""
    return lib().gemm_free_scratch(None if all_streams else _stream(stream),
                                   1 if all_streams else 0)


def gemm_set_trace(buffer, nbytes: int) -> int:
    """C-ABI ``gemm_set_trace``: per-block event times of later launches go
    to ``buffer`` (device memory, ``nbytes`` long); ``None`` turns tracing off."""
    return lib().gemm_set_trace(_ptr(buffer), nbytes)


def gemm_set_timeout_ns(ns: int) -> int:
    return lib().gemm_set_timeout_ns(ns)


def gemm_watchdog_selftest(timeout_ns: int, stream=None) -> int:
    return lib().gemm_watchdog_selftest(timeout_ns, _stream(stream))


def gemm_num_configs() -> int:
    return lib().gemm_num_configs()


def gemm_config_name(i: int) -> str:
    buf = ctypes.create_string_buffer(128)
    rc = lib().gemm_config_name(i, buf, 128)
    if rc:
        raise GemmError(rc, "gemm_config_name")
    return buf.value.decode()


def gemm_select_config(M, N, K, dtype, epilogue) -> int:
    return lib().gemm_select_config(M, N, K, dtype, epilogue)


def gemm_force_config(i: int) -> int:
    return lib().gemm_force_config(i)


def gemm_smem_ring_bytes(bm, bn, bk, stages, elem_bytes) -> int:
    return lib().gemm_smem_ring_bytes(bm, bn, bk, stages, elem_bytes)


def gemm_k_iterations(K, bk) -> int:
    return lib().gemm_k_iterations(K, bk)


def gemm_tile_coord(tile, grid_m, grid_n, group_m):
    m, n = ctypes.c_int(), ctypes.c_int()
    rc = lib().gemm_tile_coord(tile, grid_m, grid_n, group_m, ctypes.byref(m), ctypes.byref(n))
    if rc:
        raise GemmError(rc, "gemm_tile_coord")
    return m.value, n.value


# ------------------------------------------------------- torch helpers

def dtype_code(in_dtype, out_f32: bool = False) -> int:
    import torch
    if in_dtype == torch.float16:
        return GEMM_F16_OUT_F32 if out_f32 else GEMM_F16
    if in_dtype == torch.bfloat16:
        return GEMM_BF16_OUT_F32 if out_f32 else GEMM_BF16
    if in_dtype == torch.float32:  # multiplied as tf32, fp32 out
        return GEMM_F32_TF32
    raise TypeError(f"unsupported input dtype {in_dtype}")


def matmul(a, b, bias=None, relu: bool = False, b_col_major: bool = False, out=None,
           out_f32: bool = False, stream=None):
    """C = act(a @ B + bias) through the C ABI.

    a: (M, K) device tensor with unit column stride.  b: (K, N) with unit
    column stride, or with ``b_col_major`` the (N, K) storage of B.  The
    output is allocated with torch unless ``out`` is given."""
    import torch
    M, K = a.shape
    N = b.shape[0] if b_col_major else b.shape[1]
    code = dtype_code(a.dtype, out_f32)
    if out is None:
        out = torch.empty(M, N, device=a.device,
                          dtype=torch.float32 if (out_f32 or code == GEMM_F32_TF32) else a.dtype)
    epi = (GEMM_EPI_BIAS if bias is not None else 0) | (GEMM_EPI_RELU if relu else 0) | \
        (GEMM_B_COL_MAJOR if b_col_major else 0)
    rc = gemm(M, N, K, a, a.stride(0), b, b.stride(0), out, out.stride(0), bias, epi, code,
              stream)
    if rc:
        raise GemmError(rc)
    return out


def bmm(a, b, bias=None, relu: bool = False, b_col_major: bool = False, out=None,
        out_f32: bool = False, stream=None):
    """Strided-batched C_i = act(a_i @ B_i + bias_i) through the C ABI.

    a: (batch, M, K); b: (batch, K, N), or (batch, N, K) with
    ``b_col_major`` (a batch stride of 0 -- e.g. from ``expand`` -- shares
    one operand across batches); bias: (batch, N) or (N,) or None."""
    import torch
    batch, M, K = a.shape
    N = b.shape[1] if b_col_major else b.shape[2]
    code = dtype_code(a.dtype, out_f32)
    if out is None:
        out = torch.empty(batch, M, N, device=a.device,
                          dtype=torch.float32 if out_f32 else a.dtype)
    epi = (GEMM_EPI_BIAS if bias is not None else 0) | (GEMM_EPI_RELU if relu else 0) | \
        (GEMM_B_COL_MAJOR if b_col_major else 0)
    sbias = 0 if bias is None or bias.dim() == 1 else bias.stride(0)
    rc = gemm_strided_batched(batch, M, N, K, a, a.stride(1), a.stride(0), b, b.stride(1),
                              b.stride(0), out, out.stride(1), out.stride(0), bias, sbias, epi,
                              code, stream)
    if rc:
        raise GemmError(rc, "gemm_strided_batched")
    return out


def conv2d(x, w, bias=None, relu: bool = False, stride=(1, 1), pad=(0, 0), dil=(1, 1),
           out_f32: bool = False, stream=None):
    """NHWC convolution through the C ABI: x (batch, H, W, cin), w (KH, KW, cin,
    cout) -> (batch, OH, OW, cout)."""
    import torch
    batch, H, W, cin = x.shape
    KH, KW, _, cout = w.shape
    OH = (H + 2 * pad[0] - dil[0] * (KH - 1) - 1) // stride[0] + 1
    OW = (W + 2 * pad[1] - dil[1] * (KW - 1) - 1) // stride[1] + 1
    y = torch.empty(batch, OH, OW, cout, device=x.device,
                    dtype=torch.float32 if out_f32 else x.dtype)
    epi = (GEMM_EPI_BIAS if bias is not None else 0) | (GEMM_EPI_RELU if relu else 0)
    rc = conv2d_im2col(batch, H, W, cin, cout, KH, KW, stride[0], stride[1], pad[0], pad[1],
                       dil[0], dil[1], x, w, y, bias, epi, dtype_code(x.dtype, out_f32), stream)
    if rc:
        raise GemmError(rc, "conv2d_im2col")
    return y


def grouped_matmul(x, w, group_rows_dev, bias=None, relu: bool = False,
                   b_col_major: bool = False, out=None, out_f32: bool = False, stream=None):
    """Y[rows of g] = act(X[rows of g] @ W[g] + bias[g]) for all groups in one launch.

    x: (R, K); w: (G, K, N) or (G, N, K) with ``b_col_major``;
    group_rows_dev: int32 (G,) device tensor."""
    import torch
    R, K = x.shape
    G = w.shape[0]
    N = w.shape[1] if b_col_major else w.shape[2]
    code = dtype_code(x.dtype, out_f32)
    if out is None:
        out = torch.empty(R, N, device=x.device, dtype=torch.float32 if out_f32 else x.dtype)
    epi = (GEMM_EPI_BIAS if bias is not None else 0) | (GEMM_EPI_RELU if relu else 0) | \
        (GEMM_B_COL_MAJOR if b_col_major else 0)
    rc = grouped_gemm(G, group_rows_dev, R, N, K, x, x.stride(0), w, w.stride(1), w.stride(0),
                      out, out.stride(0), bias, epi, code, stream)
    if rc:
        raise GemmError(rc, "grouped_gemm")
    return out


def header_functions() -> list[str]:
    """Names of the functions include/dense_gemm.h declares."""
    import re
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^GEMM_API [^(]*?\b([a-z_][a-z0-9_]*)\(", text, flags=re.M)

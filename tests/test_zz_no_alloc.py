"""The scratch-free split-K entry point, gemm_splitk_noalloc.

gemm() gets split-K scratch from cudaMalloc once per stream.  Some callers
cannot allow that: a service whose own allocator owns the device memory,
or a latency-critical loop that cannot take cudaMalloc's implicit device
synchronisation.  gemm_splitk_noalloc takes its scratch from a fixed array
inside the library instead.  Here it is called through the C ABI twice in a
row, and each output is compared with what gemm() (the existing entry point)
returns for the same inputs, within the tolerance the parity tests use.

This file is collected last, so a run that stops at the first failure has
already run every other test.  It passes alone in a fresh process as well as
after the rest of the suite.
"""
import pytest
import torch

import dense_gemm_16_b200 as dg
from gpu_helpers import Guarded, compare

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, b_col, seed):
    gen = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=gen).half().cuda()
    B = torch.randn(*((N, K) if b_col else (K, N)), generator=gen).half().cuda()
    bias = torch.randn(N, generator=gen).half().cuda()
    return A, B, bias


@pytest.mark.parametrize("M,N,K,b_col,splits", [
    (512, 640, 4096, False, 4),   # 128 x 128 tiles, row-major B
    (300, 520, 2000, True, 3),    # ragged tiles, column-major B
    (16, 4096, 8192, True, 8),    # skinny: B's columns on the MMA rows
])
def test_noalloc_matches_gemm_twice(M, N, K, b_col, splits):
    A, B, bias = _inputs(M, N, K, b_col, seed=M + N + K)
    epi = dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU | (dg.GEMM_B_COL_MAJOR if b_col else 0)
    ldb = K if b_col else N
    ref = Guarded(M, N, N, torch.float16)
    assert dg.gemm(M, N, K, A, K, B, ldb, ref.ptr, N, bias, epi, dg.GEMM_F16) == 0
    torch.cuda.synchronize()
    expect = ref.matrix().double().cpu().numpy()
    for _ in range(2):  # the shared array keeps the last call's contents
        g = Guarded(M, N, N, torch.float16)
        rc = dg.gemm_splitk_noalloc(M, N, K, A, K, B, ldb, g.ptr, N, bias, epi, dg.GEMM_F16,
                                    splits)
        assert rc == 0, dg.gemm_status_string(rc)
        torch.cuda.synchronize()
        assert dg.gemm_device_status() == 0
        compare(g.matrix().double().cpu().numpy(), expect, 2, "noalloc vs gemm")
        g.check_canaries()


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 4096 x 4096 in 128 x 128 tiles with 8 pieces needs 1024*8*64 KiB of partials
    M = N = K = 4096
    A, B, _ = _inputs(64, 64, 64, False, seed=5)  # never read: rejected first
    g = Guarded(8, 8, 8, torch.float16)
    rc = dg.gemm_splitk_noalloc(M, N, K, A, K, B, N, g.ptr, N, None, 0, dg.GEMM_F16, 8)
    assert rc == dg.GEMM_ERR_UNSUPPORTED
    assert dg.gemm_splitk_noalloc(4, 4, 4, A, 64, B, 64, g.ptr, 8, None, 0, dg.GEMM_F16,
                                  0) == dg.GEMM_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((g.ibuf.cpu() == g.sent).all())  # nothing was launched

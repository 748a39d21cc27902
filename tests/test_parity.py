"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on
the seeded workloads (every element for the small configurations, a seeded
sample of 4096 outputs plus tile-boundary rows/columns for the large ones),
bit-exact integer cases, edge cases, every compiled tile config, and
sentinel guard bands around C to catch any store outside it."""
import numpy as np
import pytest
import torch

import dense_gemm_16_b200 as dg
import oracle
import workloads
from gpu_helpers import THREADS, Guarded, compare, in_name, pad_cols, run_gemm

pytestmark = pytest.mark.gpu


def _dense_case(w, sampled: bool):
    A, B, bias = workloads.make_inputs(w)
    dA, dB = A.cuda(), B.cuda()
    dbias = bias.cuda() if bias is not None else None
    g = run_gemm(dA, dB, dbias, w.M, w.N, w.K, b_col=w.b_colmajor, relu=w.relu)
    got = g.matrix().double().cpu().numpy()
    g.check_canaries()
    ldb = w.K if w.b_colmajor else w.N
    if not sampled:
        ref = oracle.gemm(w.M, w.N, w.K, A, w.K, B, ldb, b_colmajor=w.b_colmajor, bias=bias,
                          relu=w.relu, dtype=w.dtype, threads=THREADS)
        compare(got, ref, 2, w.name)
    else:
        rows, cols = workloads.sample_indices(w.M, w.N)
        ref = oracle.gemm_at(w.M, w.N, w.K, A, w.K, B, ldb, rows, cols,
                             b_colmajor=w.b_colmajor, bias=bias, relu=w.relu, dtype=w.dtype,
                             threads=THREADS)
        compare(got[rows, cols], ref, 2, w.name)
    assert np.isfinite(got).all()


@pytest.mark.parametrize("name", ["square256_f16", "m1024n1024k2048_f16",
                                  "m1024n1024k2048_f16_bias_relu", "m1000n1000k2000_f16_bcol",
                                  "m16n8192k8192_f16_bcol"])
def test_config_every_element(name):
    _dense_case(workloads.get(name), sampled=False)


@pytest.mark.parametrize("name", ["square4096_bf16", "square4096_f16", "square8192_bf16",
                                  "square8192_f16", "m4096n4096k512_f16_bcol"])
def test_config_sampled(name):
    _dense_case(workloads.get(name), sampled=True)


@pytest.mark.parametrize("config", [-1, 13, 24, 34])
def test_moe_grouped_sampled(config):
    w = workloads.get("moe32_m8192n1408k4096_bf16_relu")
    X, W, rows_per, bias = workloads.make_grouped_inputs(w)
    total = int(rows_per.sum())
    dX, dW = X.cuda(), W.cuda()
    drows = torch.from_numpy(rows_per).cuda()
    g = Guarded(total, w.N, w.N, torch.bfloat16)
    assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.grouped_gemm(w.experts, drows, total, w.N, w.K, dX, w.K, dW, w.N, w.K * w.N,
                             g.ptr, w.N, None, dg.GEMM_EPI_RELU, dg.GEMM_BF16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    got = g.matrix().double().cpu().numpy()
    g.check_canaries()
    r, c = workloads.sample_indices(total, w.N, group_rows=rows_per)
    ref = oracle.grouped_gemm_at(rows_per, w.N, w.K, X, w.K, W, w.N, w.K * w.N, r, c, relu=True,
                                 dtype="bf16", threads=THREADS)
    compare(got[r, c], ref, 2, w.name)


# ------------------------------------------------ bit-exact integer cases

@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("b_col", [False, True])
@pytest.mark.parametrize("config", [0, 1, 4, 5, 8, 9, 10, 11, 12, 13, 23, 24, 28, 29, 30, 31,
                                    32, 34, 35, 36, 37, 38])
def test_exact_integers(dtype, b_col, config):
    """Integer inputs in [-2, 2] with K <= 4096: every partial sum is an
    exact integer below 2^24, so the fp32 accumulator is exact in any order
    and the fp32 output must equal the oracle bit for bit; the 16-bit output
    must equal the round-to-nearest-even of that exact value."""
    M, N, K = 300, 520, 1000
    gen = torch.Generator().manual_seed(77 + config)
    A = torch.randint(-2, 3, (M, K), generator=gen).to(dtype)
    B = torch.randint(-2, 3, (N, K) if b_col else (K, N), generator=gen).to(dtype)
    bias = torch.randint(-4, 5, (N,), generator=gen).to(dtype)
    ref = oracle.gemm(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                      relu=True, dtype=in_name(A), threads=THREADS)
    assert dg.gemm_force_config(config) == 0
    try:
        g32 = run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=b_col, relu=True,
                       out_f32=True)
        g16 = run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=b_col, relu=True)
    finally:
        dg.gemm_force_config(-1)
    got32 = g32.matrix().double().cpu().numpy()
    assert np.array_equal(got32, ref)
    expect16 = torch.from_numpy(ref).to(dtype)  # RNE of the exact value
    assert torch.equal(g16.matrix().cpu(), expect16)
    g32.check_canaries()
    g16.check_canaries()


# ----------------------------------------------------------- edge cases

@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (7, 9, 5), (130, 200, 72), (129, 257, 65),
                                   (256, 16, 64), (64, 8, 1000), (3, 4100, 70)])
@pytest.mark.parametrize("b_col", [False, True])
def test_ragged_shapes(M, N, K, b_col):
    gen = torch.Generator().manual_seed(M * 31 + N * 7 + K)
    A = (torch.rand(M, K, generator=gen) * 2 - 1).half()
    B = (torch.rand(*((N, K) if b_col else (K, N)), generator=gen) * 2 - 1).half()
    bias = (torch.rand(N, generator=gen) * 2 - 1).half()
    # leading dimensions with padding (NaN-filled: any read past the edge shows)
    lda = (K + 15) // 8 * 8
    ldb = ((K if b_col else N) + 15) // 8 * 8
    dA = pad_cols(A.cuda(), lda)
    dB = pad_cols(B.cuda(), ldb)
    g = run_gemm(dA, dB, bias.cuda(), M, N, K, b_col=b_col, relu=True, ldc=(N + 23) // 8 * 8)
    ref = oracle.gemm(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                      relu=True, threads=THREADS)
    compare(g.matrix().double().cpu().numpy(), ref, 2, f"{M}x{N}x{K}")
    g.check_canaries()


@pytest.mark.parametrize("out_f32", [False, True])
def test_k_zero_writes_act_bias(out_f32):
    M, N = 37, 50
    bias = torch.linspace(-3, 3, N).half()
    g = run_gemm(torch.empty(0, 0, dtype=torch.half, device="cuda"),
                 torch.empty(0, 0, dtype=torch.half, device="cuda"), bias.cuda(), M, N, 0,
                 relu=True, out_f32=out_f32)
    ref = oracle.gemm(M, N, 0, None, 0, None, 0, bias=bias, relu=True)
    compare(g.matrix().double().cpu().numpy(), ref, 4 if out_f32 else 2, "K=0")
    g.check_canaries()


def test_empty_m_or_n_is_a_noop():
    g = Guarded(4, 8, 8, torch.float16)
    A = torch.ones(4, 8, dtype=torch.half, device="cuda")
    assert dg.gemm(0, 8, 8, A, 8, A, 8, g.ptr, 8, None, 0, dg.GEMM_F16) == 0
    assert dg.gemm(4, 0, 8, A, 8, A, 8, g.ptr, 8, None, 0, dg.GEMM_F16) == 0
    torch.cuda.synchronize()
    assert bool((g.ibuf.cpu() == g.sent).all())


DENSE_CONFIGS = list(range(25)) + list(range(28, 39))  # 25..27 are grouped-only


@pytest.mark.parametrize("config", DENSE_CONFIGS)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("out_f32", [False, True])
def test_every_config_on_ragged_problem(config, dtype, out_f32):
    assert config < dg.gemm_num_configs()
    name = dg.gemm_config_name(config)
    swap = name.startswith(("swap", "cskswap"))
    M, N, K = (29 if swap else 333), 712, 328
    gen = torch.Generator().manual_seed(1000 + config)
    A = torch.randn(M, K, generator=gen).to(dtype)
    layouts = [True] if swap else [False, True]
    for b_col in layouts:
        B = torch.randn(*((N, K) if b_col else (K, N)), generator=gen).to(dtype)
        bias = torch.randn(N, generator=gen).to(dtype)
        ref = oracle.gemm(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                          dtype=in_name(A), threads=THREADS)
        assert dg.gemm_force_config(config) == 0
        try:
            g = run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=b_col, out_f32=out_f32)
        finally:
            dg.gemm_force_config(-1)
        compare(g.matrix().double().cpu().numpy(), ref, 4 if out_f32 else 2,
                f"{name} b_col={b_col}")
        g.check_canaries()


PAIR_SK_CONFIGS = [36, 37, 38]  # CTA-pair stream-K, hybrid, and stream-K on 256 x 256 tiles


@pytest.mark.parametrize("config", PAIR_SK_CONFIGS)
@pytest.mark.parametrize("M,N,K,b_col", [(1000, 1504, 2000, False), (2304, 2560, 1536, True),
                                         (777, 1104, 4104, False)])
def test_pair_stream_k_every_element(config, M, N, K, b_col):
    """Stream-K over CTA pairs: pieces cross tile edges, each CTA of a pair
    fixes up its own 128 rows; every element against the oracle, and a
    second launch (counters left at zero) is bit-identical."""
    name = dg.gemm_config_name(config)
    gen = torch.Generator().manual_seed(5000 + config + M)
    A = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    B = torch.randn(*((N, K) if b_col else (K, N)), generator=gen).to(torch.bfloat16)
    bias = torch.randn(N, generator=gen).to(torch.bfloat16)
    ref = oracle.gemm(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                      relu=True, dtype="bf16", threads=THREADS)
    assert dg.gemm_force_config(config) == 0
    try:
        outs = [run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=b_col, relu=True)
                for _ in range(2)]
    finally:
        dg.gemm_force_config(-1)
    first = outs[0].matrix().cpu()
    assert torch.equal(outs[1].matrix().cpu(), first)
    compare(first.double().numpy(), ref, 2, f"{name} {M}x{N}x{K}")
    for g in outs:
        g.check_canaries()


@pytest.mark.parametrize("config", PAIR_SK_CONFIGS)
@pytest.mark.parametrize("name", ["square4096_bf16", "square8192_f16"])
def test_pair_stream_k_sampled(config, name):
    w = workloads.get(name)
    assert dg.gemm_force_config(config) == 0
    try:
        _dense_case(w, sampled=True)
    finally:
        dg.gemm_force_config(-1)


@pytest.mark.parametrize("config", [None, 0, 1, 11, 13, 28])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("offset", [0, 1, 3])
def test_bias_at_element_alignment(config, dtype, offset):
    """The bias needs only its element alignment: a vector that starts 1 or 3
    elements past a 16-byte boundary, with N not a multiple of 16, must give
    the same result as an aligned one (the epilogue loads the tile's bias
    with vector loads only where they are aligned and inside N)."""
    if dtype == torch.float32 and config not in (None, 0, 1):
        pytest.skip("fp32 inputs run on the single-CTA 128 x 128 / 128 x 256 tf32 tiles only")
    M, N, K = 300, 1000, 192
    gen = torch.Generator().manual_seed(7000 + offset + (config or 0))
    A = torch.randint(-2, 3, (M, K), generator=gen).to(dtype)
    B = torch.randint(-2, 3, (K, N), generator=gen).to(dtype)
    bias = torch.randint(-4, 5, (N,), generator=gen).to(dtype)
    ref = oracle.gemm(M, N, K, A, K, B, N, bias=bias, relu=True, dtype=in_name(A),
                      threads=THREADS) if dtype != torch.float32 else \
        oracle.gemm_f32(M, N, K, A, K, B, N, bias=bias, relu=True, threads=THREADS)
    dbias = torch.zeros(N + 8, dtype=dtype, device="cuda")
    dbias[offset:offset + N] = bias.cuda()
    if config is not None:
        assert dg.gemm_force_config(config) == 0
    try:
        g = run_gemm(A.cuda(), B.cuda(), dbias[offset:offset + N], M, N, K, relu=True,
                     out_f32=dtype != torch.float32 and offset == 1)
    finally:
        dg.gemm_force_config(-1)
    # small integers: every partial sum is exact in fp32 in any order, so an
    # fp32 output equals the oracle and a 16-bit one its round-to-nearest-even
    out_f32 = dtype == torch.float32 or offset == 1
    expect = ref if out_f32 else torch.from_numpy(ref).to(dtype).double().numpy()
    got = g.matrix().double().cpu().numpy()
    assert np.array_equal(got, expect), \
        dg.gemm_config_name(config) if config is not None else "table"
    g.check_canaries()


def test_swap_config_rejects_row_major_b():
    n = [i for i in range(dg.gemm_num_configs()) if dg.gemm_config_name(i).startswith("swap")][0]
    A = torch.ones(16, 64, dtype=torch.half, device="cuda")
    B = torch.ones(64, 64, dtype=torch.half, device="cuda")
    C = torch.empty(16, 64, dtype=torch.half, device="cuda")
    assert dg.gemm_force_config(n) == 0
    try:
        assert dg.gemm(16, 64, 64, A, 64, B, 64, C, 64, None, 0,
                       dg.GEMM_F16) == dg.GEMM_ERR_UNSUPPORTED
    finally:
        dg.gemm_force_config(-1)


def test_configs_of_the_other_kind_are_rejected():
    # a grouped-only config on a dense call, a swapped (skinny) config on a
    # grouped call: UNSUPPORTED, and nothing is written
    A = torch.ones(64, 64, dtype=torch.half, device="cuda")
    B = torch.ones(64, 64, dtype=torch.half, device="cuda")
    C = torch.zeros(64, 64, dtype=torch.half, device="cuda")
    rows = torch.tensor([32, 32], dtype=torch.int32, device="cuda")
    Bg = torch.ones(2, 64, 64, dtype=torch.half, device="cuda")
    pair = [i for i in range(dg.gemm_num_configs()) if dg.gemm_config_name(i).startswith("swap")][0]
    try:
        assert dg.gemm_force_config(25) == 0
        assert dg.gemm(64, 64, 64, A, 64, B, 64, C, 64, None, 0,
                       dg.GEMM_F16) == dg.GEMM_ERR_UNSUPPORTED
        assert dg.gemm_force_config(pair) == 0
        assert dg.grouped_gemm(2, rows, 64, 64, 64, A, 64, Bg, 64, 64 * 64, C, 64, None, 0,
                               dg.GEMM_F16) == dg.GEMM_ERR_UNSUPPORTED
    finally:
        dg.gemm_force_config(-1)
    torch.cuda.synchronize()
    assert int(C.abs().sum()) == 0


@pytest.mark.parametrize("config", [1, 13, 21, 8])  # single CTA, pair, swapped stream-K, split-K
def test_trace_records_ordered_events_per_block(config):
    M, N, K = (16, 8192, 1024) if config == 21 else (1024, 1024, 512)
    A = torch.randn(M, K, dtype=torch.half, device="cuda")
    B = torch.randn(N, K, dtype=torch.half, device="cuda")
    C = torch.empty(M, N, dtype=torch.half, device="cuda")
    buf = torch.zeros(148 * dg.GEMM_TRACE_EVENTS, dtype=torch.int64, device="cuda")
    assert dg.gemm_set_trace(buf, buf.numel() * 8) == 0
    assert dg.gemm_force_config(config) == 0
    try:
        assert dg.gemm(M, N, K, A, K, B, K, C, N, None, dg.GEMM_B_COL_MAJOR, dg.GEMM_F16) == 0
        torch.cuda.synchronize()
    finally:
        dg.gemm_force_config(-1)
        dg.gemm_set_trace(None, 0)
    t = buf.view(148, dg.GEMM_TRACE_EVENTS).cpu().numpy()
    started = t[:, dg.GEMM_TRACE_ENTRY] > 0
    assert started.sum() > 0
    for row in t[started]:
        assert row[dg.GEMM_TRACE_ENTRY] <= row[dg.GEMM_TRACE_SETUP] <= row[dg.GEMM_TRACE_EXIT]
        if row[dg.GEMM_TRACE_FIRST_DATA] > 0:  # a block with work
            assert row[dg.GEMM_TRACE_SETUP] <= row[dg.GEMM_TRACE_FIRST_LOAD]
            assert row[dg.GEMM_TRACE_FIRST_LOAD] <= row[dg.GEMM_TRACE_FIRST_DATA]
            assert row[dg.GEMM_TRACE_FIRST_DATA] <= row[dg.GEMM_TRACE_LAST_MMA] <= row[dg.GEMM_TRACE_EXIT]
        if row[dg.GEMM_TRACE_FIRST_EPI] > 0:
            assert row[dg.GEMM_TRACE_FIRST_EPI] <= row[dg.GEMM_TRACE_EPI_DONE] <= row[dg.GEMM_TRACE_EXIT]
    # tracing changes no result: the same call untraced gives the same bits
    C2 = torch.empty_like(C)
    assert dg.gemm_force_config(config) == 0
    try:
        assert dg.gemm(M, N, K, A, K, B, K, C2, N, None, dg.GEMM_B_COL_MAJOR, dg.GEMM_F16) == 0
        torch.cuda.synchronize()
    finally:
        dg.gemm_force_config(-1)
    assert torch.equal(C, C2)


CSK = [31, 32]  # CTA-pair split-K reduced in distributed shared memory


@pytest.mark.parametrize("config", CSK)
@pytest.mark.parametrize("M,N,K,b_col", [
    (74 * 128, 128, 256, False),  # 74 tiles of 128 x 128: every pair of SMs busy
    (300, 200, 136, True),        # three K blocks: halves of 2 and 1
    (1, 8, 128, False),           # one row, two K blocks
])
def test_pair_split_k_every_element(config, M, N, K, b_col):
    assert dg.gemm_config_name(config).startswith("csk")
    bn = 128 if config == 31 else 64
    if ((M + 127) // 128) * ((N + bn - 1) // bn) > 74:
        pytest.skip("more tiles than SM pairs")
    gen = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=gen).half()
    B = torch.randn(*((N, K) if b_col else (K, N)), generator=gen).half()
    bias = torch.randn(N, generator=gen).half()
    ref = oracle.gemm(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                      relu=True, dtype="f16", threads=THREADS)
    assert dg.gemm_force_config(config) == 0
    try:
        g = run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=b_col, relu=True)
    finally:
        dg.gemm_force_config(-1)
    compare(g.matrix().double().cpu().numpy(), ref, 2, "pair split-K")
    g.check_canaries()


def test_table_choice_of_pair_split_k_and_its_batched_fallback():
    # 512 x 512 x 2048 matches no rule: the heuristic takes the pair split-K
    # kernel; 1024 x 1024 x 2048 in a batch of 2 has 128 tiles, more than the
    # SM pairs, so the batched call runs 128 x 128 tiles instead
    assert dg.gemm_config_name(dg.gemm_select_config(512, 512, 2048, dg.GEMM_F16, 0)) \
        .startswith("csk")
    gen = torch.Generator().manual_seed(31)
    A = torch.randn(512, 2048, generator=gen).half()
    B = torch.randn(2048, 512, generator=gen).half()
    ref = oracle.gemm(512, 512, 2048, A, 2048, B, 512, dtype="f16", threads=THREADS)
    g = run_gemm(A.cuda(), B.cuda(), None, 512, 512, 2048)
    compare(g.matrix().double().cpu().numpy(), ref, 2, "heuristic pair split-K")
    g.check_canaries()
    M = N = 1024
    K = 2048
    A2 = torch.randn(2, M, K, generator=gen).half()
    B2 = torch.randn(2, K, N, generator=gen).half()
    C2 = torch.empty(2, M, N, dtype=torch.half, device="cuda")
    rc = dg.gemm_strided_batched(2, M, N, K, A2.cuda(), K, M * K, B2.cuda(), N, K * N, C2, N,
                                 M * N, None, 0, 0, dg.GEMM_F16)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    for b in range(2):
        r, c = workloads.sample_indices(M, N, n=512, seed=b)
        ref = oracle.gemm_at(M, N, K, A2[b], K, B2[b], N, r, c, dtype="f16", threads=THREADS)
        compare(C2[b].double().cpu().numpy()[r, c], ref, 2, f"batched fallback {b}")


@pytest.mark.parametrize("M,N,K", [(16, 8192, 2048), (29, 712, 328), (1, 1000, 136)])
def test_pair_split_k_swapped_every_element(M, N, K):
    # skinny problems: B column-major, C^T in the accumulators, 8 KB handed over
    config = 33
    assert dg.gemm_config_name(config).startswith("cskswap")
    gen = torch.Generator().manual_seed(M * 7 + K)
    A = torch.randn(M, K, generator=gen).half()
    B = torch.randn(N, K, generator=gen).half()
    bias = torch.randn(N, generator=gen).half()
    ref = oracle.gemm(M, N, K, A, K, B, K, b_colmajor=True, bias=bias, relu=True, dtype="f16",
                      threads=THREADS)
    assert dg.gemm_force_config(config) == 0
    try:
        g = run_gemm(A.cuda(), B.cuda(), bias.cuda(), M, N, K, b_col=True, relu=True)
    finally:
        dg.gemm_force_config(-1)
    compare(g.matrix().double().cpu().numpy(), ref, 2, "swapped pair split-K")
    g.check_canaries()


@pytest.mark.parametrize("config", CSK)
def test_pair_split_k_rejects_what_it_cannot_split(config):
    # more tiles than SM pairs, or a single K block: UNSUPPORTED, nothing written
    A = torch.ones(4096, 256, dtype=torch.half, device="cuda")
    B = torch.ones(256, 4096, dtype=torch.half, device="cuda")
    C = torch.zeros(4096, 4096, dtype=torch.half, device="cuda")
    assert dg.gemm_force_config(config) == 0
    try:
        assert dg.gemm(4096, 4096, 256, A, 256, B, 4096, C, 4096, None, 0,
                       dg.GEMM_F16) == dg.GEMM_ERR_UNSUPPORTED
        assert dg.gemm(128, 128, 64, A, 256, B, 4096, C, 4096, None, 0,
                       dg.GEMM_F16) == dg.GEMM_ERR_UNSUPPORTED
    finally:
        dg.gemm_force_config(-1)
    torch.cuda.synchronize()
    assert int(C.abs().sum()) == 0


def test_freeing_scratch_keeps_later_calls_right():
    # split-K scratch for a side stream, freed, then allocated anew by the
    # next call; freeing every stream's scratch leaves the library usable
    M, N, K = 256, 384, 4096
    gen = torch.Generator().manual_seed(8)
    A = torch.randn(M, K, generator=gen).half()
    B = torch.randn(N, K, generator=gen).half()
    ref = oracle.gemm(M, N, K, A, K, B, K, b_colmajor=True, dtype="f16", threads=THREADS)
    s = torch.cuda.Stream()
    sk = [i for i in range(dg.gemm_num_configs()) if dg.gemm_config_name(i) == "tc1_128x128_s6_g8_k4"][0]
    assert dg.gemm_force_config(sk) == 0
    try:
        for free_all in (False, True, False):
            with torch.cuda.stream(s):
                g = run_gemm(A.cuda(), B.cuda(), None, M, N, K, b_col=True, stream=s)
                compare(g.matrix().double().cpu().numpy(), ref, 2, f"after free (all={free_all})")
            assert dg.gemm_free_scratch(s, all_streams=free_all) == 0
    finally:
        dg.gemm_force_config(-1)
    assert dg.gemm_free_scratch(s) == 0  # nothing left to free


def test_runs_on_a_side_stream():
    s = torch.cuda.Stream()
    w = workloads.get("square256_f16")
    A, B, _ = workloads.make_inputs(w)
    with torch.cuda.stream(s):
        dA, dB = A.cuda(), B.cuda()
        out = dg.matmul(dA, dB, stream=s)
    s.synchronize()
    ref = oracle.gemm(256, 256, 256, A, 256, B, 256, threads=THREADS)
    compare(out.double().cpu().numpy(), ref, 2, "side stream")


@pytest.mark.parametrize("config", [None, 8, 23, 36])
def test_calls_replay_in_a_cuda_graph(config):
    """gemm() and grouped_gemm() captured into one CUDA graph (after an
    uncaptured call on the capture stream has sized its scratch) replay
    correctly on fresh inputs, again and again: split-K and stream-K
    counters are left at zero by every launch."""
    name = dg.gemm_config_name(config) if config is not None else "table"
    M, N, K = 640, 768, 1024
    rows_per = np.array([100, 0, 300, 240], dtype=np.int32)
    G, total = len(rows_per), int(rows_per.sum())
    dA = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dB = torch.empty(K, N, dtype=torch.bfloat16, device="cuda")
    dbias = torch.empty(N, dtype=torch.bfloat16, device="cuda")
    dC = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(total, K, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(G, K, N, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(total, N, dtype=torch.bfloat16, device="cuda")
    drows = torch.from_numpy(rows_per).cuda()
    epi = dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU
    s = torch.cuda.Stream()

    def calls():
        rc = dg.gemm(M, N, K, dA, K, dB, N, dC, N, dbias, epi, dg.GEMM_BF16, s)
        assert rc == 0, dg.gemm_status_string(rc)
        rc = dg.grouped_gemm(G, drows, total, N, K, dX, K, dW, N, K * N, dY, N, None,
                             dg.GEMM_EPI_RELU, dg.GEMM_BF16, s)
        assert rc == 0, dg.gemm_status_string(rc)

    if config is not None:
        assert dg.gemm_force_config(config) == 0
    try:
        dA.zero_(); dB.zero_(); dbias.zero_(); dX.zero_(); dW.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            calls()  # sizes this stream's scratch outside the capture
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            calls()
    finally:
        dg.gemm_force_config(-1)
    for rep in range(3):
        gen = torch.Generator().manual_seed(8000 + rep + (config or 0))
        A = torch.randn(M, K, generator=gen).bfloat16()
        B = torch.randn(K, N, generator=gen).bfloat16()
        bias = torch.randn(N, generator=gen).bfloat16()
        X = torch.randn(total, K, generator=gen).bfloat16()
        W = (torch.randn(G, K, N, generator=gen) * 0.1).bfloat16()
        dA.copy_(A); dB.copy_(B); dbias.copy_(bias); dX.copy_(X); dW.copy_(W)
        dC.fill_(float("nan")); dY.fill_(float("nan"))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert dg.gemm_device_status() == 0
        ref = oracle.gemm(M, N, K, A, K, B, N, bias=bias, relu=True, dtype="bf16",
                          threads=THREADS)
        compare(dC.double().cpu().numpy(), ref, 2, f"{name} graph replay {rep}")
        refg = oracle.grouped_gemm(rows_per, N, K, X, K, W, N, K * N, relu=True, dtype="bf16",
                                   threads=THREADS)
        compare(dY.double().cpu().numpy(), refg, 2, f"{name} grouped graph replay {rep}")
    del graph


# --------------------------------------------------------------- grouped

# 128 x 256 / 128 x 128 row tiles; swapped operands (one CTA, then CTA pairs)
# 23, 24: stream-K over the groups' tiles; 34, 35: the hybrid; 4, 13: CTA pairs
GROUPED_CONFIGS = [0, 1, 4, 13, 23, 24, 25, 26, 27, 34, 35]


@pytest.mark.parametrize("b_col", [False, True])
@pytest.mark.parametrize("out_f32", [False, True])
@pytest.mark.parametrize("config", GROUPED_CONFIGS)
def test_grouped_every_element(b_col, out_f32, config):
    if 25 <= config <= 27:
        assert dg.gemm_config_name(config).startswith("gswap")
    rows_per = np.array([0, 3, 130, 1, 0, 257, 64, 0], dtype=np.int32)
    G, N, K = len(rows_per), 200, 136
    total = int(rows_per.sum())
    gen = torch.Generator().manual_seed(5 + config)
    X = torch.randn(total, K, generator=gen).bfloat16()
    W = (torch.randn(*((G, N, K) if b_col else (G, K, N)), generator=gen) * 0.1).bfloat16()
    bias = torch.randn(G, N, generator=gen).bfloat16()
    ref = oracle.grouped_gemm(rows_per, N, K, X, K, W, K if b_col else N, N * K,
                              b_colmajor=b_col, bias=bias, relu=True, dtype="bf16",
                              threads=THREADS)
    dt = torch.float32 if out_f32 else torch.bfloat16
    ldc = N + 8
    g = Guarded(total, N, ldc, dt)
    epi = dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU | (dg.GEMM_B_COL_MAJOR if b_col else 0)
    assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.grouped_gemm(G, torch.from_numpy(rows_per).cuda(), total, N, K, X.cuda(), K,
                             W.cuda(), K if b_col else N, N * K, g.ptr, ldc, bias.cuda(), epi,
                             dg.GEMM_BF16_OUT_F32 if out_f32 else dg.GEMM_BF16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    compare(g.matrix().double().cpu().numpy(), ref, 4 if out_f32 else 2, "grouped")
    g.check_canaries()


@pytest.mark.parametrize("config", [4, 11, 13])
@pytest.mark.parametrize("N", [196, 200, 512, 1000])
@pytest.mark.parametrize("out_f32", [False, True])
def test_grouped_pair_stores_every_element(config, N, out_f32):
    """Grouped CTA-pair tiles leave by staged row-segment stores masked at
    each group's last row (N whole 16-byte vectors) or by per-row register
    stores (N=196 in 16-bit); groups end inside a warp's 32 rows, inside a
    CTA's 128 and inside a pair's 256."""
    rows_per = np.array([0, 300, 256, 1, 511, 33], dtype=np.int32)
    G, K = len(rows_per), 200
    total = int(rows_per.sum())
    gen = torch.Generator().manual_seed(90 + config + N)
    X = torch.randn(total, K, generator=gen).bfloat16()
    W = (torch.randn(G, N, K, generator=gen) * 0.1).bfloat16()  # column-major B: any N
    bias = torch.randn(G, N, generator=gen).bfloat16()
    ref = oracle.grouped_gemm(rows_per, N, K, X, K, W, K, N * K, b_colmajor=True, bias=bias,
                              relu=True, dtype="bf16", threads=THREADS)
    dt = torch.float32 if out_f32 else torch.bfloat16
    ldc = (N + 15) // 8 * 8
    g = Guarded(total, N, ldc, dt)
    assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.grouped_gemm(G, torch.from_numpy(rows_per).cuda(), total, N, K, X.cuda(), K,
                             W.cuda(), K, N * K, g.ptr, ldc, bias.cuda(),
                             dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU | dg.GEMM_B_COL_MAJOR,
                             dg.GEMM_BF16_OUT_F32 if out_f32 else dg.GEMM_BF16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    compare(g.matrix().double().cpu().numpy(), ref, 4 if out_f32 else 2,
            f"{dg.gemm_config_name(config)} N={N}")
    g.check_canaries()


@pytest.mark.parametrize("config", [-1, 4, 13, 24, 25, 26])
def test_grouped_counts_beyond_total_are_clipped_and_reported(config):
    rows_per = np.array([5, 300, 40], dtype=np.int32)  # sums to 345
    total, N, K = 200, 64, 64                           # caller says 200
    X = torch.randn(total, K).bfloat16()
    W = torch.randn(3, K, N).bfloat16()
    g = Guarded(total, N, N, torch.bfloat16)
    assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.grouped_gemm(3, torch.from_numpy(rows_per).cuda(), total, N, K, X.cuda(), K,
                             W.cuda(), N, K * N, g.ptr, N, None, 0, dg.GEMM_BF16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == dg.GEMM_ERR_INVALID_ARG
    g.check_canaries()
    # the rows that exist are still right: group 0 rows 0..4, group 1 rows 5..199
    ref = oracle.grouped_gemm(np.array([5, 195], dtype=np.int32), N, K, X, K, W, N, K * N,
                              dtype="bf16", threads=THREADS)
    compare(g.matrix().double().cpu().numpy(), ref, 2, "clipped groups")


def _grouped_problem(rows_per, N, K, seed, dtype=torch.bfloat16, b_col=False):
    G = len(rows_per)
    total = int(np.sum(rows_per))
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(total, K, generator=gen).to(dtype)
    W = (torch.randn(*((G, N, K) if b_col else (G, K, N)), generator=gen) * 0.05).to(dtype)
    bias = torch.randn(G, N, generator=gen).to(dtype)
    return X, W, bias


@pytest.mark.parametrize("config", [25, 26, 4, 13])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_grouped_swap_many_groups_every_element(config, dtype):
    # 40 groups: empty, 1..15 rows (one 16-row box), exact multiples of 16,
    # 256 (one full tile), 257 and 600 (two and three near-equal row blocks)
    rng = np.random.default_rng(77)
    rows_per = np.concatenate([[0, 1, 15, 16, 17, 255, 256, 257, 600, 0, 48, 112],
                               rng.integers(0, 200, size=28)]).astype(np.int32)
    N, K = 392, 200
    name = "f16" if dtype == torch.float16 else "bf16"
    X, W, bias = _grouped_problem(rows_per, N, K, seed=config, dtype=dtype)
    total = int(rows_per.sum())
    ref = oracle.grouped_gemm(rows_per, N, K, X, K, W, N, N * K, bias=bias, relu=True,
                              dtype=name, threads=THREADS)
    g = Guarded(total, N, N, dtype)
    assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.grouped_gemm(len(rows_per), torch.from_numpy(rows_per).cuda(), total, N, K,
                             X.cuda(), K, W.cuda(), N, N * K, g.ptr, N, bias.cuda(),
                             dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU,
                             dg.GEMM_F16 if dtype == torch.float16 else dg.GEMM_BF16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    compare(g.matrix().double().cpu().numpy(), ref, 2, "grouped swap, 40 groups")
    g.check_canaries()


@pytest.mark.parametrize("config", [25, 26])
def test_grouped_swap_tile_queue_resets_between_launches_and_streams(config):
    # The tile queue's counter lives in each stream's scratch and every
    # launch must leave it at 0: ten launches in a row on one stream, then
    # two streams at once, each result checked in full.
    rows_per = np.array([70, 0, 300, 5, 129], dtype=np.int32)
    N, K = 256, 128
    X, W, _ = _grouped_problem(rows_per, N, K, seed=9)
    total = int(rows_per.sum())
    ref = oracle.grouped_gemm(rows_per, N, K, X, K, W, N, N * K, dtype="bf16", threads=THREADS)
    dX, dW, drows = X.cuda(), W.cuda(), torch.from_numpy(rows_per).cuda()
    assert dg.gemm_force_config(config) == 0
    try:
        outs = []
        for _ in range(10):
            y = torch.empty(total, N, dtype=torch.bfloat16, device="cuda")
            assert dg.grouped_gemm(5, drows, total, N, K, dX, K, dW, N, N * K, y, N, None, 0,
                                   dg.GEMM_BF16) == 0
            outs.append(y)
        streams = [torch.cuda.Stream() for _ in range(2)]
        torch.cuda.synchronize()
        for st in streams:
            with torch.cuda.stream(st):
                for _ in range(3):
                    y = torch.empty(total, N, dtype=torch.bfloat16, device="cuda")
                    assert dg.grouped_gemm(5, drows, total, N, K, dX, K, dW, N, N * K, y, N,
                                           None, 0, dg.GEMM_BF16) == 0
                    outs.append(y)
        torch.cuda.synchronize()
    finally:
        dg.gemm_force_config(-1)
    assert dg.gemm_device_status() == 0
    for i, y in enumerate(outs):
        compare(y.double().cpu().numpy(), ref, 2, f"launch {i}")


# -------------------------------------------------------------- watchdog

def test_watchdog_times_out_cleanly_and_context_survives():
    assert dg.gemm_watchdog_selftest(2_000_000) == dg.GEMM_ERR_DEVICE_TIMEOUT
    assert dg.gemm_device_status() == 0  # cleared by the self-test
    w = workloads.get("square256_f16")
    A, B, _ = workloads.make_inputs(w)
    out = dg.matmul(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    ref = oracle.gemm(256, 256, 256, A, 256, B, 256, threads=THREADS)
    compare(out.double().cpu().numpy(), ref, 2, "after watchdog")


# --------------------------------------------------------------- split-K

def _split_configs():
    return [i for i in range(dg.gemm_num_configs())
            if "_k" in dg.gemm_config_name(i) or dg.gemm_config_name(i).endswith("_sk")]


@pytest.mark.parametrize("swap", [False, True])
def test_split_k_is_deterministic_and_reusable(swap):
    """Partial tiles are summed in split order by whichever block finishes a
    tile last, so repeated runs are bit-identical; the arrival counters are
    left at zero, so a second launch on the same stream is right too."""
    cfgs = [i for i in _split_configs() if dg.gemm_config_name(i).startswith("swap") == swap]
    M, N, K = (16, 4096, 4096) if swap else (512, 640, 4096)
    gen = torch.Generator().manual_seed(31)
    A = torch.randn(M, K, generator=gen).half()
    B = torch.randn(N, K, generator=gen).half()
    ref = oracle.gemm_at(M, N, K, A, K, B, K, *workloads.sample_indices(M, N, n=2048),
                         b_colmajor=True, threads=THREADS)
    rows, cols = workloads.sample_indices(M, N, n=2048)
    for cid in cfgs:
        assert dg.gemm_force_config(cid) == 0
        try:
            outs = [run_gemm(A.cuda(), B.cuda(), None, M, N, K, b_col=True) for _ in range(3)]
        finally:
            dg.gemm_force_config(-1)
        first = outs[0].matrix().cpu()
        for g in outs[1:]:
            assert torch.equal(g.matrix().cpu(), first)
        compare(first.double().numpy()[rows, cols], ref, 2, dg.gemm_config_name(cid))


def test_split_k_on_concurrent_streams():
    cid = [i for i in _split_configs() if dg.gemm_config_name(i).startswith("tc1")][0]
    M, N, K = 384, 512, 2048
    gen = torch.Generator().manual_seed(41)
    As = [torch.randn(M, K, generator=gen).half() for _ in range(3)]
    B = torch.randn(K, N, generator=gen).half()
    dB = B.cuda()
    streams = [torch.cuda.Stream() for _ in range(3)]
    outs = []
    assert dg.gemm_force_config(cid) == 0
    try:
        for A, s in zip(As, streams):
            with torch.cuda.stream(s):
                dA = A.cuda()
                outs.append(dg.matmul(dA, dB, stream=s))
        torch.cuda.synchronize()
    finally:
        dg.gemm_force_config(-1)
    for A, o in zip(As, outs):
        ref = oracle.gemm(M, N, K, A, K, B, N, threads=THREADS)
        compare(o.double().cpu().numpy(), ref, 2, "split-K on a side stream")


# ------------------------------------------------------- strided batches

class BatchGuard:
    """`batch` outputs M x N (leading dimension ldc) stride_c elements apart
    in one sentinel-filled buffer: the gaps between batches and the ldc
    padding must stay untouched."""

    def __init__(self, batch, M, N, ldc, stride_c, dtype, pad=128):
        self.b, self.M, self.N, self.ldc, self.sc, self.pad = batch, M, N, ldc, stride_c, pad
        self.buf = torch.empty(pad + batch * stride_c + pad, dtype=dtype, device="cuda")
        self.ibuf = self.buf.view(torch.int32 if dtype == torch.float32 else torch.int16)
        from gpu_helpers import _SENT16, _SENT32
        self.sent = _SENT32 if dtype == torch.float32 else _SENT16
        self.ibuf.fill_(self.sent)
        self.ptr = self.buf.data_ptr() + pad * self.buf.element_size()

    def matrix(self, b):
        o = self.pad + b * self.sc
        return self.buf[o:o + self.M * self.ldc].view(self.M, self.ldc)[:, :self.N]

    def check_canaries(self):
        raw = self.ibuf.cpu()
        mask = torch.ones_like(raw, dtype=torch.bool)
        for b in range(self.b):
            o = self.pad + b * self.sc
            body = mask[o:o + self.M * self.ldc].view(self.M, self.ldc)
            body[:, :self.N] = False
        assert bool((raw[mask] == self.sent).all()), "write outside the batch outputs"


@pytest.mark.parametrize("config", [None, 0, 1, 4, 13, 8, 23, 2, 36, 37])
@pytest.mark.parametrize("b_col", [False, True])
@pytest.mark.parametrize("share", ["none", "a", "b"])
def test_strided_batched(config, b_col, share):
    name = dg.gemm_config_name(config) if config is not None else "table"
    if name.startswith("swap") and not b_col:
        pytest.skip("swapped tiles need column-major B")
    batch = 3
    M, N, K = (20 if name.startswith("swap") else 300), 264, 200
    gen = torch.Generator().manual_seed(4000 + (config or 0) + 7 * b_col)
    lda, ldb, ldc = K + 8, (K + 16 if b_col else N + 8), N + 8
    sa = 0 if share == "a" else M * lda + 64
    sb = 0 if share == "b" else (N if b_col else K) * ldb + 32
    sc, sbias = M * ldc + 96, N + 8
    A = torch.randn(max(1, batch if sa else 1), M, K, generator=gen).half()
    B = torch.randn(max(1, batch if sb else 1), *((N, K) if b_col else (K, N)), generator=gen).half()
    bias = torch.randn(batch, N, generator=gen).half()
    # device buffers with the requested strides (padding NaN-filled)
    dA = torch.full((max(1, batch if sa else 1) * max(sa, M * lda) + 64,), float("nan"),
                    dtype=torch.half, device="cuda")
    dB = torch.full((max(1, batch if sb else 1) * max(sb, B.shape[1] * ldb) + 64,), float("nan"),
                    dtype=torch.half, device="cuda")
    for i in range(A.shape[0]):
        dA[i * sa:i * sa + M * lda].view(M, lda)[:, :K] = A[i].cuda()
    for i in range(B.shape[0]):
        r, c = B.shape[1], B.shape[2]
        dB[i * sb:i * sb + r * ldb].view(r, ldb)[:, :c] = B[i].cuda()
    dbias = torch.zeros(batch * sbias, dtype=torch.half, device="cuda")
    for i in range(batch):
        dbias[i * sbias:i * sbias + N] = bias[i].cuda()
    g = BatchGuard(batch, M, N, ldc, sc, torch.float16)
    epi = dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU | (dg.GEMM_B_COL_MAJOR if b_col else 0)
    if config is not None:
        assert dg.gemm_force_config(config) == 0
    try:
        rc = dg.gemm_strided_batched(batch, M, N, K, dA, lda, sa, dB, ldb, sb, g.ptr, ldc, sc,
                                     dbias, sbias, epi, dg.GEMM_F16)
    finally:
        dg.gemm_force_config(-1)
    assert rc == 0, dg.gemm_status_string(rc)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    for i in range(batch):
        Ai = A[i if sa else 0]
        Bi = B[i if sb else 0]
        ref = oracle.gemm(M, N, K, Ai, K, Bi, K if b_col else N, b_colmajor=b_col, bias=bias[i],
                          relu=True, threads=THREADS)
        compare(g.matrix(i).double().cpu().numpy(), ref, 2, f"{name} batch {i}")
    g.check_canaries()


def test_batched_k_zero_and_shared_bias():
    batch, M, N = 2, 5, 24
    bias = torch.linspace(-2, 2, N).half()
    g = BatchGuard(batch, M, N, N, M * N + 40, torch.float16)
    rc = dg.gemm_strided_batched(batch, M, N, 0, None, 0, 0, None, 0, 0, g.ptr, N, M * N + 40,
                                 bias.cuda(), 0, dg.GEMM_EPI_BIAS | dg.GEMM_EPI_RELU, dg.GEMM_F16)
    assert rc == 0
    torch.cuda.synchronize()
    ref = oracle.gemm(M, N, 0, None, 0, None, 0, bias=bias, relu=True)
    for i in range(batch):
        compare(g.matrix(i).double().cpu().numpy(), ref, 2, "K=0 batch")
    g.check_canaries()


def test_bmm_helper_matches_torch_layouts():
    gen = torch.Generator().manual_seed(9)
    a = torch.randn(4, 130, 96, generator=gen).bfloat16().cuda()
    b = torch.randn(4, 96, 72, generator=gen).bfloat16().cuda()
    out = dg.bmm(a, b)
    torch.cuda.synchronize()
    for i in range(4):
        ref = oracle.gemm(130, 72, 96, a[i].cpu(), 96, b[i].cpu(), 72, dtype="bf16",
                          threads=THREADS)
        compare(out[i].double().cpu().numpy(), ref, 2, "bmm")


# ------------------------------------------- fp32 inputs multiplied as tf32

def _tf32_bound(A, B, bias, M, N, K, b_col, ref):
    """Error bound for fp32 inputs read as tf32: each input keeps 10 fraction
    bits (relative error below 2^-10), so a product is off by less than
    (2^-9 + 2^-20)|a b|; fp32 accumulation of K terms adds at most
    K * 2^-24 * sum|a b| in any order, bias and ReLU one more rounding."""
    S = oracle.gemm_f32(M, N, K, np.abs(A.numpy()), K, np.abs(B.numpy()), K if b_col else N,
                        b_colmajor=b_col, bias=None if bias is None else np.abs(bias.numpy()),
                        threads=THREADS)
    return (2.0 ** -9 + 2.0 ** -20 + K * 2.0 ** -23) * S + 2.0 ** -22 * np.abs(ref) + 1e-30


@pytest.mark.parametrize("config", [None, 0, 1, 8, 23])
@pytest.mark.parametrize("b_col", [False, True])
def test_tf32_within_its_error_bound(config, b_col):
    M, N, K = 333, 520, 712
    gen = torch.Generator().manual_seed(600 + (config or 0) + b_col)
    A = torch.randn(M, K, generator=gen)
    B = torch.randn(*((N, K) if b_col else (K, N)), generator=gen)
    bias = torch.randn(N, generator=gen)
    ref = oracle.gemm_f32(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col, bias=bias,
                          relu=True, threads=THREADS)
    if config is not None:
        assert dg.gemm_force_config(config) == 0
    try:
        out = dg.matmul(A.cuda(), B.cuda(), bias=bias.cuda(), relu=True, b_col_major=b_col)
        torch.cuda.synchronize()
    finally:
        dg.gemm_force_config(-1)
    assert dg.gemm_device_status() == 0
    got = out.double().cpu().numpy()
    bound = _tf32_bound(A, B, bias, M, N, K, b_col, ref)
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert (err <= bound).all(), f"max err/bound {float((err / bound).max()):.3f}"


@pytest.mark.parametrize("b_col", [False, True])
def test_tf32_exact_on_small_integers(b_col):
    """Small integers are exact in tf32 and every partial sum is an integer
    below 2^24, so the result is exact in any summation order."""
    M, N, K = 200, 264, 600
    gen = torch.Generator().manual_seed(77)
    A = torch.randint(-3, 4, (M, K), generator=gen).float()
    B = torch.randint(-3, 4, (N, K) if b_col else (K, N), generator=gen).float()
    ref = oracle.gemm_f32(M, N, K, A, K, B, K if b_col else N, b_colmajor=b_col,
                          threads=THREADS)
    out = dg.matmul(A.cuda(), B.cuda(), b_col_major=b_col)
    torch.cuda.synchronize()
    assert np.array_equal(out.double().cpu().numpy(), ref)


def test_tf32_batched_and_grouped_rejection():
    gen = torch.Generator().manual_seed(3)
    a = torch.randn(2, 96, 64, generator=gen).cuda()
    b = torch.randn(2, 64, 40, generator=gen).cuda()
    out = dg.bmm(a, b)
    torch.cuda.synchronize()
    for i in range(2):
        ref = oracle.gemm_f32(96, 40, 64, a[i].cpu(), 64, b[i].cpu(), 40, threads=THREADS)
        bound = _tf32_bound(a[i].cpu(), b[i].cpu(), None, 96, 40, 64, False, ref)
        assert (np.abs(out[i].double().cpu().numpy() - ref) <= bound).all()
    x = torch.randn(8, 64).cuda()
    w = torch.randn(1, 64, 16).cuda()
    rows = torch.tensor([8], dtype=torch.int32).cuda()
    y = torch.empty(8, 16).cuda()
    assert dg.grouped_gemm(1, rows, 8, 16, 64, x, 64, w, 16, 1024, y, 16, None, 0,
                           dg.GEMM_F32_TF32) == dg.GEMM_ERR_UNSUPPORTED


# ------------------------------------------------------ im2col convolution

@pytest.mark.parametrize("shape", [
    # batch, H, W, cin, cout, KH, KW, stride, pad, dil
    (2, 14, 14, 64, 128, 3, 3, (1, 1), (1, 1), (1, 1)),    # 3x3 same-padding
    (1, 17, 23, 32, 64, 3, 3, (2, 2), (1, 1), (1, 1)),     # stride 2, ragged image
    (2, 12, 12, 16, 40, 3, 3, (1, 1), (2, 2), (2, 2)),     # dilated
    (3, 9, 10, 64, 96, 1, 1, (1, 1), (0, 0), (1, 1)),      # 1x1 (a plain GEMM)
    (2, 20, 18, 3, 16, 5, 5, (1, 2), (2, 1), (1, 1)),      # 3 input channels (scalar gather)
])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_conv2d_im2col(shape, dtype):
    batch, H, W, cin, cout, KH, KW, stride, pad, dil = shape
    gen = torch.Generator().manual_seed(sum(shape[:7]))
    x = (torch.rand(batch, H, W, cin, generator=gen) * 2 - 1).to(dtype)
    w = (torch.randn(KH, KW, cin, cout, generator=gen) * 0.2).to(dtype)
    bias = torch.randn(cout, generator=gen).to(dtype)
    y = dg.conv2d(x.cuda(), w.cuda(), bias=bias.cuda(), relu=True, stride=stride, pad=pad,
                  dil=dil)
    torch.cuda.synchronize()
    assert dg.gemm_device_status() == 0
    ref = oracle.conv2d_nhwc(x, w, stride=stride, pad=pad, dil=dil, bias=bias, relu=True,
                             dtype="bf16" if dtype == torch.bfloat16 else "f16",
                             threads=THREADS)
    compare(y.double().cpu().numpy(), ref, 2, f"conv {shape}")

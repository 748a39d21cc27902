"""Pins for the CPU oracle: each check compares it with something other than
itself (torch's own fp16/bf16 conversions, pure-Python brute force on tiny
exact inputs, identity/permutation matrices, closed forms for all-ones
inputs, linearity, and the hand-worked case in tests/golden/).  A plausible
mistake in the oracle -- a dropped bias, ReLU before the bias, a wrong sign,
a transposed or mis-strided operand, a wrong decoder exponent -- fails at
least one of them (tests/test_oracle_mutations.py plants such mistakes and
checks exactly that)."""
import itertools
import os
import random

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16_bits(values, dtype="f16"):
    t = torch.tensor(values, dtype=torch.float64).to(
        torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


# ----------------------------------------------------------------- decoders

@pytest.mark.parametrize("dtype,tdt", [("f16", torch.float16), ("bf16", torch.bfloat16)])
def test_decoder_exhaustive_against_torch(dtype, tdt):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(bits, dtype)
    theirs = torch.from_numpy(bits.view(np.int16).copy()).view(tdt).double().numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], theirs[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(theirs[~nan]))


def test_decoder_known_values():
    # IEEE binary16: 1.0 = 0x3C00, -2 = 0xC000, max normal 65504 = 0x7BFF,
    # smallest subnormal 2^-24 = 0x0001, smallest normal 2^-14 = 0x0400.
    assert oracle.decode_scalar(0x3C00, "f16") == 1.0
    assert oracle.decode_scalar(0xC000, "f16") == -2.0
    assert oracle.decode_scalar(0x7BFF, "f16") == 65504.0
    assert oracle.decode_scalar(0x0001, "f16") == 2.0 ** -24
    assert oracle.decode_scalar(0x0400, "f16") == 2.0 ** -14
    # bfloat16 = top half of binary32: 1.0 = 0x3F80, -2 = 0xC000, 2^-133 = 0x0001
    assert oracle.decode_scalar(0x3F80, "bf16") == 1.0
    assert oracle.decode_scalar(0xC000, "bf16") == -2.0
    assert oracle.decode_scalar(0x0001, "bf16") == 2.0 ** -133
    assert oracle.decode_scalar(0x7F7F, "bf16") == (2 - 2 ** -7) * 2.0 ** 127


# ----------------------------------------------------------- brute force

_EXACT = [-2.0, -1.5, -1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0, 1.5, 2.0]


def _brute(A, B, M, N, K, bias=None, relu=False):
    """Pure-Python definition on Python floats (all products and sums here
    are exact dyadic rationals far inside double range)."""
    C = [[0.0] * N for _ in range(M)]
    for i in range(M):
        for j in range(N):
            s = 0.0
            for k in range(K):
                s += A[i][k] * B[k][j]
            if bias is not None:
                s += bias[j]
            if relu:
                s = max(s, 0.0)
            C[i][j] = s
    return C


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("b_colmajor", [False, True])
@pytest.mark.parametrize("epi", ["none", "bias", "bias_relu", "relu"])
def test_bruteforce_tiny(dtype, b_colmajor, epi):
    rnd = random.Random(f"{dtype}-{b_colmajor}-{epi}")
    for M, N, K in itertools.product([1, 2, 3], [1, 2, 4], [1, 3, 4]):
        A = [[rnd.choice(_EXACT) for _ in range(K)] for _ in range(M)]
        B = [[rnd.choice(_EXACT) for _ in range(N)] for _ in range(K)]
        bias = [rnd.choice(_EXACT) for _ in range(N)] if "bias" in epi else None
        relu = "relu" in epi
        # padded leading dimensions whose padding would poison any stray read
        lda, ldb = K + 2, (K + 3 if b_colmajor else N + 1)
        a_buf = np.full(M * lda, 999.0)
        for i in range(M):
            a_buf[i * lda:i * lda + K] = A[i]
        if b_colmajor:
            b_buf = np.full(N * ldb, -777.0)
            for j in range(N):
                for k in range(K):
                    b_buf[j * ldb + k] = B[k][j]
        else:
            b_buf = np.full(K * ldb, -777.0)
            for k in range(K):
                b_buf[k * ldb:k * ldb + N] = B[k]
        got = oracle.gemm(M, N, K, f16_bits(a_buf, dtype), lda, f16_bits(b_buf, dtype), ldb,
                          b_colmajor=b_colmajor,
                          bias=None if bias is None else f16_bits(bias, dtype),
                          relu=relu, dtype=dtype)
        exp = np.array(_brute(A, B, M, N, K, bias, relu))
        assert np.array_equal(got, exp), (M, N, K)


def test_golden_worked_example():
    fields = {}
    with open(os.path.join(GOLDEN, "worked_gemm_2x3x2.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *vals = line.split()
                fields[key] = [float(v) for v in vals]
    M, N, K = int(fields["M"][0]), int(fields["N"][0]), int(fields["K"][0])
    for dtype in ["f16", "bf16"]:
        A, B, bias = (f16_bits(fields[k], dtype) for k in ("A", "B", "bias"))
        plain = oracle.gemm(M, N, K, A, K, B, N, dtype=dtype)
        with_bias = oracle.gemm(M, N, K, A, K, B, N, bias=bias, dtype=dtype)
        both = oracle.gemm(M, N, K, A, K, B, N, bias=bias, relu=True, dtype=dtype)
        assert plain.ravel().tolist() == fields["C_plain"]
        assert with_bias.ravel().tolist() == fields["C_bias"]
        assert both.ravel().tolist() == fields["C_bias_relu"]


# ------------------------------------------------- structural properties

def _rand_bits(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    t = (torch.rand(*shape, generator=g) * 2 - 1).to(
        torch.float16 if dtype == "f16" else torch.bfloat16)
    return t


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("b_colmajor", [False, True])
def test_identity(dtype, b_colmajor):
    M, K = 37, 70
    A = _rand_bits((M, K), dtype, 5)
    I = torch.eye(K, dtype=A.dtype)
    got = oracle.gemm(M, K, K, A, K, I, K, b_colmajor=b_colmajor, dtype=dtype)
    assert np.array_equal(got, A.double().numpy())


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_permutation(dtype):
    M, K = 19, 48
    A = _rand_bits((M, K), dtype, 6)
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(3))
    P = torch.zeros(K, K, dtype=A.dtype)
    P[perm, torch.arange(K)] = 1  # (A.P)[:, j] = A[:, perm[j]]
    got = oracle.gemm(M, K, K, A, K, P, K, dtype=dtype)
    assert np.array_equal(got, A.double().numpy()[:, perm.numpy()])
    # column-major storage of the same P
    Pc = P.t().contiguous()
    got_c = oracle.gemm(M, K, K, A, K, Pc, K, b_colmajor=True, dtype=dtype)
    assert np.array_equal(got_c, got)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_all_ones_closed_forms(dtype):
    M, N, K = 9, 13, 300
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    ones_kn = torch.ones(K, N, dtype=tdt)
    g = torch.Generator().manual_seed(11)
    A_int = torch.randint(-3, 4, (M, K), generator=g)
    A = A_int.to(tdt)
    got = oracle.gemm(M, N, K, A, K, ones_kn, N, dtype=dtype)
    rowsum = [sum(int(v) for v in A_int[i].tolist()) for i in range(M)]  # Python ints
    assert np.array_equal(got, np.repeat(np.array(rowsum, dtype=np.float64)[:, None], N, 1))
    got2 = oracle.gemm(M, N, K, torch.ones(M, K, dtype=tdt), K, ones_kn, N, dtype=dtype)
    assert np.all(got2 == float(K))


def test_linearity_in_A():
    rng = np.random.default_rng(7)
    M, N, K = 23, 17, 129
    A1, A2 = rng.standard_normal((M, K)), rng.standard_normal((M, K))
    B = rng.standard_normal((K, N))
    lhs = oracle.gemm_f64(A1 + A2, B)
    rhs = oracle.gemm_f64(A1, B) + oracle.gemm_f64(A2, B)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    # scaling by 2 is exact in binary floating point
    assert np.array_equal(oracle.gemm_f64(2 * A1, B), 2 * oracle.gemm_f64(A1, B))


def test_bias_then_relu_order_and_sign():
    # A.B = -1 everywhere, bias = +2  ->  relu(-1 + 2) = 1 (ReLU before the bias would give 2)
    for dtype in ["f16", "bf16"]:
        A = f16_bits([-1.0], dtype)
        B = f16_bits([1.0, 1.0], dtype)
        bias = f16_bits([2.0, -0.5], dtype)
        got = oracle.gemm(1, 2, 1, A, 1, B, 2, bias=bias, relu=True, dtype=dtype)
        assert got.tolist() == [[1.0, 0.0]]
        # A = 0: C = relu(bias) broadcast over rows
        Z = f16_bits([0.0] * 6, dtype)
        B3 = f16_bits([1.5] * 6, dtype)
        got = oracle.gemm(2, 2, 3, Z, 3, B3, 2, bias=bias, relu=True, dtype=dtype)
        assert got.tolist() == [[2.0, 0.0], [2.0, 0.0]]


def test_k_zero_is_bias_only():
    bias = f16_bits([3.0, -4.0, 0.5])
    got = oracle.gemm(2, 3, 0, None, 0, None, 0, bias=bias, relu=True)
    assert got.tolist() == [[3.0, 0.0, 0.5]] * 2
    got = oracle.gemm(2, 3, 0, None, 0, None, 0)
    assert np.all(got == 0.0)


@pytest.mark.parametrize("b_colmajor", [False, True])
def test_sampled_matches_brute_force(b_colmajor):
    rnd = random.Random(99)
    M, N, K = 5, 7, 6
    A = [[rnd.choice(_EXACT) for _ in range(K)] for _ in range(M)]
    B = [[rnd.choice(_EXACT) for _ in range(N)] for _ in range(K)]
    bias = [rnd.choice(_EXACT) for _ in range(N)]
    exp = _brute(A, B, M, N, K, bias, True)
    lda = K + 3
    a_buf = [999.0] * (M * lda)
    for i in range(M):
        a_buf[i * lda:i * lda + K] = A[i]
    if b_colmajor:  # stored (N, K) with padding
        ldb = K + 2
        b_buf = [-55.0] * (N * ldb)
        for j in range(N):
            for k in range(K):
                b_buf[j * ldb + k] = B[k][j]
    else:
        ldb = N + 5
        b_buf = [-55.0] * (K * ldb)
        for k in range(K):
            b_buf[k * ldb:k * ldb + N] = B[k]
    rows = np.array([i for i in range(M) for j in range(N)])
    cols = np.array([j for i in range(M) for j in range(N)])
    got = oracle.gemm_at(M, N, K, f16_bits(a_buf), lda, f16_bits(b_buf), ldb, rows, cols,
                         b_colmajor=b_colmajor, bias=f16_bits(bias), relu=True)
    assert got.tolist() == [exp[i][j] for i, j in zip(rows, cols)]


# ------------------------------------------------------------------ grouped

def test_grouped_bruteforce_with_empty_and_single_row_groups():
    rnd = random.Random(5)
    group_rows = [0, 3, 1, 0, 2]
    G, N, K = len(group_rows), 4, 5
    total = sum(group_rows)
    X = [[rnd.choice(_EXACT) for _ in range(K)] for _ in range(total)]
    W = [[[rnd.choice(_EXACT) for _ in range(N)] for _ in range(K)] for _ in range(G)]
    bias = [[rnd.choice(_EXACT) for _ in range(N)] for _ in range(G)]
    exp, r0 = [], 0
    for g, m in enumerate(group_rows):
        exp += _brute(X[r0:r0 + m], W[g], m, N, K, bias[g], True)
        r0 += m
    w_flat = [v for g in range(G) for row in W[g] for v in row]
    got = oracle.grouped_gemm(group_rows, N, K, f16_bits(sum(X, []), "bf16"), K,
                              f16_bits(w_flat, "bf16"), N, K * N,
                              bias=f16_bits(sum(bias, []), "bf16"), relu=True, dtype="bf16")
    assert got.tolist() == exp
    rows = np.arange(total).repeat(N)
    cols = np.tile(np.arange(N), total)
    got_at = oracle.grouped_gemm_at(group_rows, N, K, f16_bits(sum(X, []), "bf16"), K,
                                    f16_bits(w_flat, "bf16"), N, K * N, rows, cols,
                                    bias=f16_bits(sum(bias, []), "bf16"), relu=True,
                                    dtype="bf16")
    assert got_at.tolist() == [exp[r][c] for r, c in zip(rows, cols)]


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.gemm_at(2, 2, 1, f16_bits([1, 1]), 1, f16_bits([1, 1]), 2,
                       np.array([2]), np.array([0]))  # row out of range
    with pytest.raises(ValueError):
        oracle.grouped_gemm([1, -1], 2, 1, f16_bits([1]), 1, f16_bits([1, 1, 1, 1]), 2, 2)


def test_tolerance_helper():
    ok, *_ = oracle.within_tolerance(np.array([1.021]), np.array([1.0]), 1e-2, 1e-2)
    assert not ok
    ok, *_ = oracle.within_tolerance(np.array([1.0199]), np.array([1.0]), 1e-2, 1e-2)
    assert ok
    ok, *_ = oracle.within_tolerance(np.array([np.nan]), np.array([1.0]), 1e-2, 1e-2)
    assert not ok


# ------------------------------------------------------------ fp32 inputs

@pytest.mark.parametrize("b_colmajor", [False, True])
def test_f32_bruteforce_with_strides(b_colmajor):
    rnd = random.Random(f"f32-{b_colmajor}")
    vals = _EXACT + [3.0e-5, -7.5, 1024.125, 1.0 / 3.0]
    for M, N, K in [(1, 1, 1), (2, 3, 4), (3, 5, 2)]:
        A = [[np.float32(rnd.choice(vals)) for _ in range(K)] for _ in range(M)]
        B = [[np.float32(rnd.choice(vals)) for _ in range(N)] for _ in range(K)]
        bias = [np.float32(rnd.choice(vals)) for _ in range(N)]
        lda, ldb = K + 3, (K + 1 if b_colmajor else N + 2)
        a_buf = np.full(M * lda, 1e30, dtype=np.float32)
        for i in range(M):
            a_buf[i * lda:i * lda + K] = A[i]
        if b_colmajor:
            b_buf = np.full(N * ldb, -1e30, dtype=np.float32)
            for j in range(N):
                for k in range(K):
                    b_buf[j * ldb + k] = B[k][j]
        else:
            b_buf = np.full(K * ldb, -1e30, dtype=np.float32)
            for k in range(K):
                b_buf[k * ldb:k * ldb + N] = B[k]
        got = oracle.gemm_f32(M, N, K, a_buf, lda, b_buf, ldb, b_colmajor=b_colmajor,
                              bias=np.array(bias, dtype=np.float32), relu=True)
        # exact reference with Python fractions on the fp32 values
        from fractions import Fraction
        for i in range(M):
            for j in range(N):
                s_ = sum(Fraction(float(A[i][k])) * Fraction(float(B[k][j])) for k in range(K))
                s_ += Fraction(float(bias[j]))
                s_ = max(s_, Fraction(0))
                assert abs(Fraction(got[i, j]) - s_) <= abs(s_) * Fraction(1, 2 ** 50), (i, j)


# ------------------------------------------------------------ convolution

def _conv_brute(x, w, stride, pad, dil, bias, relu):
    """Direct convolution on nested Python lists of exact floats."""
    batch, H, W, cin = len(x), len(x[0]), len(x[0][0]), len(x[0][0][0])
    KH, KW, cout = len(w), len(w[0]), len(w[0][0][0])
    OH, OW = oracle.conv_out_size(H, W, KH, KW, stride, pad, dil)
    y = [[[[0.0] * cout for _ in range(OW)] for _ in range(OH)] for _ in range(batch)]
    for n in range(batch):
        for oh in range(OH):
            for ow in range(OW):
                for co in range(cout):
                    s_ = 0.0
                    for kh in range(KH):
                        for kw in range(KW):
                            ih = oh * stride[0] - pad[0] + kh * dil[0]
                            iw = ow * stride[1] - pad[1] + kw * dil[1]
                            if 0 <= ih < H and 0 <= iw < W:
                                for ci in range(cin):
                                    s_ += x[n][ih][iw][ci] * w[kh][kw][ci][co]
                    if bias is not None:
                        s_ += bias[co]
                    y[n][oh][ow][co] = max(s_, 0.0) if relu else s_
    return y


@pytest.mark.parametrize("geom", [((1, 1), (0, 0), (1, 1)), ((1, 1), (1, 1), (1, 1)),
                                  ((2, 1), (1, 2), (1, 1)), ((1, 2), (2, 1), (2, 1)),
                                  ((1, 1), (0, 1), (2, 2))])
def test_conv_bruteforce(geom):
    stride, pad, dil = geom
    rnd = random.Random(str(geom))
    batch, H, W, cin, cout, KH, KW = 2, 5, 4, 3, 2, 3, 2
    x = [[[[rnd.choice(_EXACT) for _ in range(cin)] for _ in range(W)] for _ in range(H)]
         for _ in range(batch)]
    w = [[[[rnd.choice(_EXACT) for _ in range(cout)] for _ in range(cin)] for _ in range(KW)]
         for _ in range(KH)]
    bias = [rnd.choice(_EXACT) for _ in range(cout)]
    xt = torch.tensor(x, dtype=torch.float64).half()
    wt = torch.tensor(w, dtype=torch.float64).half()
    got = oracle.conv2d_nhwc(xt, wt, stride=stride, pad=pad, dil=dil,
                             bias=torch.tensor(bias).half(), relu=True)
    assert np.array_equal(got, np.array(_conv_brute(x, w, stride, pad, dil, bias, True)))


def test_conv_delta_filter_copies_the_input():
    x = _rand_bits((2, 6, 7, 4), "bf16", 21)
    w = torch.zeros(3, 3, 4, 4, dtype=torch.bfloat16)
    for c in range(4):
        w[1, 1, c, c] = 1  # centre tap, channel c -> c
    got = oracle.conv2d_nhwc(x, w, pad=(1, 1), dtype="bf16")
    assert np.array_equal(got, x.double().numpy())


def test_conv_1x1_is_a_matrix_product():
    x = _rand_bits((2, 3, 5, 8), "f16", 22)
    w = _rand_bits((1, 1, 8, 6), "f16", 23)
    got = oracle.conv2d_nhwc(x, w)
    xs = x.double().numpy().reshape(-1, 8)
    ws = w.double().numpy().reshape(8, 6)
    exp = [[sum(xs[r, k] * ws[k, c] for k in range(8)) for c in range(6)] for r in range(xs.shape[0])]
    assert np.allclose(got.reshape(-1, 6), np.array(exp), rtol=0, atol=1e-12)

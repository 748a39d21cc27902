"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds the workload definitions (shapes, dtypes, layouts, value
distributions, seeds) and the random generators that fill them.  It holds
none of the GEMM's arithmetic: neither the oracle nor the CUDA path is
imported here, and both sides receive the same tensors from it.

The shapes are the pages' own: the 1024x1024x2048 fp16 case of
"用Triton跨芯片优化GEMM" section 2.3, the 2048/4096/8192 cubes of the results
table in the crowd-sourced tuning page (section 3.4), and its "square /
skinny / batch / large-K" families (section 4.3 of the first page); the MoE
layer of 32 experts stands for the "dozens of GEMMs" the first page names in
section 2.3.  No public dataset is involved: every value is drawn here.

Recipe (all CPU, then copied to the device by the caller):
  * uniform[-1, 1]: torch.rand(float32, Generator(seed)) * 2 - 1, cast RNE;
  * normal(0, s):   torch.randn(float32, Generator(seed)) * s, cast RNE;
  * MoE routing:    numpy.random.default_rng(seed): p ~ Dirichlet(1 * ones(E)),
                    rows ~ Multinomial(total_rows, p); rows sorted by expert.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

_TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def uniform_pm1(shape, dtype: str, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    x = torch.rand(*shape, generator=g, dtype=torch.float32)
    return (x * 2.0 - 1.0).to(_TORCH_DT[dtype])


def normal(shape, dtype: str, seed: int, std: float = 1.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    return (x * std).to(_TORCH_DT[dtype])


def small_ints(shape, dtype: str, seed: int, lo: int = -2, hi: int = 2) -> torch.Tensor:
    """Integers in [lo, hi]: every partial sum of a K <= 4096 product stays an
    integer below 2^24, so fp32 accumulation is exact in any order."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randint(lo, hi + 1, tuple(shape), generator=g).to(_TORCH_DT[dtype])


def moe_group_rows(num_experts: int, total_rows: int, seed: int) -> np.ndarray:
    """Rows per expert: Multinomial(total_rows, Dirichlet(1)) with a fixed seed."""
    rng = np.random.default_rng(int(seed))
    p = rng.dirichlet(np.ones(num_experts))
    return rng.multinomial(total_rows, p).astype(np.int32)


@dataclass
class Workload:
    name: str
    M: int
    N: int
    K: int
    dtype: str                   # input dtype: "f16" or "bf16"
    out: str = ""                # output dtype; "" = same as input
    dist: str = "uniform"        # "uniform" | "normal" | "ints"
    seed: int = 0
    b_colmajor: bool = False
    bias: bool = False
    relu: bool = False
    bias_seed: int = 0
    # grouped (MoE) workloads
    experts: int = 0
    w_std: float = 1.0
    group_rows: Optional[np.ndarray] = field(default=None, repr=False)

    @property
    def out_dtype(self) -> str:
        return self.out or self.dtype

    @property
    def grouped(self) -> bool:
        return self.experts > 0

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


def _w(**kw) -> Workload:
    return Workload(**kw)


# The five configurations of the path (the first is the small case the oracle
# checks in full in well under a second).
WORKLOADS = {w.name: w for w in [
    _w(name="square256_f16", M=256, N=256, K=256, dtype="f16", seed=1),
    _w(name="m1024n1024k2048_f16", M=1024, N=1024, K=2048, dtype="f16", seed=2),
    _w(name="m1024n1024k2048_f16_bias_relu", M=1024, N=1024, K=2048, dtype="f16", seed=2,
       bias=True, relu=True, bias_seed=3),
    _w(name="square4096_bf16", M=4096, N=4096, K=4096, dtype="bf16", dist="normal", seed=4),
    _w(name="square4096_f16", M=4096, N=4096, K=4096, dtype="f16", dist="normal", seed=5),
    _w(name="square8192_bf16", M=8192, N=8192, K=8192, dtype="bf16", dist="normal", seed=6),
    _w(name="square8192_f16", M=8192, N=8192, K=8192, dtype="f16", dist="normal", seed=7),
    _w(name="m1000n1000k2000_f16_bcol", M=1000, N=1000, K=2000, dtype="f16", seed=8,
       b_colmajor=True),
    _w(name="m4096n4096k512_f16_bcol", M=4096, N=4096, K=512, dtype="f16", seed=9,
       b_colmajor=True),
    _w(name="m16n8192k8192_f16_bcol", M=16, N=8192, K=8192, dtype="f16", seed=10,
       b_colmajor=True),
    # profiling case: operands (144 MiB) larger than L2, small enough for a full ncu capture
    _w(name="square6144_bf16", M=6144, N=6144, K=6144, dtype="bf16", dist="normal", seed=12),
    _w(name="moe32_m8192n1408k4096_bf16_relu", M=8192, N=1408, K=4096, dtype="bf16",
       dist="normal", seed=11, relu=True, experts=32, w_std=0.02),
    # two more routings with the same generator: few large experts, and many
    # experts with a narrow N (the swept grouped classes)
    _w(name="moe8_m16384n4096k4096_bf16_relu", M=16384, N=4096, K=4096, dtype="bf16",
       dist="normal", seed=11, relu=True, experts=8, w_std=0.02),
    _w(name="moe64_m8192n768k2048_bf16_relu", M=8192, N=768, K=2048, dtype="bf16",
       dist="normal", seed=11, relu=True, experts=64, w_std=0.02),
]}


def get(name: str) -> Workload:
    w = WORKLOADS[name]
    if w.grouped and w.group_rows is None:
        w.group_rows = moe_group_rows(w.experts, w.M, w.seed)
    return w


def make_inputs(w: Workload):
    """(A, B, bias) on the CPU for a dense workload.

    A is (M, K) row-major.  B is (K, N) row-major, or stored (N, K) when
    ``b_colmajor`` (B[k, n] at n*ldb + k).  bias is (N,) or None."""
    if w.grouped:
        raise ValueError("use make_grouped_inputs for grouped workloads")
    if w.dist == "uniform":
        gen = lambda shape, seed: uniform_pm1(shape, w.dtype, seed)
    elif w.dist == "normal":
        gen = lambda shape, seed: normal(shape, w.dtype, seed)
    else:
        gen = lambda shape, seed: small_ints(shape, w.dtype, seed)
    A = gen((w.M, w.K), w.seed)
    B = gen((w.N, w.K) if w.b_colmajor else (w.K, w.N), w.seed + 100003)
    bias = uniform_pm1((w.N,), w.dtype, w.bias_seed) if w.bias else None
    return A, B, bias


def make_grouped_inputs(w: Workload):
    """(X, W, group_rows, bias) on the CPU for a grouped workload.

    X is (sum rows, K) with rows sorted by expert; W is (E, K, N) row-major
    (or (E, N, K) when ``b_colmajor``); group_rows is int32 (E,)."""
    w = get(w.name) if w.group_rows is None else w
    X = normal((int(w.group_rows.sum()), w.K), w.dtype, w.seed)
    shape = (w.experts, w.N, w.K) if w.b_colmajor else (w.experts, w.K, w.N)
    W = normal(shape, w.dtype, w.seed + 100003, std=w.w_std)
    bias = uniform_pm1((w.experts, w.N), w.dtype, w.bias_seed) if w.bias else None
    return X, W, np.asarray(w.group_rows, dtype=np.int32), bias


def sample_indices(M: int, N: int, n: int = 4096, seed: int = 1234, tile_m: int = 128,
                   tile_n: int = 128, group_rows=None, per_group: int = 8):
    """The sampled-check index set: n uniform draws over [0,M) x [0,N) from
    default_rng(seed), plus the four corners, the last row / column of every
    tile boundary, and (grouped) at least ``per_group`` elements from every
    non-empty group."""
    rng = np.random.default_rng(seed)
    rows = list(rng.integers(0, M, size=n))
    cols = list(rng.integers(0, N, size=n))
    for r, c in [(0, 0), (0, N - 1), (M - 1, 0), (M - 1, N - 1)]:
        rows.append(r)
        cols.append(c)
    for r in range(tile_m - 1, M, tile_m):
        rows.append(r)
        cols.append(int(rng.integers(0, N)))
    for c in range(tile_n - 1, N, tile_n):
        rows.append(int(rng.integers(0, M)))
        cols.append(c)
    if group_rows is not None:
        start = 0
        for m in np.asarray(group_rows, dtype=np.int64):
            if m > 0:
                for _ in range(per_group):
                    rows.append(int(start + rng.integers(0, m)))
                    cols.append(int(rng.integers(0, N)))
                rows.append(int(start + m - 1))
                cols.append(int(rng.integers(0, N)))
            start += int(m)
    return np.asarray(rows, dtype=np.int64), np.asarray(cols, dtype=np.int64)

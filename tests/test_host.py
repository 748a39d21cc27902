"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every function include/dense_gemm.h declares, its host helpers reproduce the
pages' worked numbers, and every argument error is reported before anything
touches CUDA."""
import ctypes
import os

import pytest

import dense_gemm_16_b200 as dg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(dg.LIB_PATH):
        from dense_gemm_16_b200 import build
        build.build()
    return dg.lib()


def test_exports_every_declared_symbol():
    names = dg.header_functions()
    assert {"gemm", "grouped_gemm", "gemm_status_string"} <= set(names)
    L = dg.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_version_and_status_strings():
    assert "sm_100a" in dg.gemm_version()
    for s in [0, -1, -2, -3, -4, -5]:
        assert dg.gemm_status_string(s).startswith("GEMM_")
    assert "unknown" in dg.gemm_status_string(12345)


def _golden_rows(kind):
    with open(os.path.join(GOLDEN, "pages_worked_numbers.txt")) as f:
        for line in f:
            if line.startswith(kind + " "):
                yield dict(kv.split("=") for kv in line.split()[1:])


def test_pages_smem_formula():
    rows = list(_golden_rows("smem_ring"))
    assert rows
    for r in rows:
        got = dg.gemm_smem_ring_bytes(int(r["BM"]), int(r["BN"]), int(r["BK"]),
                                      int(r["stages"]), int(r["elem_bytes"]))
        assert got == int(r["expect"])
    assert dg.gemm_smem_ring_bytes(-1, 1, 1, 1, 1) == -1


def test_pages_k_iterations():
    for r in _golden_rows("k_iters"):
        assert dg.gemm_k_iterations(int(r["K"]), int(r["BK"])) == int(r["expect"])
    assert dg.gemm_k_iterations(2000, 64) == 32  # ragged K rounds up
    assert dg.gemm_k_iterations(1, 0) == -1


def test_pages_raster_block_counts():
    """9x9 tile grid: the first 9 tiles read 90 input blocks in row-major
    order and 54 in 3x3 grouped order (9 K-blocks per panel)."""
    for r in _golden_rows("raster"):
        gm, gn, tiles, kb = (int(r[k]) for k in ("grid_m", "grid_n", "tiles", "k_blocks"))
        coords = [dg.gemm_tile_coord(t, gm, gn, int(r["group_m"])) for t in range(tiles)]
        a_panels = {m for m, _ in coords}
        b_panels = {n for _, n in coords}
        assert (len(a_panels) + len(b_panels)) * kb == int(r["expect"])


@pytest.mark.parametrize("gm,gn,group", [(9, 9, 3), (7, 5, 8), (32, 16, 8), (5, 1, 4), (1, 7, 1)])
def test_raster_is_a_permutation(gm, gn, group):
    seen = {dg.gemm_tile_coord(t, gm, gn, group) for t in range(gm * gn)}
    assert seen == {(m, n) for m in range(gm) for n in range(gn)}


def test_raster_group_one_is_row_major():
    for t in range(35):
        assert dg.gemm_tile_coord(t, 5, 7, 1) == (t // 7, t % 7)


def test_configs_listed_and_forcing_bounds():
    n = dg.gemm_num_configs()
    assert n >= 3
    names = [dg.gemm_config_name(i) for i in range(n)]
    assert len(set(names)) == n
    with pytest.raises(dg.GemmError):
        dg.gemm_config_name(n)
    assert dg.gemm_force_config(n) == dg.GEMM_ERR_UNSUPPORTED
    assert dg.gemm_force_config(-2) == dg.GEMM_ERR_UNSUPPORTED
    assert dg.gemm_force_config(0) == 0
    assert dg.gemm_select_config(4096, 4096, 4096, dg.GEMM_BF16, 0) == 0
    assert dg.gemm_force_config(-1) == 0


def test_select_config_shape_classes():
    bcol = dg.GEMM_B_COL_MAJOR
    skinny = dg.gemm_select_config(16, 8192, 8192, dg.GEMM_F16, bcol)
    assert dg.gemm_config_name(skinny).startswith("swap")
    big = dg.gemm_select_config(8192, 8192, 8192, dg.GEMM_BF16, 0)
    assert not dg.gemm_config_name(big).startswith("swap")
    assert dg.gemm_select_config(-1, 1, 1, 0, 0) == dg.GEMM_ERR_INVALID_ARG
    assert dg.gemm_select_config(1, 1, 1, 9, 0) == dg.GEMM_ERR_UNSUPPORTED


@pytest.mark.parametrize("M,N,K,dtype,epi,prefix", [
    (8192, 8192, 8192, "bf16", 0, "pair_256x512"),  # measured rule: CTA-pair 256 x 512 tiles
    (4096, 4096, 4096, "bf16", 0, "pair_256x512"),
    (1024, 1024, 2048, "f16", 0, "csk_"),           # the pages' shape: CTA-pair split-K
    (512, 512, 2048, "f16", 0, "csk_"),             # no rule: few tiles, long K -> pair split-K
    (512, 512, 256, "f16", 0, "tc1_128x128"),       # few tiles, short K -> 128 x 128 tiles
    (3000, 3000, 3000, "bf16", 0, "pair_256x256"),  # no rule: >= 128 pair tiles, K >= 1024
    (16, 8192, 8192, "f16", 0x100, "swap_128x16"),  # skinny, B column-major -> swapped operands
    (24, 4096, 4096, "f16", 0x100, "swap_128x32"),
])
def test_table_and_fallback_choices(M, N, K, dtype, epi, prefix):
    code = dg.GEMM_BF16 if dtype == "bf16" else dg.GEMM_F16
    cid = dg.gemm_select_config(M, N, K, code, epi)
    assert dg.gemm_config_name(cid).startswith(prefix), dg.gemm_config_name(cid)


# Fake, never-dereferenced device addresses: every case below must be
# rejected by the host checks before any CUDA call.
P = 1 << 20  # 16-byte aligned


@pytest.mark.parametrize("args,expect", [
    # (M, N, K, A, lda, B, ldb, C, ldc, bias, epi, dtype)
    ((4, 4, 4, P, 8, P, 8, P, 8, None, 0, 7), dg.GEMM_ERR_UNSUPPORTED),           # dtype
    ((4, 4, 4, P, 8, P, 8, P, 8, None, 0x10, 0), dg.GEMM_ERR_UNSUPPORTED),        # epilogue bit
    ((-1, 4, 4, P, 8, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),          # negative M
    ((4, 4, -3, P, 8, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),          # negative K
    ((4, 4, 4, None, 8, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),        # null A
    ((4, 4, 4, P, 8, None, 8, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),        # null B
    ((4, 4, 4, P, 8, P, 8, None, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),        # null C
    ((4, 4, 4, P, 8, P, 8, P, 8, None, 1, 0), dg.GEMM_ERR_INVALID_ARG),           # bias flag, no bias
    ((4, 4, 16, P, 8, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),          # lda < K
    ((4, 16, 4, P, 8, P, 8, P, 16, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),         # ldb < N
    ((4, 4, 16, P, 16, P, 8, P, 8, None, 0x100, 0), dg.GEMM_ERR_INVALID_ARG),     # col-major ldb < K
    ((4, 16, 4, P, 8, P, 16, P, 8, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),         # ldc < N
    ((4, 4, 4, P + 2, 8, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_MISALIGNED),        # A pointer
    ((4, 4, 4, P, 8, P + 8, 8, P, 8, None, 0, 0), dg.GEMM_ERR_MISALIGNED),        # B pointer
    ((4, 4, 4, P, 8, P, 8, P + 4, 8, None, 0, 0), dg.GEMM_ERR_MISALIGNED),        # C pointer
    ((4, 4, 4, P, 12, P, 8, P, 8, None, 0, 0), dg.GEMM_ERR_MISALIGNED),           # lda % 8
    ((4, 4, 4, P, 8, P, 10, P, 8, None, 0, 0), dg.GEMM_ERR_MISALIGNED),           # ldb % 8
    ((4, 4, 4, P, 8, P, 8, P, 6, None, 0, 0), dg.GEMM_ERR_MISALIGNED),            # ldc*2 % 16
    ((4, 4, 4, P, 8, P, 8, P, 6, None, 0, 2), dg.GEMM_ERR_MISALIGNED),            # ldc*4 % 16 (f32)
    ((4, 4, 4, P, 8, P, 8, P, 8, P + 1, 1, 0), dg.GEMM_ERR_MISALIGNED),           # bias alignment
])
def test_gemm_argument_errors(args, expect):
    M, N, K, A, lda, B, ldb, C, ldc, bias, epi, dtype = args
    assert dg.lib().gemm(M, N, K, A, lda, B, ldb, C, ldc, bias, epi, dtype, None) == expect


def test_gemm_empty_is_a_noop_without_touching_cuda():
    L = dg.lib()
    assert L.gemm(0, 5, 5, None, 0, None, 0, None, 0, None, 0, 0, None) == 0
    assert L.gemm(5, 0, 5, None, 0, None, 0, None, 0, None, 0, 0, None) == 0


@pytest.mark.parametrize("args,expect", [
    # (G, rows, total, N, K, A, lda, B, ldb, stride_b, C, ldc, bias, epi, dtype)
    ((0, P, 8, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 1), dg.GEMM_ERR_INVALID_ARG),      # no groups
    ((1025, P, 8, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 1), dg.GEMM_ERR_INVALID_ARG),   # too many
    ((2, None, 8, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 1), dg.GEMM_ERR_INVALID_ARG),   # null rows
    ((2, P, -1, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 1), dg.GEMM_ERR_INVALID_ARG),     # total < 0
    ((2, P, 8, 8, 8, P, 8, P, 8, 56, P, 8, None, 0, 1), dg.GEMM_ERR_INVALID_ARG),      # overlapping B
    ((2, P, 8, 8, 8, P, 8, P, 8, 68, P, 8, None, 0, 1), dg.GEMM_ERR_MISALIGNED),       # stride_b*2 % 16
    ((2, P + 2, 8, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 1), dg.GEMM_ERR_MISALIGNED),   # rows pointer
    ((2, P, 8, 8, 8, P, 8, P, 8, 64, P, 8, None, 0, 5), dg.GEMM_ERR_UNSUPPORTED),      # dtype
])
def test_grouped_argument_errors(args, expect):
    assert dg.lib().grouped_gemm(*args, None) == expect


def test_valid_call_without_a_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    L = dg.lib()
    assert L.gemm(4, 4, 4, P, 8, P, 8, P, 8, None, 0, 0, None) == dg.GEMM_ERR_CUDA
    assert L.gemm_device_status(None, 0) == dg.GEMM_ERR_CUDA


@pytest.mark.parametrize("args,expect", [
    # (batch, M, N, K, A, lda, sA, B, ldb, sB, C, ldc, sC, bias, sbias, epi, dtype)
    ((-1, 4, 8, 8, P, 8, 64, P, 8, 64, P, 8, 32, None, 0, 0, 0), dg.GEMM_ERR_INVALID_ARG),
    ((2, 4, 8, 8, P, 8, 16, P, 8, 64, P, 8, 32, None, 0, 0, 0), dg.GEMM_ERR_INVALID_ARG),   # A overlaps
    ((2, 4, 8, 8, P, 8, 32, P, 8, 40, P, 8, 32, None, 0, 0, 0), dg.GEMM_ERR_INVALID_ARG),   # B overlaps
    ((2, 4, 8, 8, P, 8, 32, P, 8, 64, P, 8, 24, None, 0, 0, 0), dg.GEMM_ERR_INVALID_ARG),   # C overlaps
    ((2, 4, 8, 8, P, 8, 36, P, 8, 64, P, 8, 32, None, 0, 0, 0), dg.GEMM_ERR_MISALIGNED),    # sA*2 % 16
    ((2, 4, 8, 8, P, 8, 32, P, 8, 64, P, 8, 36, None, 0, 0, 0), dg.GEMM_ERR_MISALIGNED),    # sC*2 % 16
    ((2, 4, 8, 8, P, 8, 32, P, 8, 64, P, 8, 32, None, -8, 0, 0), dg.GEMM_ERR_INVALID_ARG),  # sbias < 0
])
def test_batched_argument_errors(args, expect):
    assert dg.lib().gemm_strided_batched(*args, None) == expect


def test_batched_empty_is_a_noop():
    assert dg.lib().gemm_strided_batched(0, 4, 4, 4, P, 8, 32, P, 8, 32, P, 8, 32, None, 0, 0, 0,
                                         None) == 0


@pytest.mark.parametrize("args,expect", [
    # (batch, H, W, cin, cout, KH, KW, sh, sw, ph, pw, dh, dw, x, w, y, bias, epi, dtype)
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, P, P, P, None, 0, 9), dg.GEMM_ERR_UNSUPPORTED),
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, P, P, P, None, 0x100, 0), dg.GEMM_ERR_UNSUPPORTED),
    ((1, 8, 8, 4, 8, 3, 3, 0, 1, 1, 1, 1, 1, P, P, P, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),
    ((1, 2, 2, 4, 8, 5, 5, 1, 1, 0, 0, 1, 1, P, P, P, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, None, P, P, None, 0, 0), dg.GEMM_ERR_INVALID_ARG),
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, P, P, P, None, 1, 0), dg.GEMM_ERR_INVALID_ARG),
    ((1, 8, 8, 4, 12, 3, 3, 1, 1, 1, 1, 1, 1, P, P, P, None, 0, 0), dg.GEMM_ERR_MISALIGNED),
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, P + 2, P, P, None, 0, 0), dg.GEMM_ERR_MISALIGNED),
    ((1, 8, 8, 4, 8, 3, 3, 1, 1, 1, 1, 1, 1, P, P, P, None, 0, 4), dg.GEMM_ERR_UNSUPPORTED),
])
def test_conv_argument_errors(args, expect):
    assert dg.lib().conv2d_im2col(*args, None) == expect


def test_trace_setting_checks_alignment_and_turns_off():
    # no GPU needed: the call only records the buffer
    assert dg.gemm_set_trace(0x1003, 4096) == dg.GEMM_ERR_MISALIGNED
    assert dg.gemm_set_trace(None, 0) == dg.GEMM_OK
    assert dg.gemm_set_trace(0x1000, 8) == dg.GEMM_OK  # too small for one block: off
    assert dg.GEMM_TRACE_EVENTS == 8 and dg.GEMM_TRACE_EXIT == 7


# ------------------------------------------------ the sweep's rule writer

_TABLE = """// head
// BEGIN RULES (written by the sweep)
static const Rule kRules[] = {
    {64, 64, 64, 64, 64, 64, 0, 0, 1},  // sq64: cfgB 10 TFLOP/s
    {96, 96, 96, 96, 96, 96, 0, 0, 1},  // sq96 (sustained): cfgB 20 TFLOP/s
    {0, 0, 0, 0, 0, 0, -1, -1, -1},  // sentinel
};
// END RULES
// tail
"""


def _row(cls, n, times, sustained=False):
    best = min(times, key=times.get)
    ids = {"cfgA": 0, "cfgB": 1, "cfgC": 2}
    return {"class": cls, "M": n, "N": n, "K": n, "b_col": False, "grouped": False,
            "sustained": sustained, "times_ms": times, "best": best, "best_id": ids[best],
            "best_tflops": 0.0, "ids": ids}


def _rules(path):
    import re
    text = open(path).read()
    found = re.findall(r"^\s*\{(\d+), .*?, (-?\d+)\},  // ([^\n]+)$", text, flags=re.M)
    return [f for f in found if f[2] != "sentinel"], text


def test_sweep_rule_writer(tmp_path):
    from dense_gemm_16_b200 import sweep
    path = tmp_path / "table.h"
    path.write_text(_TABLE)
    sweep.write_rules([
        _row("sq64", 64, {"cfgA": 0.995, "cfgB": 1.0}),     # within the margin: keep cfgB
        _row("sq96", 96, {"cfgA": 0.5, "cfgB": 1.0}),       # burst sweep: keep the sustained rule
        _row("sq128", 128, {"cfgC": 0.5, "cfgB": 1.0}),     # new class
    ], path=str(path))
    rules, text = _rules(path)
    by_m = {int(m): (int(cid), note) for m, cid, note in rules}
    assert by_m[64][0] == 1 and "sq64: cfgB" in by_m[64][1]
    assert by_m[96] == (1, "sq96 (sustained): cfgB 20 TFLOP/s")
    assert by_m[128][0] == 2 and "sq128: cfgC" in by_m[128][1]
    assert text.startswith("// head") and text.rstrip().endswith("// tail")
    assert "sentinel" in text and len(rules) == 3
    # a clear win replaces the incumbent; a sustained sweep replaces a
    # sustained rule, once, with the tag kept
    sweep.write_rules([
        _row("sq64", 64, {"cfgA": 0.9, "cfgB": 1.0}),
        _row("sq96", 96, {"cfgC": 0.5, "cfgB": 1.0}, sustained=True),
    ], path=str(path))
    rules, _ = _rules(path)
    by_m = {int(m): (int(cid), note) for m, cid, note in rules}
    assert by_m[64][0] == 0 and "sq64: cfgA" in by_m[64][1]
    assert by_m[96][0] == 2 and by_m[96][1].startswith("sq96 (sustained): cfgC")
    assert len(rules) == 3

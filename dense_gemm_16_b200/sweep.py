"""Offline tile-config sweep: time every compiled config on each shape class
and write the winners into csrc/config_table.h.

The counterpart of the pages' compile-time parameter search ("用Triton跨芯片
优化GEMM" section 3.3; the crowd-sourced tuning page, sections 3.2 and 5.2):
enumerate the candidates (here: the configs compiled into the library, already
pruned by the shared-memory budget when they were instantiated), time each
with an L2 flush before every repetition, take the median of several batches,
keep the fastest, and record every candidate's time -- failures included --
in a log.

    python -m dense_gemm_16_b200.sweep [--write] [--log PATH] [--reps R] [--batches B]

Needs a GPU.  --write rewrites the RULES block of csrc/config_table.h; the
library must then be rebuilt.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
TABLE = os.path.join(HERE, "csrc", "config_table.h")

# Shape classes: (name, M, N, K, dtype, b_col, grouped, experts) -- the
# configurations of the path plus neighbours that bound each class.
CLASSES = [
    ("square256", 256, 256, 256, "f16", False),
    ("m1024n1024k2048", 1024, 1024, 2048, "f16", False),
    ("square2048", 2048, 2048, 2048, "f16", False),
    ("square4096", 4096, 4096, 4096, "bf16", False),
    ("square8192", 8192, 8192, 8192, "bf16", False),
    ("m1000n1000k2000_bcol", 1000, 1000, 2000, "f16", True),
    ("m4096n4096k512_bcol", 4096, 4096, 512, "f16", True),
    ("m16n8192k8192_bcol", 16, 8192, 8192, "f16", True),
]


def _time_config(dg, torch, cid, M, N, K, dtype, b_col, reps, batches, flush):
    lib = dg.lib()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    A = torch.randn(M, K, device="cuda", dtype=tdt)
    B = torch.randn(*((N, K) if b_col else (K, N)), device="cuda", dtype=tdt)
    C = torch.empty(M, N, device="cuda", dtype=tdt)
    code = dg.dtype_code(tdt)
    epi = dg.GEMM_B_COL_MAJOR if b_col else 0
    ldb = K if b_col else N
    stream = torch.cuda.current_stream().cuda_stream
    if lib.gemm_force_config(cid):
        return None, "bad id"
    try:
        def call():
            return lib.gemm(M, N, K, A.data_ptr(), K, B.data_ptr(), ldb, C.data_ptr(), N, None,
                            epi, code, stream)
        rc = call()
        if rc:
            return None, dg.gemm_status_string(rc)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        if dg.gemm_device_status():
            return None, "device status"
        meds = []
        for _ in range(batches):
            ts = []
            for _ in range(reps):
                flush.fill_(1)
                s = torch.cuda.Event(enable_timing=True)
                e = torch.cuda.Event(enable_timing=True)
                s.record()
                call()
                e.record()
                ts.append((s, e))
            torch.cuda.synchronize()
            meds.append(statistics.median(a.elapsed_time(b) for a, b in ts))
        return statistics.median(meds), ""
    finally:
        lib.gemm_force_config(-1)


def run(reps=20, batches=3, log=None):
    import torch

    import dense_gemm_16_b200 as dg
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device="cuda")
    names = [dg.gemm_config_name(i) for i in range(dg.gemm_num_configs())]
    results = []
    for cname, M, N, K, dtype, b_col in CLASSES:
        row = {"class": cname, "M": M, "N": N, "K": K, "dtype": dtype, "b_col": b_col,
               "times_ms": {}, "errors": {}}
        for cid, name in enumerate(names):
            if name.startswith("swap") and not b_col:
                row["errors"][name] = "needs column-major B"
                continue
            t, err = _time_config(dg, torch, cid, M, N, K, dtype, b_col, reps, batches, flush)
            if t is None:
                row["errors"][name] = err
            else:
                row["times_ms"][name] = t
        best = min(row["times_ms"], key=row["times_ms"].get)
        row["best"] = best
        row["best_id"] = names.index(best)
        row["best_tflops"] = 2.0 * M * N * K / (row["times_ms"][best] * 1e-3) / 1e12
        results.append(row)
        print(json.dumps(row), flush=True)
    if log:
        with open(log, "w") as f:
            for r in results:
                f.write(json.dumps(r) + "\n")
    return results


def write_rules(results, path=TABLE):
    """Rewrite the RULES block: one exact-shape rule per class (dense)."""
    lines = ["static const Rule kRules[] = {"]
    for r in results:
        lines.append(
            f"    {{{r['M']}, {r['M']}, {r['N']}, {r['N']}, {r['K']}, {r['K']}, "
            f"{int(r['b_col'])}, 0, {r['best_id']}}},  // {r['class']}: {r['best']} "
            f"{r['best_tflops']:.0f} TFLOP/s")
    lines.append("    {0, 0, 0, 0, 0, 0, -1, -1, -1},  // sentinel")
    lines.append("};")
    text = open(path).read()
    new = re.sub(r"(// BEGIN RULES \(written by the sweep\)\n).*?(// END RULES)",
                 lambda m: m.group(1) + "\n".join(lines) + "\n" + m.group(2), text, flags=re.S)
    with open(path, "w") as f:
        f.write(new)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--batches", type=int, default=3)
    ap.add_argument("--log", default=None)
    ap.add_argument("--write", action="store_true")
    a = ap.parse_args(argv)
    sys.path.insert(0, ROOT)
    res = run(a.reps, a.batches, a.log)
    if a.write:
        write_rules(res)


if __name__ == "__main__":
    main()

"""Offline tile-config sweep: time every compiled config on each shape class
and write the winners into csrc/config_table.h.

The counterpart of the pages' compile-time parameter search ("用Triton跨芯片
优化GEMM" section 3.3; the crowd-sourced tuning page, sections 3.2 and 5.2):
enumerate the candidates (here: the configs compiled into the library, already
pruned by the shared-memory budget when they were instantiated), time each
with an L2 flush before every repetition, interleaving the candidates in
several rounds so that clock and temperature drift hit them alike, take the
median,
keep the fastest, and record every candidate's time -- failures included --
in a log.

    python -m dense_gemm_16_b200.sweep [--write] [--log PATH] [--reps R] [--rounds N]
                                      [--only CLASS ...]

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


def _bench_rounds(dg, torch, calls, reps, rounds, flush):
    """Time every candidate in `calls` ({config id: launch fn}) `rounds` times,
    interleaved (so clock and thermal drift hit all candidates alike): each
    round runs `reps` launches per candidate, L2 flushed before each, and
    keeps the median; the result per candidate is the median over rounds."""
    lib = dg.lib()
    per = {cid: [] for cid in calls}
    errors = {}
    for cid, call in list(calls.items()):  # one checked launch each
        lib.gemm_force_config(cid)
        try:
            rc = call()
            torch.cuda.synchronize()
            st = dg.gemm_device_status()
        finally:
            lib.gemm_force_config(-1)
        if rc or st:
            errors[cid] = dg.gemm_status_string(rc or st)
            del calls[cid]
    for _ in range(rounds):
        for cid, call in calls.items():
            lib.gemm_force_config(cid)
            try:
                ts = []
                for _ in range(reps):
                    if flush is not None:
                        flush.fill_(1)
                    s = torch.cuda.Event(enable_timing=True)
                    e = torch.cuda.Event(enable_timing=True)
                    s.record()
                    call()
                    e.record()
                    ts.append((s, e))
                torch.cuda.synchronize()
            finally:
                lib.gemm_force_config(-1)
            per[cid].append(statistics.median(a.elapsed_time(b) for a, b in ts))
    return {cid: statistics.median(v) for cid, v in per.items() if v}, errors


def _dense_calls(dg, torch, names, M, N, K, dtype, b_col):
    lib = dg.lib()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    A = torch.randn(M, K, device="cuda", dtype=tdt)
    B = torch.randn(*((N, K) if b_col else (K, N)), device="cuda", dtype=tdt)
    C = torch.empty(M, N, device="cuda", dtype=tdt)
    code = dg.dtype_code(tdt)
    epi = dg.GEMM_B_COL_MAJOR if b_col else 0
    ldb = K if b_col else N
    stream = torch.cuda.current_stream().cuda_stream
    keep = (A, B, C)

    def make():
        return lambda: lib.gemm(M, N, K, keep[0].data_ptr(), K, keep[1].data_ptr(), ldb,
                                keep[2].data_ptr(), N, None, epi, code, stream)
    calls, skipped = {}, {}
    for cid, name in enumerate(names):
        if name.startswith("swap") and not b_col:
            skipped[cid] = "needs column-major B"
        elif name.startswith("gswap"):
            skipped[cid] = "grouped only"
        else:
            calls[cid] = make()
    return calls, skipped, keep


# Grouped classes: (name, experts, total rows, N, K, dtype) with the seeded
# Dirichlet/multinomial routing of the MoE workload.
GROUPED_CLASSES = [
    ("moe32_n1408_k4096", 32, 8192, 1408, 4096, "bf16"),
    ("moe8_n4096_k4096", 8, 16384, 4096, 4096, "bf16"),
    ("moe64_n768_k2048", 64, 8192, 768, 2048, "bf16"),
]


def _grouped_calls(dg, torch, names, E, R, N, K, dtype):
    import workloads
    lib = dg.lib()
    rows = workloads.moe_group_rows(E, R, 11)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    X = torch.randn(R, K, device="cuda", dtype=tdt)
    W = torch.randn(E, K, N, device="cuda", dtype=tdt) * 0.02
    Y = torch.empty(R, N, device="cuda", dtype=tdt)
    drows = torch.from_numpy(rows).cuda()
    code = dg.dtype_code(tdt)
    stream = torch.cuda.current_stream().cuda_stream
    keep = (X, W, Y, drows)

    def call():
        return lib.grouped_gemm(E, keep[3].data_ptr(), R, N, K, keep[0].data_ptr(), K,
                                keep[1].data_ptr(), N, K * N, keep[2].data_ptr(), N, None,
                                dg.GEMM_EPI_RELU, code, stream)
    calls, skipped = {}, {}
    for cid, name in enumerate(names):
        if name.startswith(("swap", "csk", "pair_256x128")) or "_k" in name:
            skipped[cid] = "not a grouped kernel (or split-K, which grouped ignores)"
        elif name.startswith("pair") and name.endswith(("_sk", "_hy")):
            skipped[cid] = "grouped CTA pairs run whole tiles (the same kernel as without _sk/_hy)"
        else:
            calls[cid] = call
    return calls, skipped, keep


def run(reps=10, rounds=5, log=None, only=None, sustained=False):
    """sustained=True: launches back to back without the L2 flush, the regime
    of a long run under the power cap (use inputs larger than L2)."""
    import torch

    import dense_gemm_16_b200 as dg
    flush = None if sustained else torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32,
                                               device="cuda")
    names = [dg.gemm_config_name(i) for i in range(dg.gemm_num_configs())]
    results = []
    jobs = [(c[0], False, c) for c in CLASSES] + [(c[0], True, c) for c in GROUPED_CLASSES]
    for cname, grouped, spec in jobs:
        if only and cname not in only:
            continue
        if grouped:
            _, E, R, N, K, dtype = spec
            M, b_col = R, False
            calls, skipped, keep = _grouped_calls(dg, torch, names, E, R, N, K, dtype)
        else:
            _, M, N, K, dtype, b_col = spec
            calls, skipped, keep = _dense_calls(dg, torch, names, M, N, K, dtype, b_col)
        times, errors = _bench_rounds(dg, torch, calls, reps, rounds, flush)
        errors.update(skipped)
        row = {"class": cname, "M": M, "N": N, "K": K, "dtype": dtype, "b_col": b_col,
               "grouped": grouped, "sustained": sustained,
               "times_ms": {names[c]: t for c, t in times.items()},
               "errors": {names[c]: e for c, e in errors.items()}}
        best = min(times, key=times.get)
        row["best"] = names[best]
        row["best_id"] = best
        row["ids"] = {names[c]: c for c in times}
        row["best_tflops"] = 2.0 * M * N * K / (times[best] * 1e-3) / 1e12
        results.append(row)
        print(json.dumps(row), flush=True)
        del keep
    if log:
        with open(log, "w") as f:
            for r in results:
                f.write(json.dumps(r) + "\n")
    return results


# A new winner replaces the incumbent of a class only if it is faster by more
# than this fraction in the same sweep (run-to-run noise is about 1%).
KEEP_MARGIN = 0.01


def _rule_line(r, cid, name):
    t = r["times_ms"][name]
    tflops = 2.0 * r["M"] * r["N"] * r["K"] / (t * 1e-3) / 1e12
    tag = " (sustained)" if r.get("sustained") else ""
    return (f"    {{{r['M']}, {r['M']}, {r['N']}, {r['N']}, {r['K']}, {r['K']}, "
            f"{int(r['b_col'])}, {int(r.get('grouped', False))}, {cid}}},  "
            f"// {r['class']}{tag}: {name} {tflops:.0f} TFLOP/s")


def write_rules(results, path=TABLE):
    """Rewrite the RULES block: one exact-shape rule per swept class.  Rules
    of classes not in `results` are kept as they are; so is a class's rule
    when its config is within KEEP_MARGIN of the sweep's best, and a rule
    chosen under sustained load when the new sweep was not (a burst sweep
    does not overrule it)."""
    text = open(path).read()
    m = re.search(r"// BEGIN RULES \(written by the sweep\)\n(.*?)// END RULES", text, flags=re.S)
    old = {}  # class -> (line, config name, sustained)
    for line in m.group(1).splitlines():
        c = re.search(r"//\s*([^:(]+?)\s*(\(sustained\))?:\s*(\S+)", line)
        if c and line.strip().startswith("{"):
            old[c.group(1)] = (line, c.group(3), c.group(2) is not None)
    new = {}
    for r in results:
        best_name, best_id = r["best"], r["best_id"]
        inc = old.get(r["class"])
        if inc is not None:
            _, inc_name, inc_sustained = inc
            if inc_sustained and not r.get("sustained"):
                continue  # keep the rule measured under sustained load
            if inc_name in r["times_ms"] and \
                    r["times_ms"][best_name] >= (1.0 - KEEP_MARGIN) * r["times_ms"][inc_name]:
                best_name = inc_name
                best_id = _config_id(inc_name, r, best_id)
        new[r["class"]] = _rule_line(r, best_id, best_name)
    merged = {k: v[0] for k, v in old.items()}
    merged.update(new)
    lines = ["static const Rule kRules[] = {"] + list(merged.values())
    lines.append("    {0, 0, 0, 0, 0, 0, -1, -1, -1},  // sentinel")
    lines.append("};")
    out = re.sub(r"(// BEGIN RULES \(written by the sweep\)\n).*?(// END RULES)",
                 lambda mm: mm.group(1) + "\n".join(lines) + "\n" + mm.group(2), text, flags=re.S)
    with open(path, "w") as f:
        f.write(out)


def _config_id(name, row, fallback):
    """The config id of `name`: from the row's id map when the sweep recorded
    one, else from the compiled table's names in config_table.h."""
    ids = row.get("ids")
    if ids and name in ids:
        return ids[name]
    names = re.findall(r'^\s*\{"([^"]+)",', open(TABLE).read(), flags=re.M)
    return names.index(name) if name in names else fallback


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--rounds", type=int, default=5)
    ap.add_argument("--log", default=None)
    ap.add_argument("--only", nargs="*", default=None, help="class names to sweep")
    ap.add_argument("--sustained", action="store_true",
                    help="back-to-back launches, no L2 flush")
    ap.add_argument("--write", action="store_true")
    ap.add_argument("--from-log", default=None,
                    help="write the rules from a saved --log file instead of sweeping")
    a = ap.parse_args(argv)
    sys.path.insert(0, ROOT)
    if a.from_log:
        with open(a.from_log) as f:
            write_rules([json.loads(line) for line in f if line.strip()])
        return
    res = run(a.reps, a.rounds, a.log, a.only, a.sustained)
    if a.write:
        write_rules(res)


if __name__ == "__main__":
    main()

"""Benchmark of the tiled GEMM hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one gemm() call through the C ABI on one batch of synthetic,
device-resident inputs: all stages of the path (argument checks and tensor
maps on the host; TMA ring, tcgen05 MMA into TMEM, fused epilogue and store on
the device) run inside it.  The default workload is the large square bf16
GEMM M = N = K = 8192 on which the dense-tensor-peak target is stated; its
operands (A + B = 256 MiB) are larger than the 126 MB L2, so no flush is
needed between steps (smaller workloads flush L2 by writing a 256 MiB
buffer between steps, outside the timed events).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; a barrier and a device synchronise on both sides
of the timed region; the max over ranks.  `value` = all ranks' FLOPs / that
time (TFLOP/s).  With N > 1 each rank runs an independent replica of the
workload (the path has no collective); scaling is weak.

`e2e` repeats the step with the inputs copied from pinned host memory and
the output copied back inside the timed region.  `roofline` compares the
GEMM kernel's average launch time with the measured dense bf16 tensor peak
(MEASURED_PEAKS.json, else the machine's fallback figure).  `cpu_baseline` times
the fp64 CPU oracle on a bounded sample of the same workload's outputs.
`--impl reference` times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GEMM TFLOP/s (fp32 acc) and % of B200 dense fp16/bf16 tensor peak, 1 GPU"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "square8192_bf16"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}


# ------------------------------------------------------------------ helpers

def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Sources every launch depends on (host path, shared device code, the table).
_COMMON_SOURCES = ("ptx.cuh", "kernel_common.cuh", "raster.h", "dispatch.h", "config_table.h",
                   "gemm_api.cu")


def _source_sha(files=None) -> str:
    """Hash of the named csrc files (all of them when None)."""
    csrc = os.path.join(ROOT, "dense_gemm_16_b200", "csrc")
    names = sorted(files) if files else sorted(os.listdir(csrc))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on this workload with the same sources of the kernel that runs it (the
    entry lists them: the common files plus that kernel's own); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get(workload)
    if not entry or entry.get("source_sha") != _source_sha(entry.get("sources")):
        return None
    return entry.get("dram_bytes_per_launch")


def _workload_config(w, world: int) -> dict:
    """The workload part of a bench line's `config`, the same for both arms
    (our arm adds its L2 regime and the config the table chose)."""
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "in_dtype": w.dtype,
            "acc_dtype": "f32", "out_dtype": w.out_dtype,
            "b_layout": "col-major" if w.b_colmajor else "row-major",
            "epilogue": ("bias+" if w.bias else "") + ("relu" if w.relu else "none"),
            "experts": w.experts or None, "parallelism": f"replicas x{world}"}


def _roofline(flops: float, alg_bytes: float, ms_per_step: float, total_ms: float,
              back_to_back: bool, dtype: str, peaks=None) -> dict:
    """The roofline object of one bench line (traffic is added by the caller).

    The bound is the slower of FLOPs at the dense tensor peak and the
    algorithmic bytes at the HBM copy bandwidth.  Back-to-back launches for
    half a second or more run under the power cap, so their tensor peak is
    the sustained cuBLAS figure; otherwise the burst figure."""
    peaks, peak_src = peaks if peaks is not None else _peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = back_to_back and total_ms >= 500.0
    peak = float(peaks.get("bf16_tflops_sustained", burst)) if sustained else burst
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    t_tensor = flops / (peak * 1e12)
    t_hbm = alg_bytes / (hbm * 1e9)
    if t_hbm > t_tensor:
        gbs = alg_bytes / (ms_per_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "peak_source": f"{peak_src} HBM copy bandwidth"}
    else:
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16 dense "
                + ("(sustained: back-to-back launches under the power cap)" if sustained
                   else "(burst)")
                + ("; fp16 has the same dense rate" if dtype == "f16" else ""),
                "frac_of_burst": round(achieved / burst, 4)}
    roof["bound_times_us"] = {"tensor": round(t_tensor * 1e6, 2), "hbm": round(t_hbm * 1e6, 2)}
    return roof


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self._t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def _max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------- oracle timing

def time_oracle(w, budget_s: float = 12.0, threads: int | None = None):
    """Time the CPU oracle on a bounded sample of the workload's outputs.
    Returns (tflops, seconds, n_elements, threads_used)."""
    import numpy as np

    import oracle
    import workloads
    threads = threads or os.cpu_count() or 1
    used = oracle.threads_used(threads)
    if w.grouped:
        X, W, rows, _ = workloads.make_grouped_inputs(w)
        total = int(rows.sum())

        def run(n):
            r, c = workloads.sample_indices(total, w.N, n=n, seed=4321)
            r, c = r[:n], c[:n]
            t0 = time.perf_counter()
            oracle.grouped_gemm_at(rows, w.N, w.K, X, w.K, W, w.N, w.K * w.N, r, c,
                                   relu=w.relu, dtype=w.dtype, threads=threads)
            return time.perf_counter() - t0
    else:
        A, B, bias = workloads.make_inputs(w)
        ldb = w.K if w.b_colmajor else w.N

        def run(n):
            r, c = workloads.sample_indices(w.M, w.N, n=n, seed=4321)
            r, c = r[:n], c[:n]
            t0 = time.perf_counter()
            oracle.gemm_at(w.M, w.N, w.K, A, w.K, B, ldb, r, c, b_colmajor=w.b_colmajor,
                           bias=bias, relu=w.relu, dtype=w.dtype, threads=threads)
            return time.perf_counter() - t0
    # calibrate on a sample large enough that per-call overheads do not
    # inflate the per-element estimate, then size the timed sample to the budget
    n = max(used * 64, 4096)
    dt = run(n)
    n = int(min(max(n, n * budget_s / max(dt, 1e-3)), 4_000_000))
    dt = run(n)
    return 2.0 * w.K * n / dt / 1e12, dt, n, used


# --------------------------------------------------------------- our arm

def bench_ours(args, rank, local, world):
    import torch

    import dense_gemm_16_b200 as dg
    import workloads

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    stream = torch.cuda.current_stream(dev)
    lib = dg.lib()
    if args.config >= 0 and lib.gemm_force_config(args.config):
        raise SystemExit(f"unknown config id {args.config}")

    if w.grouped:
        X, W, rows, bias = workloads.make_grouped_inputs(w)
        total = int(rows.sum())
        host = [X.pin_memory(), W.pin_memory(), torch.from_numpy(rows).pin_memory()]
        dev_in = [h.to(dev) for h in host]
        out = torch.empty(total, w.N, dtype=X.dtype, device=dev)
        out_host = torch.empty(total, w.N, dtype=X.dtype).pin_memory()
        epi = dg.GEMM_EPI_RELU if w.relu else 0
        code = dg.dtype_code(X.dtype)

        def step(ins, o):
            rc = lib.grouped_gemm(w.experts, ins[2].data_ptr(), total, w.N, w.K, ins[0].data_ptr(),
                                  w.K, ins[1].data_ptr(), w.N, w.K * w.N, o.data_ptr(), w.N, None,
                                  epi, code, stream.cuda_stream)
            if rc:
                raise dg.GemmError(rc, "grouped_gemm")
        flops = 2.0 * total * w.N * w.K
        in_bytes = X.numel() * 2 + sum(int(r) > 0 for r in rows) * w.K * w.N * 2
        out_bytes = total * w.N * 2
    else:
        A, B, bias = workloads.make_inputs(w)
        host = [A.pin_memory(), B.pin_memory()] + ([bias.pin_memory()] if bias is not None else [])
        dev_in = [h.to(dev) for h in host]
        out = torch.empty(w.M, w.N, dtype=A.dtype, device=dev)
        out_host = torch.empty(w.M, w.N, dtype=A.dtype).pin_memory()
        epi = (dg.GEMM_EPI_BIAS if bias is not None else 0) | (dg.GEMM_EPI_RELU if w.relu else 0) | \
            (dg.GEMM_B_COL_MAJOR if w.b_colmajor else 0)
        code = dg.dtype_code(A.dtype)
        ldb = w.K if w.b_colmajor else w.N

        def step(ins, o):
            rc = lib.gemm(w.M, w.N, w.K, ins[0].data_ptr(), w.K, ins[1].data_ptr(), ldb,
                          o.data_ptr(), w.N, ins[2].data_ptr() if len(ins) > 2 else None, epi,
                          code, stream.cuda_stream)
            if rc:
                raise dg.GemmError(rc)
        flops = w.flops()
        in_bytes = (w.M * w.K + w.K * w.N + (w.N if bias is not None else 0)) * 2
        out_bytes = w.M * w.N * 2

    h2d_bytes = sum(h.numel() * h.element_size() for h in host)
    d2h_bytes = out_host.numel() * out_host.element_size()
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)

    # warm-up (also loads the kernels and fills the library's caches)
    for _ in range(args.warmup):
        step(dev_in, out)
    torch.cuda.synchronize(dev)
    status = dg.gemm_device_status(stream)
    if status:
        raise dg.GemmError(status, "warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    _barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i)
            starts[i].record(stream)
            step(dev_in, out)
            stops[i].record(stream)
        torch.cuda.synchronize(dev)
        _barrier(world, dev)
    per = [s.elapsed_time(e) for s, e in zip(starts, stops)]
    status = dg.gemm_device_status(stream)
    if status:
        raise dg.GemmError(status, "timed region")
    total_ms = sum(per)
    total_ms = _max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = flops * args.steps * world / (total_ms * 1e-3) / 1e12

    # end to end: every step copies its inputs from pinned host memory, runs
    # the GEMM and copies its result back to pinned host memory, all inside
    # the timed region.  Two buffer sets and three streams let step i+1's
    # upload overlap step i's GEMM and download (PCIe is full duplex); the
    # order between them is kept with events.
    e2e_steps = max(3, min(args.steps, 20))
    e_start = torch.cuda.Event(enable_timing=True)
    e_stop = torch.cuda.Event(enable_timing=True)
    h2d_s = torch.cuda.Stream(dev)
    d2h_s = torch.cuda.Stream(dev)
    ins = [[torch.empty_like(d) for d in dev_in] for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    hosts_out = [out_host, torch.empty_like(out_host).pin_memory()]

    def run_e2e(n):
        up = [torch.cuda.Event() for _ in range(2)]    # buffer b's inputs landed
        done = [torch.cuda.Event() for _ in range(2)]  # the GEMM on buffer b finished
        down = [torch.cuda.Event() for _ in range(2)]  # buffer b's result is on the host
        used = [False, False]
        h2d_s.wait_stream(stream)
        d2h_s.wait_stream(stream)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(h2d_s):
                if used[b]:
                    h2d_s.wait_event(done[b])  # the last GEMM that read buffer b
                for h, d in zip(host, ins[b]):
                    d.copy_(h, non_blocking=True)
                up[b].record(h2d_s)
            stream.wait_event(up[b])
            if used[b]:
                stream.wait_event(down[b])  # buffer b's last result has left
            step(ins[b], outs[b])
            done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(done[b])
                hosts_out[b].copy_(outs[b], non_blocking=True)
                down[b].record(d2h_s)
            used[b] = True
        for b in range(2):
            if used[b]:
                stream.wait_event(down[b])

    run_e2e(2)
    torch.cuda.synchronize(dev)
    _barrier(world, dev)
    e_start.record(stream)
    run_e2e(e2e_steps)
    e_stop.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = _max_over_ranks(e_start.elapsed_time(e_stop), world, dev)
    e2e_value = flops * e2e_steps * world / (e2e_ms * 1e-3) / 1e12

    roof = _roofline(flops, in_bytes + out_bytes, ms_per_step, total_ms, flush is None,
                     w.dtype)
    alg_bytes = in_bytes + out_bytes
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    burst = float(_peaks()[0].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    roof["traffic"] = _traffic(w.name)
    roof["algorithmic_bytes"] = alg_bytes
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f16", "data": "synthetic",
        "config": dict(
            _workload_config(w, world),
            l2="flushed between steps (256 MiB write)" if flush is not None
            else f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB)",
            config_id=lib.gemm_select_config(w.M, w.N, w.K, code, epi) if not w.grouped
            else None),
        "pct_of_peak": round(100.0 * achieved / burst, 2),
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, n, used = time_oracle(w)
        result["cpu_baseline"] = {
            "value": tf, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{n} sampled output elements of {w.name} (K={w.K} fp64 MACs each), "
                      f"{secs:.1f} s"}
    return result


# ---------------------------------------------------------- reference arm

def bench_reference(args, rank, world):
    """The CPU oracle as the reference arm (rank 0 only)."""
    import workloads
    w = workloads.get(args.workload)
    if rank != 0:
        return None
    per_step_budget = max(0.02, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    # size one step's sample to the per-step budget
    tf, secs, n, used = time_oracle(w, budget_s=per_step_budget)
    import numpy as np

    import oracle
    times = []
    if w.grouped:
        X, W, rows, _ = workloads.make_grouped_inputs(w)
        total = int(rows.sum())
        r, c = workloads.sample_indices(total, w.N, n=n, seed=4321)
        call = lambda: oracle.grouped_gemm_at(rows, w.N, w.K, X, w.K, W, w.N, w.K * w.N,
                                              r[:n], c[:n], relu=w.relu, dtype=w.dtype,
                                              threads=used)
    else:
        A, B, bias = workloads.make_inputs(w)
        ldb = w.K if w.b_colmajor else w.N
        r, c = workloads.sample_indices(w.M, w.N, n=n, seed=4321)
        call = lambda: oracle.gemm_at(w.M, w.N, w.K, A, w.K, B, ldb, r[:n], c[:n],
                                      b_colmajor=w.b_colmajor, bias=bias, relu=w.relu,
                                      dtype=w.dtype, threads=used)
    for _ in range(args.warmup):
        call()
    for _ in range(args.steps):
        t0 = time.perf_counter()
        call()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = 2.0 * w.K * n * args.steps / total / 1e12
    sample = f"{n} sampled output elements of {w.name} per step (K={w.K} fp64 MACs each)"
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _workload_config(w, world),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--config", type=int, default=-1,
                    help="force a tile config id (default: the library's table)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (for quick runs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, local, world = _dist_init(args)
    try:
        if args.impl == "reference":
            res = bench_reference(args, rank, world)
        else:
            res = bench_ours(args, rank, local, world)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

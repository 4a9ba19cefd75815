#!/usr/bin/env python
"""Benchmark of the FP8 block-scaled NT GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference] [--workload prefill|decode64|decode128]

One step = one pass of the hot path over the workload: for each (N, K) shape of the workload,
the per-token FP8 cast of the bf16 activations A [M,K] (1x128 scales, MN-major layout) and the
GEMM D = C + A·Bᵀ with 128x128-block-scaled e4m3 weights. The weights are cast once, before the
timed region (offline, as in inference); that cast is timed on its own and reported under
"weight_cast". Inputs are the seeded synthetic recipe of moe_grouped_gemm_sm_b200.synth:
A, B ~ N(0,1) and C ~ N(0,0.1) in bf16.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device synchronise,
timed with CUDA events on the launching stream; the max over ranks is reported. The working set
of one step (activations, weights, C and D of six shapes) is far larger than the 126 MB L2, so
no explicit flush is needed between steps. Per-kernel durations come from CUDA events recorded
around every launch inside the timed region. SM clocks and throttle reasons are sampled through
NVML during the timed region.

Multi-GPU: the path has no exchange step, so N GPUs run N independent replicas (one process per
GPU under torchrun), each on the full workload ("scaling": "weak"); value = all ranks' FLOPs
divided by the slowest rank's time.

--impl reference times the oracle (plain C, fp64; oracle/) on the host cores on a bounded sample
of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PREFILL_SHAPES = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]
WORKLOADS = {
    "prefill": dict(M=4096, shapes=PREFILL_SHAPES, with_c=True,
                    desc="dense FP8 NT GEMM, M=4096, (N,K) in the six DeepSeek-V3 prefill shapes, C bf16"),
    "decode64": dict(M=64, shapes=PREFILL_SHAPES, with_c=True,
                     desc="dense FP8 NT GEMM, M=64 decode, six (N,K) shapes, C bf16"),
    "decode128": dict(M=128, shapes=PREFILL_SHAPES, with_c=True,
                      desc="dense FP8 NT GEMM, M=128 decode, six (N,K) shapes, C bf16"),
}
METRIC = "FP8 block-scaled GEMM TFLOPS on 1×B200; % of FP8 peak / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


# ------------------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas only)
# ------------------------------------------------------------------------------------------------

def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(backend: str):
    import datetime

    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return dist


def reduce_max(value: float, device=None) -> float:
    """Max over ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(local_ms: float, local_flops: float, device=None):
    """Whole-job numbers: (slowest rank's ms, total FLOPs of all ranks)."""
    return reduce_max(local_ms, device), reduce_sum(local_flops, device)


# ------------------------------------------------------------------------------------------------
# peaks, clocks
# ------------------------------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a background thread."""

    def __init__(self, index: int, period_s: float = 0.02):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= int(get(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        reasons = [name for bit, name in NVML_REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------------
# workload
# ------------------------------------------------------------------------------------------------

def algorithmic_bytes(M, N, K, with_c):
    """HBM bytes one GEMM launch must move at minimum: e4m3 A and B, fp32 scales, C and D."""
    kb, nb = K // 128, (N + 127) // 128
    return M * K + N * K + 4 * (M * kb + nb * kb) + 2 * M * N + (2 * M * N if with_c else 0)


def cast_bytes(M, K):
    """Per-token cast: 2 B read and 1 B written per element, one fp32 scale per 128 elements."""
    return 3 * M * K + 4 * M * (K // 128)


def make_inputs(wl):
    from moe_grouped_gemm_sm_b200 import synth
    out = []
    for i, (N, K) in enumerate(wl["shapes"]):
        x, w, c = synth.dense_inputs(wl["M"], N, K, wl["with_c"], salt=100 + i)
        out.append((N, K, x, w, c))
    return out


# ------------------------------------------------------------------------------------------------
# CUDA arm
# ------------------------------------------------------------------------------------------------

def run_cuda(args):
    import numpy as np
    import torch

    from moe_grouped_gemm_sm_b200 import _lib, ops
    from moe_grouped_gemm_sm_b200 import build as _build

    rank, local_rank, world = rank_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist_init("nccl")
    _build.build()
    _lib.load()
    wl = WORKLOADS[args.workload]
    M, with_c = wl["M"], wl["with_c"]
    stream = torch.cuda.current_stream(device)
    sptr = stream.cuda_stream

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).to(device)

    host = make_inputs(wl)
    problems = []
    wc_ms = []
    for (N, K, x, w, c) in host:
        w_dev = to_dev(w)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ops.cast_per_block(w_dev)                             # warm the weight cast once
        e0.record(stream)
        b, sfb = ops.cast_per_block(w_dev)
        e1.record(stream)
        torch.cuda.synchronize(device)
        wc_ms.append((e0.elapsed_time(e1), 3 * N * K + 4 * ((N + 127) // 128) * (K // 128)))
        del w_dev
        a_bf16 = to_dev(x)
        cc = to_dev(c) if c is not None else None
        a_q = torch.empty((M, K), dtype=torch.uint8, device=device)
        sfa = torch.empty((K // 128, (M + 3) // 4 * 4), dtype=torch.float32, device=device)
        d = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        problems.append(dict(N=N, K=K, a=a_bf16, c=cc, aq=a_q, sfa=sfa, b=b, sfb=sfb, d=d))
    torch.cuda.synchronize(device)

    L = _lib.load()

    def launch_cast(p):
        rc = L.dg_cast_fp8_per_token(p["a"].data_ptr(), p["aq"].data_ptr(), p["sfa"].data_ptr(), 1, M, p["K"], sptr)
        if rc:
            raise _lib.DgError("dg_cast_fp8_per_token", rc)

    def launch_gemm(p):
        rc = L.dg_fp8_gemm_nt(p["aq"].data_ptr(), p["sfa"].data_ptr(), p["b"].data_ptr(), p["sfb"].data_ptr(),
                              p["c"].data_ptr() if p["c"] is not None else None, p["d"].data_ptr(), M, p["N"],
                              p["K"], sptr)
        if rc:
            raise _lib.DgError("dg_fp8_gemm_nt", rc)

    def step(evs=None):
        for i, p in enumerate(problems):
            if evs is not None:
                evs[2 * i].record(stream)
            launch_cast(p)
            if evs is not None:
                evs[2 * i + 1].record(stream)
            launch_gemm(p)
        if evs is not None:
            evs[2 * len(problems)].record(stream)

    flops_step = sum(2.0 * M * p["N"] * p["K"] for p in problems)
    launches_per_step = 2 * len(problems)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if _lib.dg_get_device_error(sptr) != 0:
        raise RuntimeError("device error word set during warm-up")

    nev = 2 * len(problems) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    local_ms = start.elapsed_time(end) / args.steps
    if _lib.dg_get_device_error(sptr) != 0:
        raise RuntimeError("device error word set during the timed region")

    # per-kernel averages over the timed steps
    cast_ms = [statistics.fmean(evs[s][2 * i].elapsed_time(evs[s][2 * i + 1]) for s in range(args.steps))
               for i in range(len(problems))]
    gemm_ms = [statistics.fmean(evs[s][2 * i + 1].elapsed_time(evs[s][2 * i + 2]) for s in range(args.steps))
               for i in range(len(problems))]

    ms_max, flops_all = aggregate(local_ms, flops_step, device)
    value = flops_all / (ms_max * 1e-3) / 1e12

    # ---------------- e2e through the public API with pinned host buffers ----------------
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    host_bufs = []
    for (N, K, x, w, c), p in zip(host, problems):
        ah = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
        ch = torch.from_numpy(np.ascontiguousarray(c).view(np.int16)).view(torch.bfloat16).pin_memory() \
            if c is not None else None
        dh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        host_bufs.append((ah, ch, dh))
    h2d = sum(ah.numel() * 2 + (ch.numel() * 2 if ch is not None else 0) for ah, ch, _ in host_bufs)
    d2h = sum(dh.numel() * 2 for _, _, dh in host_bufs)

    def e2e_step():
        for (ah, ch, dh), p in zip(host_bufs, problems):
            p["a"].copy_(ah, non_blocking=True)
            if ch is not None:
                p["c"].copy_(ch, non_blocking=True)
            a_q, sfa = ops.cast_per_token(p["a"], stream=stream)
            d = ops.fp8_gemm_nt(a_q, sfa, p["b"], p["sfb"], p["c"], out=p["d"], stream=stream)
            dh.copy_(d, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(device)
    barrier(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, device)
    e2e_value = flops_all / (e2e_ms * 1e-3) / 1e12

    # ---------------- roofline of the dominant kernel (the GEMM) ----------------
    peaks, peaks_src = load_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]            # fp8 dense = 2x bf16 (nominal ratio)
    fp8_peak_burst = 2.0 * peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    gemm_total_ms = sum(gemm_ms)
    achieved = sum(2.0 * M * p["N"] * p["K"] for p in problems) / (gemm_total_ms * 1e-3) / 1e12
    per_shape = []
    for p, gm, cm in zip(problems, gemm_ms, cast_ms):
        fl = 2.0 * M * p["N"] * p["K"]
        by = algorithmic_bytes(M, p["N"], p["K"], with_c)
        t_tc = fl / (fp8_peak * 1e12)
        t_hbm = by / (hbm * 1e9)
        per_shape.append({"N": p["N"], "K": p["K"], "gemm_us": round(gm * 1e3, 2),
                          "tflops": round(fl / (gm * 1e-3) / 1e12, 1), "gbs": round(by / (gm * 1e-3) / 1e9, 1),
                          "bound": "tensor" if t_tc >= t_hbm else "hbm",
                          "roof_frac": round(max(t_tc, t_hbm) / (gm * 1e-3), 3),
                          "cast_us": round(cm * 1e3, 2),
                          "cast_gbs": round(cast_bytes(M, p["K"]) / (cm * 1e-3) / 1e9, 1)})
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            traffic = json.load(f).get(args.workload)

    clocks = clk.summary()
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": wl["desc"], "M": M, "shapes_NK": [list(s) for s in wl["shapes"]],
                   "step": "per-token cast of A + GEMM D=C+A·Bᵀ per shape; weights cast offline",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "no flush: one step's working set is far above the 126 MB L2"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4), "traffic": traffic,
                     "kernel": "gemm_normal_kernel (6 shapes, aggregate)",
                     "peak_source": f"{peaks_src}: 2 x bf16_tflops_sustained (fp8 = 2x bf16 nominal ratio)",
                     "frac_of_burst_peak": round(achieved / fp8_peak_burst, 4)},
        "per_shape": per_shape,
        "weight_cast": {"gbs": round(sum(b for _, b in wc_ms) / (sum(t for t, _ in wc_ms) * 1e-3) / 1e9, 1),
                        "ms_total": round(sum(t for t, _ in wc_ms), 3)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "path": "pinned host A,C -> device, ops.cast_per_token + ops.fp8_gemm_nt, D -> pinned host"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, host, target_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------------------------
# oracle (CPU) arm and baseline
# ------------------------------------------------------------------------------------------------

def oracle_sample(wl, host, rows: int, cols: int):
    """Times the oracle on `rows` rows x `cols` columns of every shape (cast of those rows of A
    plus the GEMM); the weight cast is untimed setup, as in the CUDA arm. Returns (s, flops)."""
    import numpy as np

    import oracle
    total_s, total_flops = 0.0, 0.0
    for (N, K, x, w, c) in host:
        ncol = max(128, min(N, cols // 128 * 128)) if N >= 128 else N
        b, sfb = oracle.cast_per_block(w[:ncol])
        xr = np.ascontiguousarray(x[:rows])
        cr = np.ascontiguousarray(c[:rows, :ncol]) if c is not None else None
        t0 = time.perf_counter()
        a, sfa = oracle.cast_per_token(xr)
        oracle.gemm_nt(a, sfa, b, sfb, cr)
        total_s += time.perf_counter() - t0
        total_flops += 2.0 * rows * ncol * K
    return total_s, total_flops


def cpu_baseline(wl, host, target_s=15.0):
    import oracle
    s, f = oracle_sample(wl, host, 1, 1024)                    # calibration probe
    rate = f / max(s, 1e-6)
    # rows x full N per shape, sized to about target_s of CPU work
    full_cols = max(N for N, _ in wl["shapes"])
    per_row = sum(2.0 * min(N, full_cols) * K for N, K in wl["shapes"])
    rows = int(max(1, min(wl["M"], target_s * rate / per_row)))
    s, f = oracle_sample(wl, host, rows, full_cols)
    return {"value": round(f / s / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows} rows of A x all N columns of each of the {len(wl['shapes'])} shapes "
                      f"(per-token cast of those rows + fp64 GEMM), {s:.1f} s on the host"}


def run_reference(args):
    rank, _, world = rank_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    wl = WORKLOADS[args.workload]
    host = make_inputs(wl)
    s, f = oracle_sample(wl, host, 1, 256)
    rate = f / max(s, 1e-6)
    budget = max(0.02, 120.0 / max(1, args.steps + args.warmup))   # whole run within ~2 minutes
    per_row_col = sum(2.0 * K for _, K in wl["shapes"])
    cells = max(128.0, budget * rate / per_row_col)
    cols = int(min(max(N for N, _ in wl["shapes"]), max(128, cells // 128 * 128)))
    rows = int(max(1, min(wl["M"], cells / cols)))
    for _ in range(args.warmup):
        oracle_sample(wl, host, rows, cols)
    tot_s = tot_f = 0.0
    for _ in range(args.steps):
        s, f = oracle_sample(wl, host, rows, cols)
        tot_s += s
        tot_f += f
    value = tot_f / tot_s / 1e12
    sample = (f"{rows} rows x {cols} columns (capped at N) of each of the {len(wl['shapes'])} shapes per step: "
              f"per-token cast of those rows + fp64 GEMM on the host")
    out = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": wl["desc"], "M": wl["M"], "shapes_NK": [list(s) for s in wl["shapes"]]},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="prefill")
    ap.add_argument("--only", type=str, default=None,
                    help="run a single N,K shape of the workload (profiling cases)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)          # at least three untimed warm-up steps
    return a


def main(argv=None):
    args = parse_args(argv)
    if args.only:
        n, k = (int(v) for v in args.only.split(","))
        base = WORKLOADS[args.workload]
        WORKLOADS[args.workload] = dict(base, shapes=[(n, k)], desc=f"{base['desc']}; single shape N={n} K={k}")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()

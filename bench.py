#!/usr/bin/env python
"""Benchmark of the FP8 block-scaled NT GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload prefill|config1|decode64|decode128|contiguous|masked] [--only N,K]
                    [--no-workloads] [--sub-steps S]

One step = one pass of the hot path over the workload: for each problem of the workload, the
per-token FP8 cast of its bf16 activations (1x128 scales written in the MN-major layout) and
the GEMM D = C + A·Bᵀ with 128x128-block-scaled e4m3 weights (dense, M-grouped contiguous or
M-grouped masked). Weights are cast once, before the timed region (offline, as in inference);
that cast is timed on its own and reported under "weight_cast". Inputs follow the seeded
synthetic recipe of moe_grouped_gemm_sm_b200.synth: A, B ~ N(0,1) and C ~ N(0,0.1) in bf16;
contiguous experts hold U{2048..6144} rows padded to 128; masked experts U{64..256} rows.

The default workload (the one the headline number is quoted on) is the dense prefill set:
M = 4096 with (N,K) in the six DeepSeek-V3 GEMM shapes and a C addend. The same JSON line then
carries a "workloads" object with the other page configurations, each timed in its own region
with its own roofline and per-problem times: the 64x2112x7168 decode shape with C = 0
(config1), the M = 64 and M = 128 decode sets with the L2 flushed before every step (cold) and
back to back (warm), the G = 8 contiguous and the G = 16 masked MoE sets.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device synchronise,
timed with CUDA events on the launching stream; the max over ranks is reported. When one step's
working set is below 512 MB (the decode workloads), a 256 MB L2-flushing write runs at the
start of every step, outside the per-kernel event pairs; otherwise the working set alone is far
above the 126 MB L2. Per-kernel durations come from CUDA events recorded around every launch
inside the timed region. SM clocks and throttle reasons are sampled through NVML during the
timed region.

Multi-GPU: the path has no exchange step, so N GPUs run N independent replicas (one process per
GPU under torchrun), each on the full workload ("scaling": "weak"); value = all ranks' FLOPs
divided by the slowest rank's time.

--impl reference times the oracle (plain C, fp64; oracle/) on the host cores on a bounded sample
of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import ctypes
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
GROUPED_SHAPES = [(4096, 7168), (7168, 2048)]
WORKLOADS = {
    "config1": dict(kind="dense", M=64, shapes=[(2112, 7168)], with_c=False,
                    desc="dense FP8 NT GEMM, M=64, N=2112, K=7168, C = 0 (the pages' decode headline shape)"),
    "prefill": dict(kind="dense", M=4096, shapes=PREFILL_SHAPES, with_c=True,
                    desc="dense FP8 NT GEMM, M=4096, (N,K) in the six DeepSeek-V3 prefill shapes, C bf16"),
    "decode64": dict(kind="dense", M=64, shapes=PREFILL_SHAPES, with_c=True,
                     desc="dense FP8 NT GEMM, M=64 decode, six (N,K) shapes, C bf16"),
    "decode128": dict(kind="dense", M=128, shapes=PREFILL_SHAPES, with_c=True,
                      desc="dense FP8 NT GEMM, M=128 decode, six (N,K) shapes, C bf16"),
    "contiguous": dict(kind="contiguous", G=8, shapes=GROUPED_SHAPES, with_c=False,
                       desc="M-grouped contiguous FP8 GEMM, G=8, m_g ~ U{2048..6144} padded to 128, "
                            "(N,K) in {(4096,7168),(7168,2048)}; the step's cast takes the routed tokens "
                            "(shuffled) straight into the grouped layout"),
    "masked": dict(kind="masked", G=16, M_max=256, expected_m=192, shapes=GROUPED_SHAPES, with_c=False,
                   desc="M-grouped masked FP8 GEMM, G=16, M_max=256, masked_m ~ U{64..256}, expected_m=192, "
                        "(N,K) in {(4096,7168),(7168,2048)}"),
    "prefill_ue8m0": dict(kind="dense", M=4096, shapes=PREFILL_SHAPES, with_c=True, ue8m0=True,
                          desc="dense FP8 NT GEMM with UE8M0 (power-of-two) scales and the block-scaled MMA, M=4096, "
                               "the six prefill (N,K) shapes, C bf16"),
    "layouts": dict(kind="layout", M=4096, shapes=[(4096, 7168)], layouts=("nn", "tn", "tt"), with_c=True,
                    desc="dense FP8 GEMM, M=4096, N=4096, K=7168, C bf16, in the NN, TN and TT storage layouts "
                         "(the GEMM alone: operands quantised offline, MN-major ones stored transposed)"),
    "k_grouped": dict(kind="kgrouped", G=8, shapes=[(4096, 7168), (7168, 2048)], with_c=False,
                      desc="K-grouped TN FP8 GEMM (MoE weight gradient), G=8 groups of U{2048..6144} tokens "
                           "padded to 128, (M,N) in {(4096,7168),(7168,2048)}, fp32 D; step = per-channel casts "
                           "of both token-major operands + the GEMM"),
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
# workload: problems with their host inputs, FLOPs and algorithmic bytes
# ------------------------------------------------------------------------------------------------

def make_problems(wl):
    """Host-side problems of a workload (bf16 bit patterns from the seeded generator)."""
    import numpy as np

    from moe_grouped_gemm_sm_b200 import synth
    probs = []
    items = [(i, N, K, lay) for i, (N, K) in enumerate(wl["shapes"]) for lay in wl.get("layouts", ("nt",))]
    for i, N, K, lay in items:
        kind = wl["kind"]
        p = dict(kind=kind, N=N, K=K, with_c=wl["with_c"], salt=100 + i, ue8m0=wl.get("ue8m0", False))
        if kind == "layout":
            x, w, c = synth.dense_inputs(wl["M"], N, K, wl["with_c"], salt=100 + i)
            p.update(rows=wl["M"], G=1, x=x, w=w, c=c, valid_rows=wl["M"], lay=lay)
        elif kind == "kgrouped":
            # (N, K) of the entry are the gradient's (M, N); the K dimension is the tokens
            M_, N_ = N, K
            m, _ = synth.contiguous_layout(wl["G"], salt=100 + i)
            ks = [int((v + 127) // 128 * 128) for v in m]
            T = sum(ks)
            dy = synth.normal_bf16(synth.seed_for(synth.BASE_SEED, synth.STREAM_A, 100 + i), (T, M_))
            xx = synth.normal_bf16(synth.seed_for(synth.BASE_SEED, synth.STREAM_B, 100 + i), (T, N_))
            p.update(N=N_, K=T, rows=M_, G=wl["G"], x=dy, w=xx, c=None, ks=ks, valid_rows=M_)
        elif kind == "dense":
            x, w, c = synth.dense_inputs(wl["M"], N, K, wl["with_c"], salt=100 + i)
            p.update(rows=wl["M"], G=1, x=x, w=w, c=c, valid_rows=wl["M"])
        elif kind == "contiguous":
            # the routed tokens arrive in a seeded shuffled order; the step's cast writes each
            # one to its row of the expert-grouped layout (dst), as the MoE dispatch does
            m, layout, x, w = synth.contiguous_inputs(wl["G"], N, K, salt=100 + i)
            rows = np.nonzero(layout >= 0)[0].astype(np.int32)
            dst = rows[np.random.default_rng(100 + i).permutation(rows.size)]
            p.update(rows=layout.shape[0], G=wl["G"], x=np.ascontiguousarray(x[dst]), w=w, c=None, layout=layout,
                     valid_rows=int(m.sum()), dst=dst)
        else:
            mm, x, w = synth.masked_inputs(wl["G"], wl["M_max"], N, K, salt=100 + i)
            p.update(rows=wl["M_max"], G=wl["G"], x=x, w=w, c=None, masked_m=mm, valid_rows=int(mm.sum()),
                     expected_m=wl["expected_m"])
        p["flops"] = 2.0 * p["valid_rows"] * p["N"] * p["K"]
        p["bytes"] = algorithmic_bytes(p)
        probs.append(p)
    return probs


def algorithmic_bytes(p):
    """HBM bytes one GEMM launch must move at minimum: the e4m3 A rows it must read, all
    weights, fp32 scales, the D rows it must write (and C), the grouped layout or masked_m."""
    N, K, G = p["N"], p["K"], p["G"]
    kb, nb = K // 128, (N + 127) // 128
    if p["kind"] == "kgrouped":                       # A [T,M], B [T,N], per-channel scales, fp32 D
        M, T = p["rows"], K
        pad4 = lambda v: (v + 3) // 4 * 4
        return T * M + T * N + 4 * (T // 128) * (pad4(M) + pad4(N)) + 4 * G * M * N
    w = G * N * K + 4 * G * nb * kb
    if p["kind"] in ("dense", "layout"):
        M = p["rows"]
        return M * K + 4 * M * kb + w + 2 * M * N * (2 if p["with_c"] else 1)
    if p["kind"] == "contiguous":
        M = p["rows"]                                 # the padded layout is read and written whole
        return M * K + 4 * M * kb + w + 2 * M * N + 4 * M
    V = p["valid_rows"]                               # masked: only rows below masked_m matter
    return V * K + 4 * V * kb + w + 2 * V * N + 4 * G


def fp8_tensor_peak(peaks, clocks):
    """Dense fp8 peak (TFLOP/s) for the clocks a timed region ran at, and which figure it is:
    2x the burst bf16 GEMM figure when the SM clock stayed at its maximum, 2x the sustained one
    (taken under the power cap) when the power cap was active or the median clock sat below 95 %
    of the maximum."""
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", []) or (mhz is not None and bool(top) and mhz < 0.95 * top)
    if capped:
        return 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), \
            "bf16_tflops_sustained (the power cap was active or the clock below max)"
    return 2.0 * peaks["bf16_tflops"], "bf16_tflops (burst; the clock stayed at max)"


def cast_bytes(p):
    """Per-token cast of all activation rows: 2 B read and 1 B written per element, plus scales
    (K-grouped: the per-channel casts of both token-major operands; the layout workload: none)."""
    if p["kind"] == "layout":
        return 0
    if p["kind"] == "kgrouped":
        return 3 * p["K"] * (p["rows"] + p["N"]) + 4 * (p["K"] // 128) * (p["rows"] + p["N"])
    if p["kind"] == "contiguous":                    # the routed tokens only
        return 3 * p["valid_rows"] * p["K"] + 4 * p["valid_rows"] * (p["K"] // 128)
    rows = p["rows"] * (p["G"] if p["kind"] == "masked" else 1)
    return 3 * rows * p["K"] + 4 * rows * (p["K"] // 128)


# ------------------------------------------------------------------------------------------------
# CUDA arm
# ------------------------------------------------------------------------------------------------

# The page configurations measured beside the headline, each in its own timed region:
# (key in the "workloads" object, workload, L2 policy: "flush" = a 256 MB write at the start of
# every step, "warm" = back-to-back steps, None = the default rule of the workload's size).
SUB_WORKLOADS = [
    ("config1", "config1", "flush"),
    ("decode64_cold", "decode64", "flush"),
    ("decode64_warm", "decode64", "warm"),
    ("decode128_cold", "decode128", "flush"),
    ("decode128_warm", "decode128", "warm"),
    ("contiguous", "contiguous", None),
    ("masked", "masked", None),
    ("prefill_ue8m0", "prefill_ue8m0", None),
    ("layouts", "layouts", None),
    ("k_grouped", "k_grouped", None),
]


def _json_default(o):
    """numpy scalars and arrays in the result line become plain numbers and lists."""
    import numpy as np
    if isinstance(o, np.ndarray):
        return o.tolist()
    if isinstance(o, np.generic):
        return o.item()
    raise TypeError(f"not serialisable: {type(o).__name__}")


def source_digest():
    """sha1 of the CUDA sources: the DRAM traffic stored under profiles/ holds for this digest."""
    import glob
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "moe_grouped_gemm_sm_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()


def stored_traffic(workload):
    """Per-launch DRAM bytes (read + write) of the workload's GEMM from profiles/traffic.json, or
    None when none was taken or the kernels changed since (a different source digest)."""
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tpath):
        return None
    with open(tpath) as f:
        entry = json.load(f).get(workload)
    if not isinstance(entry, dict) or entry.get("source_sha1") != source_digest():
        return None
    return entry.get("bytes_per_launch")


class CudaArm:
    """Device state of the CUDA arm: the library, the stream and the cast weights, which the
    workloads that share a weight (same shape and seed) reuse."""

    def __init__(self, device):
        import torch

        from moe_grouped_gemm_sm_b200 import _lib
        self.torch, self._lib = torch, _lib
        self.device = device
        self.L = _lib.load()
        self.stream = torch.cuda.current_stream(device)
        self.weights = {}

    def bf16(self, bits):
        import numpy as np
        t = self.torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16))
        return t.view(self.torch.bfloat16).to(self.device)

    def prepare(self, wl):
        """Device operands of every problem of a workload; the weights are cast once (offline,
        as in inference) and that cast is timed on its own."""
        import numpy as np
        torch, dev = self.torch, self.device
        from moe_grouped_gemm_sm_b200 import ops
        probs = make_problems(wl)
        wc_ms = []
        for p in probs:
            if p["kind"] == "kgrouped":
                T, M, N = p["K"], p["rows"], p["N"]
                pad4 = lambda v: (v + 3) // 4 * 4
                p["a"], p["bx"] = self.bf16(p["x"]), self.bf16(p["w"])
                p["aq"] = torch.empty((T, M), dtype=torch.uint8, device=dev)
                p["bq"] = torch.empty((T, N), dtype=torch.uint8, device=dev)
                p["sfa"] = torch.zeros((T // 128, pad4(M)), dtype=torch.float32, device=dev)
                p["sfb"] = torch.zeros((T // 128, pad4(N)), dtype=torch.float32, device=dev)
                p["d"] = torch.zeros((p["G"], M, N), dtype=torch.float32, device=dev)
                p["ks_dev"] = torch.tensor(p["ks"], dtype=torch.int32, device=dev)
                p["ks_c"] = (ctypes.c_int * len(p["ks"]))(*p["ks"])
                p["launches"] = 3
                continue
            key = (p["kind"], p["salt"], p["N"], p["K"], p["G"], p["ue8m0"])
            if key not in self.weights:
                w_dev = self.bf16(p["w"])
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                if p["ue8m0"]:
                    nb_, kq_ = (p["N"] + 127) // 128, (p["K"] // 128 + 3) // 4
                    b = torch.empty((p["N"], p["K"]), dtype=torch.uint8, device=dev)
                    sfb = torch.empty((nb_, kq_), dtype=torch.int32, device=dev)

                    def wcast():
                        self._lib.dg_cast_fp8_per_block_ue8m0(w_dev, b, sfb, 1, p["N"], p["K"], self.stream)
                else:
                    def wcast():
                        return ops.cast_per_block(w_dev)
                wcast()                                               # warm the weight cast once
                e0.record(self.stream)
                out = wcast()
                if not p["ue8m0"]:
                    b, sfb = out
                e1.record(self.stream)
                torch.cuda.synchronize(dev)
                nb, kb = (p["N"] + 127) // 128, p["K"] // 128
                self.weights[key] = (b, sfb, e0.elapsed_time(e1), p["G"] * (3 * p["N"] * p["K"] + 4 * nb * kb))
                del w_dev
            p["b"], p["sfb"], t, nbytes = self.weights[key]
            wc_ms.append((t, nbytes))
            p["a"] = self.bf16(p["x"])
            p["cd"] = self.bf16(p["c"]) if p["c"] is not None else None
            batch = p["G"] if p["kind"] == "masked" else 1
            p["batch"] = batch
            p["aq"] = torch.empty(p["a"].shape, dtype=torch.uint8, device=dev)
            if p["ue8m0"]:
                p["sfa"] = torch.zeros(((p["K"] // 128 + 3) // 4, (p["rows"] + 3) // 4 * 4), dtype=torch.int32,
                                       device=dev)
            else:
                p["sfa"] = torch.empty((batch, p["K"] // 128, (p["rows"] + 3) // 4 * 4), dtype=torch.float32,
                                       device=dev)
            dshape = (p["G"], p["rows"], p["N"]) if p["kind"] == "masked" else (p["rows"], p["N"])
            p["d"] = torch.zeros(dshape, dtype=torch.bfloat16, device=dev)
            if p["kind"] == "contiguous":
                p["gl"] = torch.from_numpy(p["layout"]).to(dev)
                p["dst_dev"] = torch.from_numpy(p["dst"]).to(dev)
                p["aq"] = torch.zeros((p["rows"], p["K"]), dtype=torch.uint8, device=dev)
                p["sfa"] = torch.zeros((1, p["K"] // 128, (p["rows"] + 3) // 4 * 4), dtype=torch.float32, device=dev)
            if p["kind"] == "masked":
                p["mm"] = torch.from_numpy(p["masked_m"]).to(dev)
            p["launches"] = 2
            if p["kind"] == "layout":
                # operands quantised once (untimed), stored in the layout's order
                self.launch_cast(dict(p, kind="dense"), self.stream.cuda_stream)
                if p["lay"][0] == "t":
                    p["aq"] = p["aq"].t().contiguous()
                if p["lay"][1] == "n":
                    p["b"] = p["b"].t().contiguous()
                p["launches"] = 1
        torch.cuda.synchronize(dev)
        return probs, wc_ms

    # ---- launches through the C ABI (the same calls a user makes) ----
    def launch_cast(self, p, sptr):
        if p["kind"] == "layout":                           # operands were quantised offline
            return
        if p["kind"] == "kgrouped":
            for x, q, sf, C in ((p["a"], p["aq"], p["sfa"], p["rows"]), (p["bx"], p["bq"], p["sfb"], p["N"])):
                rc = self.L.dg_cast_fp8_per_channel(x.data_ptr(), q.data_ptr(), sf.data_ptr(), p["K"], C, sptr)
                if rc:
                    raise self._lib.DgError("dg_cast_fp8_per_channel", rc)
            return
        if p["kind"] == "contiguous":                       # the MoE dispatch: cast into the grouped layout
            rc = self.L.dg_cast_fp8_per_token_scatter(p["a"].data_ptr(), p["dst_dev"].data_ptr(), p["aq"].data_ptr(),
                                                      p["sfa"].data_ptr(), p["valid_rows"], p["rows"], p["K"], sptr)
            if rc:
                raise self._lib.DgError("dg_cast_fp8_per_token_scatter", rc)
            return
        f = self.L.dg_cast_fp8_per_token_ue8m0 if p.get("ue8m0") else self.L.dg_cast_fp8_per_token
        rc = f(p["a"].data_ptr(), p["aq"].data_ptr(), p["sfa"].data_ptr(), p["batch"], p["rows"], p["K"], sptr)
        if rc:
            raise self._lib.DgError("dg_cast_fp8_per_token", rc)

    def launch_gemm(self, p, sptr):
        L = self.L

        def ptr(t):
            return t.data_ptr() if t is not None else None
        if p["kind"] == "dense":
            f = L.dg_fp8_gemm_nt_ue8m0 if p.get("ue8m0") else L.dg_fp8_gemm_nt
            rc = f(ptr(p["aq"]), ptr(p["sfa"]), ptr(p["b"]), ptr(p["sfb"]), ptr(p["cd"]), ptr(p["d"]), p["rows"], p["N"],
                   p["K"], sptr)
        elif p["kind"] == "layout":
            f = getattr(L, "dg_fp8_gemm_" + p["lay"])
            rc = f(ptr(p["aq"]), ptr(p["sfa"]), ptr(p["b"]), ptr(p["sfb"]), ptr(p["cd"]), ptr(p["d"]), p["rows"],
                   p["N"], p["K"], sptr)
        elif p["kind"] == "kgrouped":
            rc = L.dg_k_grouped_fp8_gemm_tn_contiguous(ptr(p["aq"]), ptr(p["sfa"]), ptr(p["bq"]), ptr(p["sfb"]), None,
                                                       ptr(p["d"]), ctypes.cast(p["ks_c"], ctypes.c_void_p),
                                                       ptr(p["ks_dev"]), p["G"], p["rows"], p["N"], sptr)
        elif p["kind"] == "contiguous":
            rc = L.dg_m_grouped_fp8_gemm_nt_contiguous(ptr(p["aq"]), ptr(p["sfa"]), ptr(p["b"]), ptr(p["sfb"]),
                                                       ptr(p["cd"]), ptr(p["d"]), ptr(p["gl"]), p["rows"], p["N"],
                                                       p["K"], p["G"], sptr)
        else:
            rc = L.dg_m_grouped_fp8_gemm_nt_masked(ptr(p["aq"]), ptr(p["sfa"]), ptr(p["b"]), ptr(p["sfb"]),
                                                   ptr(p["cd"]), ptr(p["d"]), ptr(p["mm"]), p["expected_m"], p["G"],
                                                   p["rows"], p["N"], p["K"], sptr)
        if rc:
            raise self._lib.DgError("gemm", rc)

    def time_steps(self, probs, steps, warmup, l2, local_rank):
        """Times `steps` steps (per-token cast + GEMM per problem) as replays of one CUDA graph,
        with CUDA events on the launching stream, clocks sampled during the region; then the
        per-kernel durations from a second graph with an event pair around every launch."""
        torch, dev = self.torch, self.device
        stream = self.stream
        step_bytes = sum(p["bytes"] + cast_bytes(p) for p in probs)
        if l2 is None:
            l2 = "flush" if step_bytes < 512 * 2 ** 20 else "large"
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev) if l2 == "flush" else None

        # cold steps: an event pair inside the step graph brackets the work after the flush, so
        # that the step time does not include the flushing write itself
        fev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] if flush is not None else None

        def step(sptr, ev=None, fe=None):
            if flush is not None:
                flush.fill_(1)
                # then read it back: the write leaves L2 full of dirty lines, whose write-back
                # would otherwise compete with the step's reads; after the read L2 holds clean
                # lines of the flush buffer only (the step's operands are still cold)
                flush.view(torch.int32).amax()
            cur = torch.cuda.current_stream(dev)
            if fe is not None:
                fe[0].record(cur)
            for i, p in enumerate(probs):
                if ev is not None:
                    ev[3 * i].record(cur)
                self.launch_cast(p, sptr)
                if ev is not None:
                    ev[3 * i + 1].record(cur)
                self.launch_gemm(p, sptr)
                if ev is not None:
                    ev[3 * i + 2].record(cur)
            if fe is not None:
                fe[1].record(cur)

        # eager warm-up, which also names the kernel each problem takes
        for p in probs:
            self.launch_cast(p, stream.cuda_stream)
            self.launch_gemm(p, stream.cuda_stream)
            p["kernel"] = self._lib.dg_last_kernel()
            p["launches"] += self._lib.dg_last_launch_count() - 1   # a last-wave split adds one
        for _ in range(warmup):
            step(stream.cuda_stream)
        torch.cuda.synchronize(dev)
        if self._lib.dg_get_device_error(stream.cuda_stream) != 0:
            raise RuntimeError("device error word set during warm-up")

        # The timed steps replay CUDA graphs (launch-bound decode steps would otherwise measure the
        # host): `g_step` holds one step; `g_ev` the same step with an event pair around every
        # launch, replayed separately for the per-kernel durations.
        cap = torch.cuda.Stream(dev)
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3 * len(probs))]
        g_step, g_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            step(cap.cuda_stream)                                 # warm the capture stream
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(g_step, stream=cap):
                step(cap.cuda_stream, fe=fev)
            with torch.cuda.graph(g_ev, stream=cap):
                step(cap.cuda_stream, evs)
        torch.cuda.synchronize(dev)
        for _ in range(warmup):
            g_step.replay()
        torch.cuda.synchronize(dev)

        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize(dev)
        work_ms = []
        with ClockSampler(local_rank) as clk:
            start.record(stream)
            for _ in range(steps):
                g_step.replay()
                if fev is not None:                               # cold: read each step's pair
                    torch.cuda.synchronize(dev)
                    work_ms.append(fev[0].elapsed_time(fev[1]))
            end.record(stream)
            torch.cuda.synchronize(dev)
        barrier(dev)
        with_flush_ms = start.elapsed_time(end) / steps
        local_ms = statistics.fmean(work_ms) if work_ms else with_flush_ms
        if self._lib.dg_get_device_error(stream.cuda_stream) != 0:
            raise RuntimeError("device error word set during the timed region")
        cast_t = [[] for _ in probs]
        gemm_t = [[] for _ in probs]
        for _ in range(min(steps, 50)):
            g_ev.replay()
            torch.cuda.synchronize(dev)
            for i in range(len(probs)):
                cast_t[i].append(evs[3 * i].elapsed_time(evs[3 * i + 1]))
                gemm_t[i].append(evs[3 * i + 1].elapsed_time(evs[3 * i + 2]))
        del g_step, g_ev
        return dict(local_ms=local_ms, with_flush_ms=with_flush_ms if work_ms else None,
                    cast_ms=[statistics.fmean(v) for v in cast_t],
                    gemm_ms=[statistics.fmean(v) for v in gemm_t], clocks=clk.summary(), l2=l2,
                    launches_per_step=sum(p["launches"] for p in probs))   # the library's own kernels only


L2_TEXT = {"flush": "256 MB L2-flushing write, then a read of the same buffer (so that no dirty line's write-back "
                    "overlaps the step), at the start of every step (cold weights); the step time is taken by an "
                    "event pair inside the step graph after the flush, so it excludes the flush "
                    "(ms_per_step_with_flush includes it)",
           "warm": "no flush: steps back to back (weights partly L2-resident)",
           "large": "no flush: one step's working set is far above the 126 MB L2"}


def roofline_of(probs, t, workload):
    """Roofline of the dominant kernel (the GEMM) over a workload's launches, and per problem."""
    peaks, peaks_src = load_peaks()
    # fp8 dense = 2 x bf16 (nominal ratio). The denominator matches the clocks the timed region
    # ran at: the burst figure when the SM clock stayed at its maximum, the sustained one (taken
    # in a seconds-long loop under the power cap) when the power cap was active or the median
    # clock sat below 95 % of the maximum. Both fractions are reported.
    fp8_peak, peak_kind = fp8_tensor_peak(peaks, t["clocks"])
    fp8_peak_burst = 2.0 * peaks["bf16_tflops"]
    fp8_peak_sustained = 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    hbm = peaks["hbm_gbs"]
    per_problem = []
    t_roof_total = 0.0
    for p, gm, cm in zip(probs, t["gemm_ms"], t["cast_ms"]):
        t_tc = p["flops"] / (fp8_peak * 1e12)
        t_hbm = p["bytes"] / (hbm * 1e9)
        t_roof_total += max(t_tc, t_hbm)
        per_problem.append({"N": p["N"], "K": p["K"], "rows": p["rows"], "G": p["G"], "layout": p.get("lay", "nt"),
                            "kernel": p.get("kernel", ""), "flops": p["flops"], "bytes": p["bytes"],
                            "gemm_us": round(gm * 1e3, 2),
                            "tflops": round(p["flops"] / (gm * 1e-3) / 1e12, 1),
                            "gbs": round(p["bytes"] / (gm * 1e-3) / 1e9, 1),
                            "bound": "tensor" if t_tc >= t_hbm else "hbm",
                            "roof_frac": round(max(t_tc, t_hbm) / (gm * 1e-3), 3),
                            "cast_us": round(cm * 1e3, 2),
                            "cast_gbs": round(cast_bytes(p) / (cm * 1e-3) / 1e9, 1)})
    gemm_total_s = sum(t["gemm_ms"]) * 1e-3
    flops_sum = sum(p["flops"] for p in probs)
    bytes_sum = sum(p["bytes"] for p in probs)
    if flops_sum / (fp8_peak * 1e12) >= bytes_sum / (hbm * 1e9):
        achieved = flops_sum / gemm_total_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / fp8_peak, 4),
                "peak_source": f"{peaks_src}: 2 x {peak_kind}; fp8 = 2x bf16 nominal ratio",
                "frac_of_burst_peak": round(achieved / fp8_peak_burst, 4),
                "frac_of_sustained_peak": round(achieved / fp8_peak_sustained, 4)}
    else:
        achieved = bytes_sum / gemm_total_s / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": round(hbm, 1), "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": f"{peaks_src}: hbm_gbs (copy bandwidth)"}
    roof["roofline_time_frac"] = round(t_roof_total / gemm_total_s, 4)
    names = sorted({p["kernel"] for p in per_problem})
    roof["kernel"] = f"{' + '.join(names)} ({len(probs)} problems, aggregate over launches)"
    roof["timing"] = ("per-kernel CUDA events from a second graph with an event pair around every launch; the "
                      "pairs stop the GEMM's prologue from overlapping the cast (programmatic dependent launch), "
                      "so achieved slightly understates the GEMM")
    roof["traffic"] = stored_traffic(workload)
    return roof, per_problem


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
    arm = CudaArm(device)
    stream = arm.stream
    wl = WORKLOADS[args.workload]

    probs, wc_ms = arm.prepare(wl)
    t = arm.time_steps(probs, args.steps, args.warmup, None, local_rank)
    flops_step = sum(p["flops"] for p in probs)
    ms_max, flops_all = aggregate(t["local_ms"], flops_step, device)
    value = flops_all / (ms_max * 1e-3) / 1e12

    # ---------------- e2e through the public API with pinned host buffers ----------------
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for p in probs:
        p["ah"] = torch.from_numpy(np.ascontiguousarray(p["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        p["ch"] = torch.from_numpy(np.ascontiguousarray(p["c"]).view(np.int16)).view(torch.bfloat16).pin_memory() \
            if p["c"] is not None else None
        p["dh"] = torch.empty(p["d"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(p["ah"].numel() * 2 + (p["ch"].numel() * 2 if p["ch"] is not None else 0) for p in probs)
    d2h = sum(p["dh"].numel() * 2 for p in probs)

    def e2e_step():
        for p in probs:
            p["a"].copy_(p["ah"], non_blocking=True)
            if p["ch"] is not None:
                p["cd"].copy_(p["ch"], non_blocking=True)
            a_q, sfa = ops.cast_per_token(p["a"], stream=stream)
            if p["kind"] == "dense":
                d = ops.fp8_gemm_nt(a_q, sfa, p["b"], p["sfb"], p["cd"], out=p["d"], stream=stream)
            elif p["kind"] == "contiguous":
                d = ops.m_grouped_fp8_gemm_nt_contiguous(a_q, sfa, p["b"], p["sfb"], p["gl"], p["cd"], out=p["d"],
                                                         stream=stream)
            else:
                d = ops.m_grouped_fp8_gemm_nt_masked(a_q, sfa, p["b"], p["sfb"], p["mm"], p["expected_m"], p["cd"],
                                                     out=p["d"], stream=stream)
            p["dh"].copy_(d, non_blocking=True)

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

    roof, per_problem = roofline_of(probs, t, args.workload)
    clocks = t["clocks"]
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": wl["desc"], "shapes_NK": [list(s) for s in wl["shapes"]],
                   "step": "per-token cast of A + GEMM per problem; weights cast offline",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": L2_TEXT[t["l2"]]},
        "roofline": roof,
        "per_problem": per_problem,
        "weight_cast": {"gbs": round(sum(b for _, b in wc_ms) / (sum(x for x, _ in wc_ms) * 1e-3) / 1e9, 1),
                        "ms_total": round(sum(x for x, _ in wc_ms), 3)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "path": "pinned host activations (and C) -> device, ops cast + GEMM, D -> pinned host"},
        "gpu_launches": t["launches_per_step"] * args.steps,
        "launch": "each step replays a CUDA graph of its launches",
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, probs, target_s=args.cpu_seconds)
    for p in probs:
        p.clear()
    del probs
    arm.weights.clear()
    torch.cuda.empty_cache()

    # ---------------- the other page configurations, each in its own timed region ----------------
    if not args.no_workloads and not args.only:
        subs = {}
        for key, name, l2 in SUB_WORKLOADS:
            swl = WORKLOADS[name]
            sprobs, _ = arm.prepare(swl)
            st = arm.time_steps(sprobs, args.sub_steps, 3, l2, local_rank)
            sms, sflops = aggregate(st["local_ms"], sum(p["flops"] for p in sprobs), device)
            sroof, spp = roofline_of(sprobs, st, name if l2 != "warm" else key)
            subs[key] = {"workload": swl["desc"], "value": round(sflops / (sms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                         "ms_per_step": round(sms, 4), "steps": args.sub_steps, "l2": L2_TEXT[st["l2"]],
                         "ms_per_step_with_flush": (round(reduce_max(st["with_flush_ms"], device), 4)
                                                    if st["with_flush_ms"] is not None else None),
                         "gpu_launches": st["launches_per_step"] * args.sub_steps,
                         "roofline": sroof, "per_problem": spp, "clocks": st["clocks"]}
            for p in sprobs:
                p.clear()
            del sprobs
            if name != "decode64":                              # decode128 reuses decode64's weights
                arm.weights.clear()
            torch.cuda.empty_cache()
        result["workloads"] = subs

    if rank == 0:
        print(json.dumps(result, default=_json_default), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------------------------
# oracle (CPU) arm and baseline
# ------------------------------------------------------------------------------------------------

def oracle_sample(probs, rows: int, cols: int):
    """Times the oracle on `rows` rows x `cols` columns of every problem: the per-token cast of
    those activation rows and their fp64 GEMM against the matching weights (expert 0 for the
    grouped layouts, whose first rows belong to it). The weight cast is untimed setup, as in
    the CUDA arm. Returns (seconds, flops)."""
    import numpy as np

    import oracle
    total_s, total_flops = 0.0, 0.0
    for p in probs:
        N, K = p["N"], p["K"]
        ncol = N if N < 128 else max(128, min(N, cols // 128 * 128))
        w = p["w"] if p["kind"] == "dense" else p["w"][0]
        if p["kind"] == "masked":
            x, avail = p["x"][0], int(p["masked_m"][0])
        elif p["kind"] == "contiguous":
            x, avail = p["x"], int((p["layout"] == 0).sum())
        else:
            x, avail = p["x"], p["x"].shape[0]
        r = max(1, min(rows, avail))
        b, sfb = oracle.cast_per_block(w[:ncol])
        xr = np.ascontiguousarray(x[:r])
        cr = np.ascontiguousarray(p["c"][:r, :ncol]) if p["c"] is not None else None
        t0 = time.perf_counter()
        a, sfa = oracle.cast_per_token(xr)
        oracle.gemm_nt(a, sfa, b, sfb, cr)
        total_s += time.perf_counter() - t0
        total_flops += 2.0 * r * ncol * K
    return total_s, total_flops


def cpu_baseline(wl, probs, target_s=15.0):
    import oracle
    s, f = oracle_sample(probs, 1, 1024)                      # calibration probe
    rate = f / max(s, 1e-6)
    per_row = sum(2.0 * p["N"] * p["K"] for p in probs)
    rows = int(max(1, min(64 if wl["kind"] == "masked" else 4096, target_s * rate / per_row)))
    s, f = oracle_sample(probs, rows, max(p["N"] for p in probs))
    return {"value": round(f / s / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {rows} activation rows x all N columns of each of the {len(probs)} problems "
                      f"(per-token cast of those rows + fp64 GEMM), {s:.1f} s on the host"}


def run_reference(args):
    rank, _, world = rank_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    wl = WORKLOADS[args.workload]
    probs = make_problems(wl)
    s, f = oracle_sample(probs, 1, 256)
    rate = f / max(s, 1e-6)
    budget = max(0.02, 120.0 / max(1, args.steps + args.warmup))   # whole run within ~2 minutes
    per_row_col = sum(2.0 * p["K"] for p in probs)
    cells = max(128.0, budget * rate / per_row_col)
    cols = int(min(max(p["N"] for p in probs), max(128, cells // 128 * 128)))
    rows = int(max(1, cells / cols))
    for _ in range(args.warmup):
        oracle_sample(probs, rows, cols)
    tot_s = tot_f = 0.0
    for _ in range(args.steps):
        s, f = oracle_sample(probs, rows, cols)
        tot_s += s
        tot_f += f
    value = tot_f / tot_s / 1e12
    sample = (f"up to {rows} rows x {cols} columns (capped at N) of each of the {len(probs)} problems per step: "
              f"per-token cast of those rows + fp64 GEMM on the host")
    out = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": wl["desc"], "shapes_NK": [list(s) for s in wl["shapes"]]},
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
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other page configurations (the 'workloads' object)")
    ap.add_argument("--sub-steps", type=int, default=30,
                    help="timed steps of each of the other page configurations")
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

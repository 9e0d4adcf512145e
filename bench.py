#!/usr/bin/env python
"""Benchmark of the LLM.int8() mixed-precision decomposition matmul on B200.

Default workload: the 7B decode GEMV sweep -- X fp16 [T, 4096] for
T = 1, 2, 4, 8, 16 against W [11008, 4096], four systematic outlier dims,
threshold 6.0.  One step = the five llmint8_matmul calls, each on its own
weight matrix (five independent layers, so no call finds its weights in L2).
L2 is flushed (256 MiB write) before every timed step.  Metric: algorithmic
HBM bytes / time (Wq + Wscale + outlier columns of W + X + Y).

Prefill workloads (--workload 7b_prefill | 13b_up | 70b_up) report effective
TOPS = 2 T N K / time.  At N=1 the default run also measures, under "also":
the prefill workloads (70B at thresholds 6, 4 and inf), the FP8 (E4M3) and
SmoothQuant W8A8 variants on the 7B / 13B prefill shapes, and the decode step
with E4M3 codes and with a column store of outlier weights instead of the fp16
W; each entry with its roofline and the CPU oracle timed on a sample of it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the plain C statement of the method
that the tests check the kernels against) on the host cores, on a bounded
sample of the same workload.  Under torchrun, rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_mixed_precision_outlier_b200 import synth  # noqa: E402

METRIC = "LLM.int8 matmul effective TOPS (2TNK/s) vs int8 TC peak; decode GEMV HBM GB/s"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense ratio: 4.5 POPS int8 / 2.25 PFLOPS bf16
PUBLISHED = {"hbm_gbs": 8000.0, "int8_tops": 4500.0}  # B200 data-sheet figures (dense), for context
THRESHOLD = 6.0
FLUSH_BYTES = 256 << 20


class L2Flush:
    """Evicts L2 between timed steps: writes a 256 MiB buffer (2x L2), then
    reads a second one, so L2 ends up holding clean lines of neither the
    workload nor the flush.  Without the read, the timed kernels would also pay
    for writing back the flush buffer's dirty lines."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def zero_(self, gate_us: float = 0.0):
        import torch
        self.w.zero_()
        torch.amax(self.r)
        if gate_us > 0:
            # a bounded spin of the GPU (no flag, fixed cycle count): the host
            # enqueues what follows before the GPU gets to it, so the events
            # measure GPU time, not host launch latency
            torch.cuda._sleep(int(gate_us * 2000))
DECODE_TS = (1, 2, 4, 8, 16)


# ----------------------------------------------------------------- helpers

def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK, source="fallback")


def _strip_comments(src: str) -> str:
    """C/C++ source with // and /* */ comments removed and each remaining line
    stripped of surrounding whitespace; string and character literals are
    kept as they are."""
    out = []
    i, n = 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.strip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_digest() -> str:
    """sha256 over the code of the CUDA sources (comments and blank lines
    excluded): a recorded ncu traffic figure is only used while the kernels it
    was measured on are unchanged."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int8_mixed_precision_outlier_b200", "csrc")
    for f in sorted(glob.glob(os.path.join(csrc, "*.cu*"))):
        with open(f, encoding="utf-8") as fh:
            code = _strip_comments(fh.read())
        h.update(os.path.basename(f).encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def traffic_key(workload: str, tau: float) -> str:
    """The workload's name in profiles/traffic.txt: with '@tau' when the call
    runs at a threshold other than the default (the 70B sweep)."""
    return workload if tau == THRESHOLD else f"{workload}@{tau:g}"


def recorded_traffic(workload: str, kernel: str):
    """dram bytes per launch of `kernel` on `workload` (a traffic_key) from
    profiles/traffic.txt (lines: workload kernel source_digest bytes_per_launch),
    or None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    digest = source_digest()
    with open(p) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) == 4 and parts[0] == workload and parts[1] == kernel and parts[2] == digest:
                return float(parts[3])
    return None


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, world: int) -> float:
    """Max over ranks (the slowest rank sets the job's time)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int) -> float:
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x2: "applications_clocks_setting", 0x10: "sync_boost"}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML, back to back, from
    before the timed region to its end; `mark()` opens the timed window (a
    sample is also taken synchronously at each end of it)."""

    def __init__(self, cuda_index: int, period_s: float = 0.0005):
        self.samples, self.window, self.reasons, self.max_mhz, self.ok = [], [], 0, None, False
        self._stop = threading.Event()
        self._in_window = False
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = cuda_index
            if vis and all(v.strip().isdigit() for v in vis.split(",")):
                idx = int(vis.split(",")[cuda_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self._nv
        try:
            mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            return
        self.samples.append(mhz)
        if self._in_window:
            self.window.append(mhz)
            self.reasons |= r

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self._period)

    def mark(self, inside: bool):
        if self.ok:
            if inside:
                self._in_window = True
                self._sample()
            else:
                self._sample()
                self._in_window = False

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self) -> dict:
        if not self.ok or not self.window:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "NVML sampling unavailable"}
        names = [n for bit, n in REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.window)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.window), "sm_mhz_min": float(min(self.window))}


# ----------------------------------------------------------------- workloads

VARIANTS = ("llmint8", "fp8", "smoothquant", "stored")


class Workload:
    """Device-resident inputs and the list of calls one step makes.

    variant: "llmint8" (llmint8_matmul with the fp16 W), "fp8" (E4M3 codes,
    llmint8_fp8_matmul), "smoothquant" (W8A8 with factors from the workload's
    own activations at alpha 0.5, llmint8_smoothquant_matmul) or "stored"
    (llmint8_matmul_stored with the workload's systematic outlier dims in a
    column store and no fp16 W)."""

    def __init__(self, name: str, device, seed: int = 0, taus=None, variant: str = "llmint8"):
        import torch
        import int8_mixed_precision_outlier_b200 as L
        assert variant in VARIANTS, variant
        self.L, self.name, self.device, self.variant = L, name, device, variant
        cfg = synth.WORKLOADS[name]
        self.K, self.N = cfg["K"], cfg["N"]
        self.calls = []
        if name == "7b_decode":
            ws = L.alloc_workspace(16, self.N, self.K, device)
            for layer, T in enumerate(DECODE_TS):
                w = synth.workload(name, seed=seed, T=T, layer=layer)
                self._add(w, T, THRESHOLD, ws)
            self.unit, self.kind = "GB/s", "hbm"
        else:
            w = synth.workload(name, seed=seed)
            ws = L.alloc_workspace(w["T"], self.N, self.K, device)
            taus = taus if taus is not None else ((THRESHOLD,) if name != "70b_up" else w["thresholds"])
            shared = None
            for tau in taus:
                shared = self._add(w, w["T"], tau, ws, shared=shared)
            self.unit, self.kind = "TOPS", "tensor"
        torch.cuda.synchronize()
        self.bytes_per_step = sum(c["bytes"] for c in self.calls)
        self.ops_per_step = sum(c["ops"] for c in self.calls)
        self.launches_per_step = sum(self._launches(c["T"]) for c in self.calls)
        self.graph = None

    def _launches(self, T):
        if self.variant == "smoothquant":
            return 2                     # activation kernel + GEMV / GEMM
        return self.L.llmint8_kernel_launches(T, self.N, self.K)

    def capture(self):
        """One step as a CUDA graph (the kernels keep their programmatic
        dependent-launch edges); replaying it costs one host call."""
        import torch
        self.step()  # first calls on this device happen outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        torch.cuda.synchronize()
        self.graph = g
        return g

    def _add(self, w, T, tau, ws, shared=None):
        import torch
        L = self.L
        X = torch.from_numpy(w["X"]).to(self.device)
        K, N = self.K, self.N
        if shared is None:
            W = torch.from_numpy(w["W"]).to(self.device)
            shared = {"W": W}
            if self.variant == "fp8":
                shared["Wq"], shared["sw"] = L.llmint8_fp8_quantize_weight(W)
            elif self.variant == "smoothquant":
                ax = L.llmint8_column_absmax(X)
                aw = L.llmint8_column_absmax(W)
                shared["s"] = L.llmint8_smooth_factors(ax, aw, 0.5)
                shared["Wq"], shared["sw"] = L.llmint8_smoothquant_quantize_weight(W, shared["s"])
                shared["ws"] = torch.empty(int(L.load_library().llmint8_smoothquant_workspace_bytes(T, K)),
                                           dtype=torch.uint8, device=self.device)
            else:
                shared["Wq"], shared["sw"] = L.llmint8_quantize_weight(W)
            if self.variant == "stored":
                cols = torch.from_numpy(np.sort(w["dims"]).astype(np.int32)).to(self.device)
                shared["slot"], shared["Wst"] = L.llmint8_outlier_store_build(W, cols)
                shared["n_store"] = int(cols.numel())
                shared["miss"] = torch.zeros(1, dtype=torch.int32, device=self.device)
        Y = torch.empty((T, N), dtype=torch.float16, device=self.device)
        if self.variant == "smoothquant":
            nO = 0
        else:
            _, _, idx = L.llmint8_detect_quantize(X, tau)
            nO = int(idx.numel())
        algo_bytes = N * K + 4 * N + 2 * N * nO + 2 * T * K + 2 * T * N
        c = dict(X=X, Y=Y, ws=ws, tau=tau, T=T, nO=nO, bytes=algo_bytes, ops=2 * T * N * K,
                 host_X=w["X"], host_W=w["W"], dims=w["dims"])
        c.update({k: v for k, v in shared.items() if k not in ("ws",)})
        if self.variant == "smoothquant":
            c["ws"] = shared["ws"]
        self.calls.append(c)
        return shared

    def call(self, c, Y=None):
        """One library call of this workload's variant."""
        L = self.L
        Y = c["Y"] if Y is None else Y
        if self.variant == "llmint8":
            return L.llmint8_matmul(c["X"], c["Wq"], c["sw"], c["W"], c["tau"], c["ws"], Y)
        if self.variant == "fp8":
            return L.llmint8_fp8_matmul(c["X"], c["Wq"], c["sw"], c["W"], c["tau"], c["ws"], Y)
        if self.variant == "smoothquant":
            return L.llmint8_smoothquant_matmul(c["X"], c["s"], c["Wq"], c["sw"], c["ws"], Y)
        return L.llmint8_matmul_stored(c["X"], c["Wq"], c["sw"], c["slot"], c["Wst"], c["tau"], c["ws"], Y,
                                       n_miss=c["miss"])

    def step(self):
        for c in self.calls:
            self.call(c)

    def metric_value(self, seconds: float, steps: int) -> float:
        if self.unit == "GB/s":
            return self.bytes_per_step * steps / seconds / 1e9
        return self.ops_per_step * steps / seconds / 1e12

    def resident_weight_bytes(self) -> int:
        """Weight bytes one call keeps on the device for its matrix."""
        c = self.calls[0]
        n = c["Wq"].numel() + 4 * c["sw"].numel()
        if self.variant == "stored":
            return n + 2 * c["Wst"].numel() + 4 * c["slot"].numel()
        if self.variant == "smoothquant":
            return n + 4 * self.K
        return n + 2 * c["W"].numel()


def time_steps(wl: Workload, steps: int, warmup: int, world: int, flush, run=None, gate_us=0.0):
    """Events around each step on the launching stream; L2 flushed before each.
    The clock sampler runs through warm-up and timing; its window is the timed
    steps."""
    import torch
    run = run or wl.step
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        for _ in range(warmup):
            flush.zero_(gate_us)
            run()
        barrier(world)
        torch.cuda.synchronize()
        sampler.mark(True)
        for i in range(steps):
            flush.zero_(gate_us)
            starts[i].record(stream)
            run()
            ends[i].record(stream)
        torch.cuda.synchronize()
        sampler.mark(False)
    barrier(world)
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    return total_ms, sampler.summary()


def time_cold_units(wl: Workload, steps: int, flush) -> tuple[float, float]:
    """Average duration of one cold unit (flush before each step, the step's
    calls in order, one launch per event pair).

    Decode: one whole call (prep kernel + GEMV, which starts its weight stream
    while the prep kernel runs).  Prefill: the GEMM launch alone (events
    between the activation kernels and it).  Returns (ms per unit, algorithmic
    bytes or ops per unit)."""
    import torch
    L = wl.L
    runs = []
    for _ in range(steps):
        flush.zero_(gate_us=300.0)  # the host queues the whole step while the GPU waits
        for c in wl.calls:
            b = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            if wl.unit == "GB/s" or wl.variant != "llmint8":
                b.record()
                wl.call(c)
                e.record()
            else:
                L.llmint8_matmul_profile(c["X"], c["Wq"], c["sw"], c["W"], c["tau"], c["ws"], c["Y"], b, e,
                                         repeat=1)
            runs.append((b, e, c))
    torch.cuda.synchronize()
    total = sum(b.elapsed_time(e) for b, e, _ in runs)
    algo = sum(c["bytes"] if wl.unit == "GB/s" else c["ops"] for _, _, c in runs)
    return total / len(runs), algo / len(runs)


def time_back_to_back(wl: Workload, flush, repeat: int = 5) -> float:
    """Average duration of the prefill GEMM launched `repeat` times back to back
    on one workspace (the profiling entry: activation kernels once, then the
    GEMM relaunched, each launch chained to the previous one as consecutive
    layers chain), events around the repeats, L2 flushed first.  Returns ms per
    launch over three such groups."""
    import torch
    c = wl.calls[0]
    total, n = 0.0, 0
    for _ in range(3):
        flush.zero_(gate_us=300.0)
        b = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        wl.L.llmint8_matmul_profile(c["X"], c["Wq"], c["sw"], c["W"], c["tau"], c["ws"], c["Y"], b, e,
                                    repeat=repeat)
        torch.cuda.synchronize()
        total += b.elapsed_time(e)
        n += repeat
    return total / n


def main_kernel_name(wl: Workload) -> str:
    if wl.unit == "GB/s":
        return "decode_call" if wl.variant == "llmint8" else f"decode_call_{wl.variant}"
    return "gemm_pair_kernel" if wl.variant == "llmint8" else f"call_{wl.variant}"


def decode_roofline(wl: Workload, ms_per_step: float, cold_ms: float, cold_algo: float, peaks: dict,
                    traffic=None) -> dict:
    """The decode call as it runs inside the graph-replayed step: the step's
    algorithmic bytes over its device time (5 calls per step), so that the
    unit and the headline share one definition; the cold single call (events
    around one call after an L2 flush) is reported beside it as a bound."""
    achieved = wl.bytes_per_step / (ms_per_step * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    cold = cold_algo / (cold_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": "decode_prep_kernel + gemv_kernel, one call as it runs in the step "
                      f"({len(wl.calls)} calls per step; step bytes / step time)",
            "peak_source": f"{peaks['source']} hbm_gbs (copy, burst)",
            "frac_of_published": round(achieved / PUBLISHED["hbm_gbs"], 4),
            "algo_bytes_per_launch": int(wl.bytes_per_step / len(wl.calls)),
            "ms_per_launch": round(ms_per_step / len(wl.calls), 5),
            "cold_call": {"achieved": round(cold, 1), "frac": round(cold / peak, 4), "ms": round(cold_ms, 5),
                          "how": "one call between events after an L2 flush (a bound: no overlap with the "
                                 "neighbouring calls)"}}


def prefill_roofline(wl: Workload, kern_ms: float, c: dict, peaks: dict, traffic=None, kernel=None,
                     b2b_ms=None) -> dict:
    """Tensor-bound roofline of one prefill launch.  The target time splits
    the work as the method does: 2 T N |R| products on the 8-bit tensor peak
    (int8 or fp8: measured bf16 burst x 2, the nominal ratio) and 2 T N |O|
    on the fp16 peak (measured bf16 burst, the same rate).  achieved =
    2 T N K / time; peak = 2 T N K / target time, so frac = target / time."""
    T, N, K = c["T"], wl.N, wl.K
    p8 = peaks["bf16_tflops"] * INT8_PER_BF16 * 1e12
    p16 = peaks["bf16_tflops"] * 1e12
    nO = c["nO"]
    target_s = 2.0 * T * N * (K - nO) / p8 + 2.0 * T * N * nO / p16
    ops = 2.0 * T * N * K
    achieved = ops / (kern_ms * 1e-3) / 1e12
    peak = ops / target_s / 1e12
    names = {"llmint8": "gemm_pair_kernel (persistent CTA pairs, tcgen05 cta_group::2 kind::i8 + kind::f16)",
             "fp8": "whole call: activation kernels + gemm_pair_kernel<fp8> (tcgen05 kind::f8f6f4 + kind::f16)",
             "smoothquant": "whole call: smoothing quantize kernel + gemm_pair_kernel (kind::i8, no fp16 part)",
             "stored": "whole call: activation kernels with the column-store gather + gemm_pair_kernel"}
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TOPS",
            "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel or names[wl.variant],
            "peak_source": f"{peaks['source']} bf16_tflops (burst) x 2 for the 8-bit part (nominal ratio), "
                           f"x 1 for the {nO} fp16 outlier columns",
            "frac_of_published": round(achieved / PUBLISHED["int8_tops"], 4),
            "algo_ops_per_launch": int(ops), "int8_ops": int(2 * T * N * (K - nO)), "f16_flops": int(2 * T * N * nO),
            "ms_per_launch": round(kern_ms, 5),
            "how": "one GEMM launch between events after an L2 flush (cold; its ramp-up is not overlapped)",
            **({} if b2b_ms is None else {"back_to_back": {
                "achieved": round(ops / (b2b_ms * 1e-3) / 1e12, 1), "frac": round(ops / (b2b_ms * 1e-3) / 1e12 / peak, 4),
                "ms": round(b2b_ms, 5),
                "how": "the GEMM relaunched 5 times on one workspace after an L2 flush, each launch chained to the "
                       "previous one, events around the five"}})}


def e2e_steps(wl: Workload, steps: int, warmup: int, flush, world: int = 1) -> dict:
    """The public call with host buffers: pinned H2D of X, the matmul, D2H of Y,
    for every call of the step, issued as direct calls (capturing them into a
    CUDA graph measured slower: 1105 against 1174 GB/s, the ten small copies of
    a step dominate either way).  Every rank runs it; the value is all ranks'
    units over the slowest rank's time, and the copy bytes are the whole job's."""
    import torch
    hx = [torch.from_numpy(c["host_X"]).pin_memory() for c in wl.calls]
    hy = [torch.empty(c["Y"].shape, dtype=torch.float16).pin_memory() for c in wl.calls]

    def run():
        for c, x, y in zip(wl.calls, hx, hy):
            c["X"].copy_(x, non_blocking=True)
            wl.call(c)
            y.copy_(c["Y"], non_blocking=True)

    total_ms, _ = time_steps(wl, steps, warmup, world, flush, run=run)
    t_max = reduce_max(total_ms, world)
    units = reduce_sum((wl.bytes_per_step if wl.unit == "GB/s" else wl.ops_per_step) * steps, world)
    value = units / (t_max * 1e-3) / (1e9 if wl.unit == "GB/s" else 1e12)
    h2d = sum(x.numel() * 2 for x in hx) * world
    d2h = sum(y.numel() * 2 for y in hy) * world
    return {"value": round(value, 2), "unit": wl.unit,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(t_max / steps, 5),
            "how": "pinned H2D of X, llmint8 call, D2H of Y for each call of the step, direct calls"}


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(name: str, seed: int = 0, variant: str = "llmint8", tau: float = THRESHOLD, rows=None):
    """Oracle inputs and one step's calls, on a bounded sample of the workload.

    Decode: the full step (five calls).  Prefill: the first `rows` rows of X
    against the full W (detection and scales then cover those rows only).
    Each call is (fn, args, bytes, ops) with fn an oracle function."""
    from oracle import oracle as O
    from oracle import oracle_next as ON
    cfg = synth.WORKLOADS[name]

    def prepare(X, W, tau, dims):
        if variant == "fp8":
            Wq, sw = ON.fp8_quantize_weight(W)
            return ON.fp8_matmul, (X, Wq, sw, W, tau)
        if variant == "smoothquant":
            s = ON.smooth_factors(ON.column_absmax(X), ON.column_absmax(W), 0.5)
            Wq, sw = ON.smooth_quantize_weight(W, s)
            return ON.smoothquant_matmul, (X, s, Wq, sw)
        Wq, sw = O.quantize_weight(W)
        if variant == "stored":
            slot, Wst = ON.make_store(W, np.sort(dims))
            return ON.matmul_stored, (X, Wq, sw, slot, Wst, tau)
        return O.matmul, (X, Wq, sw, W, tau)

    calls = []
    if name == "7b_decode":
        for layer, T in enumerate(DECODE_TS):
            w = synth.workload(name, seed=seed, T=T, layer=layer)
            nO = int(O.compact(O.detect_outliers(w["X"], tau)).size)
            fn, args = prepare(w["X"], w["W"], tau, w["dims"])
            calls.append((fn, args, cfg["N"] * cfg["K"] + 4 * cfg["N"] + 2 * cfg["N"] * nO +
                          2 * T * cfg["K"] + 2 * T * cfg["N"], 2 * T * cfg["N"] * cfg["K"]))
        return calls, "the step's 5 calls, T=1,2,4,8,16, full N and K", "GB/s"
    w = synth.workload(name, seed=seed)
    if rows is None:
        rows = 16 if name == "70b_up" else 32
    rows = min(rows, w["T"])
    Xs = np.ascontiguousarray(w["X"][:rows])
    fn, args = prepare(Xs, w["W"], tau, w["dims"])
    T, N, K = rows, cfg["N"], cfg["K"]
    calls.append((fn, args, 0, 2 * T * N * K))
    what = "tau=%s" % tau if variant != "smoothquant" else "alpha=0.5, factors from these rows"
    return calls, f"first {rows} rows of X against the full W, {what} (ops counted for those rows)", "TOPS"


def shrink_sample(calls, frac: float):
    """The same calls on the first max(1, floor(N * frac)) output rows of W
    (rows of W are independent outputs), with the algorithmic bytes and ops
    counted for those rows.  Works on calls of oracle.matmul (X, Wq, sw, W,
    tau) as oracle_sample builds them."""
    out = []
    for fn, (X, Wq, sw, W, tau), nbytes, ops in calls:
        N, K = Wq.shape
        T = X.shape[0]
        n = max(1, int(N * frac))
        if nbytes:
            n_out = (nbytes - N * K - 4 * N - 2 * T * K - 2 * T * N) // (2 * N)  # |O| of this call
            nbytes = n * K + 4 * n + 2 * n * n_out + 2 * T * K + 2 * T * n
        out.append((fn, (X, Wq[:n], sw[:n], W[:n], tau), nbytes, 2 * T * n * K))
    return out, n


def run_oracle(calls, unit, steps: int, budget_s: float):
    from oracle import oracle as O
    done, t0 = 0, time.perf_counter()
    while done < steps:
        for fn, args, _, _ in calls:
            fn(*args)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    per = sum(c[2] for c in calls) if unit == "GB/s" else sum(c[3] for c in calls)
    value = per * done / dt / (1e9 if unit == "GB/s" else 1e12)
    return value, done, dt, O.num_threads()


def cpu_baseline(name: str, variant: str = "llmint8", tau: float = THRESHOLD, rows=None, budget_s: float = 15.0):
    calls, sample, unit = oracle_sample(name, variant=variant, tau=tau, rows=rows)
    v, done, dt, cores = run_oracle(calls, unit, 1000, budget_s)
    return {"value": round(v, 4), "unit": unit, "cores": cores, "kind": "oracle",
            "sample": sample + f"; {done} steps in {dt:.1f} s"}


# ----------------------------------------------------------------- arms

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    if world > 1:
        # rank 0 works alone: give the oracle every host core, not the one
        # OpenMP thread per rank that the launcher sets by default (torch is
        # loaded already and the oracle shares its OpenMP runtime)
        import torch
        torch.set_num_threads(len(os.sched_getaffinity(0)))
    calls, sample, unit = oracle_sample(args.workload)
    # One step to warm caches and threads and to size the sample: exactly
    # `steps` timed steps (after `warmup` untimed ones) fit in the budget.
    _, _, t1, _ = run_oracle(calls, unit, 1, float("inf"))
    frac = args.ref_budget_s / (t1 * (args.steps + args.warmup))
    if frac < 1.0:
        calls, n = shrink_sample(calls, frac)
        rows_w = f"the first {n} of the {synth.WORKLOADS[args.workload]['N']} rows of W"
        sample = sample.replace("full N and K", f"full K, {rows_w}").replace("the full W", rows_w)
    run_oracle(calls, unit, args.warmup, float("inf"))
    value, done, dt, cores = run_oracle(calls, unit, args.steps, float("inf"))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": unit,
        "n_gpus": args.gpus, "steps": done, "warmup": args.warmup,
        "ms_per_step": round(dt / done * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config(args.workload),
        "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": sample + f"; {done} steps in {dt:.1f} s"},
        "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(name: str) -> dict:
    cfg = synth.WORKLOADS[name]
    d = {"workload": name, "T": list(cfg["T"]) if isinstance(cfg["T"], tuple) else cfg["T"],
         "N": cfg["N"], "K": cfg["K"], "threshold": THRESHOLD if name != "70b_up" else
         list(cfg["thresholds"]), "l2": "flushed before every step (256 MiB write, then 256 MiB read of another buffer)",
         "parallelism": "replicas (one independent problem per GPU)",
         "timing": "step replayed as a CUDA graph; e2e uses direct API calls"}
    if name == "7b_decode":
        d["layers_per_step"] = len(DECODE_TS)
    return d


# (workload, variant, threshold): the entries of "also" at N = 1
ALSO = [("7b_prefill", "llmint8", 6.0), ("13b_up", "llmint8", 6.0), ("70b_up", "llmint8", 6.0),
        ("70b_up", "llmint8", 4.0), ("70b_up", "llmint8", float("inf")),
        ("7b_prefill", "fp8", 6.0), ("13b_up", "fp8", 6.0), ("7b_prefill", "smoothquant", None),
        ("13b_up", "smoothquant", None), ("7b_prefill", "stored", 6.0), ("7b_decode", "fp8", 6.0),
        ("7b_decode", "stored", 6.0)]

# oracle rows timed per prefill entry (about 1-10 s of CPU work each)
ORACLE_ROWS = {"7b_prefill": 256, "13b_up": 128, "70b_up": 16}


def also_entry(name, variant, tau, device, peaks, flush, steps, oracle_budget_s):
    import torch
    taus = None if tau is None else (tau,)
    w2 = Workload(name, device, taus=taus, variant=variant)
    w2.capture()
    ms, ck = time_steps(w2, steps, 3, 1, flush, run=w2.graph.replay)
    status = w2.L.llmint8_sync_status()
    c = w2.calls[0]
    entry = {"workload": name, "variant": variant, "value": round(w2.metric_value(ms * 1e-3, steps), 2),
             "unit": w2.unit, "ms_per_step": round(ms / steps, 4), "n_outliers": c["nO"],
             "threshold": tau, "clocks": ck, "device_status": w2.L.llmint8_status_string(status),
             "resident_weight_bytes": w2.resident_weight_bytes()}
    if variant == "stored":
        entry["store_columns"] = int(c["n_store"])
        entry["misses_last_call"] = int(c["miss"].item())
    if w2.unit == "GB/s":
        cold_ms, cold_algo = time_cold_units(w2, 10, flush)
        entry["roofline"] = decode_roofline(w2, ms / steps, cold_ms, cold_algo, peaks,
                                            traffic=recorded_traffic(traffic_key(name, c["tau"]),
                                                                     main_kernel_name(w2)))
    else:
        km, _ = time_cold_units(w2, 10, flush)
        b2b = time_back_to_back(w2, flush) if variant == "llmint8" else None
        entry["roofline"] = prefill_roofline(w2, km, c, peaks,
                                             traffic=recorded_traffic(traffic_key(name, c["tau"]), main_kernel_name(w2)),
                                             b2b_ms=b2b)
        call_tops = w2.ops_per_step / (ms / steps * 1e-3) / 1e12   # the whole call, graph-replayed
        entry["call_roofline_frac"] = round(call_tops / entry["roofline"]["peak"], 4)
    del w2
    torch.cuda.empty_cache()
    entry["cpu_baseline"] = cpu_baseline(name, variant=variant, tau=THRESHOLD if tau is None else tau,
                                         rows=ORACLE_ROWS.get(name), budget_s=oracle_budget_s)
    return entry


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    from int8_mixed_precision_outlier_b200 import _build
    if rank == 0:
        _build.build()
    barrier(world)
    import int8_mixed_precision_outlier_b200 as L
    L.load_library()
    peaks = load_peaks()
    flush = L2Flush(device)

    wl = Workload(args.workload, device, seed=rank)
    wl.capture()
    total_ms, clocks = time_steps(wl, args.steps, args.warmup, world, flush, run=wl.graph.replay)
    t_max = reduce_max(total_ms, world)
    units = reduce_sum((wl.bytes_per_step if wl.unit == "GB/s" else wl.ops_per_step) * args.steps, world)
    value = units / (t_max * 1e-3) / (1e9 if wl.unit == "GB/s" else 1e12)
    status = L.llmint8_sync_status()
    cold_ms, cold_algo = time_cold_units(wl, 10, flush)
    traffic = recorded_traffic(traffic_key(args.workload, wl.calls[0]["tau"]), main_kernel_name(wl))
    if wl.unit == "GB/s":
        roof = decode_roofline(wl, total_ms / args.steps, cold_ms, cold_algo, peaks, traffic=traffic)
    else:
        b2b = time_back_to_back(wl, flush) if wl.variant == "llmint8" else None
        roof = prefill_roofline(wl, cold_ms, wl.calls[0], peaks, traffic=traffic, b2b_ms=b2b)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": wl.unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": workload_config(args.workload),
        "roofline": roof,
        "gpu_launches": wl.launches_per_step * args.steps,
        "clocks": clocks, "device_status": L.llmint8_status_string(status),
    }
    line["e2e"] = e2e_steps(wl, args.steps, args.warmup, flush, world)  # collective: every rank
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget_s)
    if rank == 0 and world == 1 and args.also:
        del wl
        torch.cuda.empty_cache()
        line["also"] = [also_entry(name, variant, tau, device, peaks, flush, args.also_steps, args.also_cpu_budget_s)
                        for name, variant, tau in ALSO if not (name == args.workload and variant == "llmint8")]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(synth.WORKLOADS), default="7b_decode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", dest="also", action="store_false")
    ap.add_argument("--also-steps", type=int, default=20)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--also-cpu-budget-s", type=float, default=4.0)
    ap.add_argument("--ref-budget-s", type=float, default=120.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == "tiny":
        ap.error("the tiny configuration is a parity case, not a bench workload")
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

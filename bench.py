#!/usr/bin/env python3
"""Benchmark of the QuEST hot path on B200: one step = one pass of the whole path
over one batch of the activation workload.

Step (all kernels of libquest_b200.so, on one CUDA stream):
  1. quest_quantize_fwd   X [16384, 2048] bf16 -> 4-bit codes, trust mask bits,
                          per-128-group scales (the QAT forward quantizer)
  2. quest_trust_bwd      G [16384, 2048] bf16 + that mask -> grad_in bf16
  3. quest_quantize_operands  X and W_up [5632, 2048] -> int8 operand codes, one
                          scale per row (one launch for both operands of the layer)
  4. quest_w4a4_linear    Y [16384, 5632] bf16 = dequant(cX @ cW^T)

Metric: algorithmic GB/s of the whole step (bytes every kernel must move: inputs
read once, outputs written once) and, per part, GB/s as a fraction of the
measured HBM copy bandwidth or int8 TOPS as a fraction of the int8 tensor peak.
Multi-GPU: every rank runs its own full workload (the path shards by rows with
no exchange), weak scaling, time = max over ranks.

``--impl reference`` times the CPU oracle (single-threaded C, fp64) on a bounded
row sample of the same step instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

BITS = 4
HB = 128
R, C = 16384, 2048          # activation / gradient tensors
NW = 5632                   # up-projection width (8/3 * 2048 padded to 256)
L2_FLUSH_BYTES = 256 << 20  # per flush buffer (L2 is 126 MB)
METRIC = "QuEST quantizer GB/s (frac of HBM peak); W4A4 linear TOPS (frac of int8 TC)"
WORKLOAD = ("QuEST hot path on the 16384x2048 bf16 activation workload (Student-t nu=3, "
            "16 outlier channels x20), b=4, Hadamard block 128: quantize_fwd with trust mask "
            "(RMS per 128-group) + trust backward on a 16384x2048 N(0,1e-6) gradient + W4A4 "
            "linear vs the 5632x2048 up-projection (operands quantized with one RMS per row)")


def part_bytes():
    """Algorithmic bytes per step for each kernel (inputs read once, outputs written once)."""
    e = R * C
    return {
        "quantize_fwd": 2 * e + e // 2 + e // 8 + 4 * (e // HB),       # bf16 in, 4-bit codes, mask bits, scales
        "trust_bwd": 2 * e + e // 8 + 2 * e,                           # grad in, mask in, grad out
        "quantize_operands": 3 * e + 4 * R + 3 * NW * C + 4 * NW,      # X and W_up: bf16 in, int8 codes, row scales
        "w4a4_linear": R * C + NW * C + 4 * (R + NW) + 2 * R * NW,     # codes, scales in, bf16 out
    }


GEMM_OPS = 2 * R * NW * C
NOMINAL_HBM_GBS = 8000.0     # nominal B200 HBM3e bandwidth (about 8 TB/s); the roofline peak is the measured copy
NOMINAL_INT8_TOPS = 4500.0   # nominal B200 dense int8 tensor-core rate (used only when the probe is skipped)

# DRAM traffic per launch of the dominant kernel, from one ncu capture of the full
# workload (dram__bytes_read.sum + dram__bytes_write.sum, one pass). Reported only
# while the kernel's source files are byte-identical to the ones that were
# captured; otherwise null.
NCU_TRAFFIC = {
    "w4a4_linear": {"sources": ["bit_quantization_aware_blockwise_b200/csrc/w4a4_gemm.cu",
                                "bit_quantization_aware_blockwise_b200/csrc/tc_common.cuh"],
                    "sha256": "1c75746fed44389d0acabf3c34564f0990dde41d1b696c16a2954f95f582a6c2",
                    "dram_read": 65882752, "dram_write": 146098816},
}


def sources_sha256(paths):
    import hashlib
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(part):
    rec = NCU_TRAFFIC.get(part)
    if rec is None:
        return None
    try:
        if sources_sha256(rec["sources"]) != rec["sha256"]:
            return None
    except OSError:
        return None
    return rec["dram_read"] + rec["dram_write"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, polled from a thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    def __init__(self, torch_device_index, period_s=0.001):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device_index)
            handle = None
            try:
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.nv = pynvml
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of guessing
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def sample_now(self):
        """One synchronous sample from the calling thread (the sampling thread can be
        starved while the launching thread holds the interpreter)."""
        if self.ok:
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception:
                pass

    def start(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        nv = self.nv
        names = {
            "gpu_idle": nv.nvmlClocksEventReasonGpuIdle,
            "applications_clocks_setting": nv.nvmlClocksEventReasonApplicationsClocksSetting,
            "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
            "hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
            "sync_boost": nv.nvmlClocksEventReasonSyncBoost,
            "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
            "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
            "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
        }
        reasons = set()
        for _, rs in self.samples:
            for n, bit in names.items():
                if rs & bit and n != "gpu_idle":
                    reasons.add(n)
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ---------------------------------------------------------------------------
# distributed plumbing (timing only; the data path has no collective)
# ---------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def dist_max(value, world, device="cuda"):
    """Max of a per-rank number over all ranks (timing plumbing, not the data path)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(bytes_per_rank_step, world, ms_max):
    """Whole-job GB/s: the units every rank processed over the slowest rank's time."""
    return bytes_per_rank_step * world / (ms_max * 1e-3) / 1e9


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the B200 arm
# ---------------------------------------------------------------------------
class L2Flush:
    """Evicts L2 between timed steps, outside the timed events: a write of one buffer twice
    the size of L2, then a read of a second one. A step then starts with none of its inputs
    resident and with no dirty line of the flush's own left to be written back inside the
    timed region (a write alone leaves L2 full of dirty lines that the first kernels of
    the step would pay to evict)."""

    describe = (f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, then "
                f"{L2_FLUSH_BYTES >> 20} MiB read of a second buffer; untimed)")

    def __init__(self, dev):
        import torch
        self.torch = torch
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def zero_(self):
        self.w.zero_()
        self.torch.sum(self.r, dim=0, out=self.out)


class Step:
    """Buffers and launches of one step of the hot path (device-resident inputs)."""

    def __init__(self, dev, x, g, w):
        import torch
        import bit_quantization_aware_blockwise_b200 as q
        self.q, self.torch = q, torch
        self.dev = dev
        self.x, self.g, self.w = x, g, w
        e = R * C
        u8 = torch.uint8
        self.codes = torch.empty(q.codes_bytes(R, C, BITS), dtype=u8, device=dev)
        self.scales = torch.empty((R, C // HB), dtype=torch.float32, device=dev)
        self.mask = torch.empty(e // 8, dtype=u8, device=dev)
        self.grad_in = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
        self.cx = torch.empty((R, C), dtype=torch.int8, device=dev)
        self.sx = torch.empty((R, 1), dtype=torch.float32, device=dev)
        self.cw = torch.empty((NW, C), dtype=torch.int8, device=dev)
        self.sw = torch.empty((NW, 1), dtype=torch.float32, device=dev)
        self.y = torch.empty((R, NW), dtype=torch.bfloat16, device=dev)
        self.launches_per_step = 4

    def parts(self, stream):
        """The four launches, each a zero-argument callable (raw C-ABI calls)."""
        q, s = self.q, stream.cuda_stream
        x, g, w = self.x, self.g, self.w
        return [
            ("quantize_fwd", lambda: q.quantize_fwd_raw(
                x.data_ptr(), 0, R, C, C, BITS, HB, HB, 1.0, q.CODES_PACKED, self.codes.data_ptr(),
                self.scales.data_ptr(), q.MASK_BITS, self.mask.data_ptr(), None, 0, s)),
            ("trust_bwd", lambda: q.trust_bwd_raw(
                g.data_ptr(), self.mask.data_ptr(), q.MASK_BITS, R, C, HB, self.grad_in.data_ptr(), s)),
            ("quantize_operands", lambda: q.quantize_operands_raw(
                x.data_ptr(), R, w.data_ptr(), NW, C, q.BF16, BITS, HB, q.CODES_GEMM_OPERAND, self.cx.data_ptr(),
                self.sx.data_ptr(), self.cw.data_ptr(), self.sw.data_ptr(), s)),
            ("w4a4_linear", lambda: q.w4a4_linear_raw(
                self.cx.data_ptr(), self.sx.data_ptr(), self.cw.data_ptr(), self.sw.data_ptr(),
                R, NW, C, self.y.data_ptr(), None, s)),
        ]


def b2b_parts(dev, x, g, w, names=("quantize_fwd", "trust_bwd", "quantize_operands"), nsets=4, n=24):
    """Per-launch time (us) of the HBM-bound parts back to back: one CUDA graph of n
    launches rotating over nsets buffer sets of their own (inputs and outputs), so each
    launch reads inputs that the other sets' traffic (> 2x L2) has evicted, and no launch
    carries the fixed cost a single event-timed launch pays."""
    import torch
    side = torch.cuda.Stream(dev)
    steps = [Step(dev, x.clone(), g.clone(), w.clone()) for _ in range(nsets)]
    out = {}
    torch.cuda.synchronize()
    with torch.cuda.stream(side):   # graph replays run on the current stream: make it the timed one
        for name in names:
            sets = [dict(st.parts(side))[name] for st in steps]
            out[name] = _graph_us(lambda f: f, sets, side, n=n)
    del steps
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_b200(args, world, rank, local):
    import torch
    import bit_quantization_aware_blockwise_b200 as q
    from bit_quantization_aware_blockwise_b200 import inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q.load_library()
    peaks = load_peaks()
    x_cpu = inputs.activation_input()
    g_cpu = inputs.grad_input()
    w_cpu = inputs.weight_up()
    x, g, w = x_cpu.to(dev), g_cpu.to(dev), w_cpu.to(dev)
    step = Step(dev, x, g, w)
    stream = torch.cuda.current_stream(dev)
    parts = step.parts(stream)
    flush = L2Flush(dev)
    names = [n for n, _ in parts]

    def one_step(evs=None):
        for i, (_, f) in enumerate(parts):
            if evs is not None:
                evs[i][0].record(stream)
            f()
            if evs is not None:
                evs[i][1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        one_step()
    torch.cuda.synchronize()
    q.device_status()

    # the timed steps: one CUDA event before the step's first kernel and one after its
    # last, nothing recorded between its kernels (so each kernel's launch may overlap
    # the tail of the one before it)
    span = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    clocks = ClockSampler(local)
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t0 = time.perf_counter()
    every = max(1, args.steps // 8)
    for k in range(args.steps):
        flush.zero_()  # L2 flush between timed steps (outside the per-step events)
        span[k][0].record(stream)
        one_step()
        span[k][1].record(stream)
        if k % every == every - 1:
            clocks.sample_now()   # the queue ahead of the GPU holds this and earlier steps
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    clocks.stop()
    dist_barrier(world)
    q.device_status()
    step_ms = [a.elapsed_time(b) for a, b in span]

    # the per-kernel breakdown: the same steps again with events around every kernel
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            for _ in parts] for _ in range(args.steps)]
    dist_barrier(world)
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()
        one_step(evs[k])
    torch.cuda.synchronize()
    dist_barrier(world)
    q.device_status()
    part_ms = {n: [] for n in names}
    for k in range(args.steps):
        for i, n in enumerate(names):
            part_ms[n].append(evs[k][i][0].elapsed_time(evs[k][i][1]))
    my_ms = sum(step_ms) / args.steps
    ms = dist_max(my_ms, world)
    pbytes = part_bytes()
    step_bytes = sum(pbytes.values())
    value = aggregate_throughput(step_bytes, world, ms)

    hbm = peaks["hbm_gbs"]
    derived_int8 = peaks["bf16_tflops"] * 2.0   # nominal int8 : bf16 dense ratio 4.5 : 2.25
    b2b = b2b_parts(dev, x, g, w)
    # the int8 tensor-core peak: the rate of back-to-back kind::i8 MMAs measured on this
    # part (no memory traffic), else the nominal dense figure
    probe = None if args.no_probe else mma_probe(dev)
    pair_probe = None if args.no_probe else mma_probe(dev, pair=True)
    if probe is not None:
        int8_peak, int8_src = probe["tops"], "measured: back-to-back tcgen05 kind::i8 MMAs, one CTA per SM"
    else:
        int8_peak, int8_src = NOMINAL_INT8_TOPS, "nominal B200 dense int8 (probe skipped)"
    breakdown = {}
    for n in names:
        m = statistics.median(part_ms[n])
        d = {"ms": round(m, 5), "gbs": round(pbytes[n] / (m * 1e-3) / 1e9, 1)}
        d["frac_hbm"] = round(d["gbs"] / hbm, 4)
        d["frac_nominal_8tbs"] = round(d["gbs"] / NOMINAL_HBM_GBS, 4)
        if n in b2b:
            d["us_b2b"] = round(b2b[n], 2)
            d["gbs_b2b"] = round(pbytes[n] / (b2b[n] * 1e-6) / 1e9, 1)
            d["frac_hbm_b2b"] = round(d["gbs_b2b"] / hbm, 4)
        if n == "w4a4_linear":
            d["tops"] = round(GEMM_OPS / (m * 1e-3) / 1e12, 1)
            d["frac_int8_peak"] = round(d["tops"] / int8_peak, 4)
            d["frac_bf16x2"] = round(d["tops"] / derived_int8, 4)
        breakdown[n] = d
    dominant = max(names, key=lambda n: breakdown[n]["ms"])
    avg = {n: sum(part_ms[n]) / len(part_ms[n]) for n in names}
    if dominant == "w4a4_linear":
        achieved = GEMM_OPS / (avg[dominant] * 1e-3) / 1e12
        roofline = {"kernel": "w4a4_gemm_pair_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": round(int8_peak, 1), "unit": "TOPS",
                    "frac": round(achieved / int8_peak, 4),
                    "peak_source": int8_src,
                    "frac_of_bf16x2": round(achieved / derived_int8, 4),
                    "bf16x2_source": f"{peaks['source']} bf16 burst x 2 (nominal int8/bf16 dense ratio)",
                    "traffic": ncu_traffic(dominant), "traffic_unit": "bytes per launch (ncu DRAM read+write)"}
        if pair_probe is not None:
            # context: the same MMAs in the kernel's own instruction form (cta_group::2, M 256)
            roofline["frac_of_pair_probe"] = round(achieved / pair_probe["tops"], 4)
            roofline["pair_probe_tops"] = pair_probe["tops"]
    else:
        achieved = pbytes[dominant] / (avg[dominant] * 1e-3) / 1e9
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "peak_source": peaks["source"], "traffic": ncu_traffic(dominant),
                    "traffic_unit": "bytes per launch (ncu DRAM read+write)"}

    # ---- end to end: pinned host inputs -> device, the step, results -> host
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, dev, step, parts, x_cpu, g_cpu, w_cpu, flush, world)

    if probe is not None:
        probe["gemm_frac_of_probe"] = round(breakdown["w4a4_linear"]["tops"] / probe["tops"], 4)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp32 math on bf16 I/O; int8 x int8 -> int32 tensor cores", "data": "synthetic",
        "config": {"workload": WORKLOAD, "bits": BITS, "had_block": HB,
                   "shapes": {"x": [R, C], "grad": [R, C], "w_up": [NW, C], "y": [R, NW]},
                   "l2": L2Flush.describe,
                   "timing": "per step: one CUDA event on the launching stream before the step's "
                             "first kernel and one after its last (launch gaps included, nothing "
                             "recorded between kernels), mean over the timed steps, max over ranks; "
                             "parts: a second pass with events around every kernel",
                   "parallelism": f"dp{world} (independent row shards, no collective)"},
        "parts": breakdown,
        "parts_note": "ms/gbs/frac_hbm: one launch between CUDA events after an L2 flush (a plain device copy of "
                      "89 MB reaches 0.70 of the measured copy peak this way; an empty launch takes ~6 us); "
                      "*_b2b: per launch of a CUDA graph of 24 launches rotating over 4 buffer sets (> 2x L2)",
        "w4a4_tops": breakdown["w4a4_linear"]["tops"],
        "roofline": roofline,
        "int8_mma_probe": probe,
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "wall_s_timed_loop": round(wall, 4),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)


def mma_probe(dev, gemm_tops=None, iters=20000, reps=5, fp4=False, sparse=False, cp_every=0, bf16=False,
              pair=False):
    """Tensor-core rate with no memory traffic (back-to-back tcgen05.mma, one CTA per
    SM): kind::i8 M 128 N 256 K 32; with fp4 kind::mxf4 M 128 N 256 K 64 with unit
    block scales; with sparse the 2:4-sparse kind::i8 M 128 N 256 K 64 (logical, the
    dense-equivalent rate), metadata resident or copied every cp_every MMAs; context
    for the linear layers' fractions."""
    import statistics
    import torch
    import bit_quantization_aware_blockwise_b200 as q
    stream = torch.cuda.current_stream(dev)
    if sparse:
        launch = lambda n, st: q.probe_mma_sp_i8(n, cp_every, st)
    elif bf16:
        launch = q.probe_mma_bf16
    elif pair:
        launch = q.probe_mma_i8_pair
    else:
        launch = q.probe_mma_fp4 if fp4 else q.probe_mma_i8
    launch(iters, stream.cuda_stream)
    ts, ctas = [], 0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ctas = launch(iters, stream.cuda_stream)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    q.probe_status(stream.cuda_stream)
    ms = statistics.median(ts)
    per_unit = 2.0 * (256 if pair else 128) * 256 * (64 if (fp4 or sparse) else 16 if bf16 else 32)
    tops = per_unit * iters * (ctas // 2 if pair else ctas) / (ms * 1e-3) / 1e12
    out = {"tops": round(tops, 1), "iters": iters, "ctas": ctas,
           "note": "timed alone right after the bench loop (burst); the GEMM's roofline peak"}
    if gemm_tops is not None:
        out["gemm_frac_of_probe"] = round(gemm_tops / tops, 4)
    return out


def run_e2e(args, dev, step, parts, x_cpu, g_cpu, w_cpu, flush, world):
    """End to end through the C ABI: every step copies its three inputs from pinned host
    memory, runs the path and copies its five outputs back to pinned host memory. Steps
    are pipelined over two buffer sets and three streams (upload of step k+1 and download
    of step k-1 overlap the kernels of step k, the two copy directions run concurrently);
    the time per step is the span of all steps over their number."""
    import torch
    xp, gp, wp = x_cpu.pin_memory(), g_cpu.pin_memory(), w_cpu.pin_memory()
    sets = [step, Step(dev, step.x.clone(), step.g.clone(), step.w.clone())]
    outs = [[st.codes, st.scales, st.mask, st.grad_in, st.y] for st in sets]
    host_outs = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs[0]] for _ in sets]
    s_up, s_run, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    launches = [st.parts(s_run) for st in sets]
    n = max(4, min(args.steps, 12))

    def run(nsteps):
        ev_up = [torch.cuda.Event() for _ in range(nsteps)]
        ev_run = [torch.cuda.Event() for _ in range(nsteps)]
        ev_down = [torch.cuda.Event() for _ in range(nsteps)]
        for k in range(nsteps):
            b = k % 2
            with torch.cuda.stream(s_up):
                if k >= 2:
                    s_up.wait_event(ev_run[k - 2])        # set b's inputs were last read by step k-2
                sets[b].x.copy_(xp, non_blocking=True)
                sets[b].g.copy_(gp, non_blocking=True)
                sets[b].w.copy_(wp, non_blocking=True)
                ev_up[k].record(s_up)
            s_run.wait_event(ev_up[k])
            if k >= 2:
                s_run.wait_event(ev_down[k - 2])          # set b's outputs were copied out
            for _, f in launches[b]:
                f()
            ev_run[k].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_run[k])
                for h, o in zip(host_outs[b], outs[b]):
                    h.copy_(o, non_blocking=True)
                ev_down[k].record(s_down)

    run(2)
    torch.cuda.synchronize()
    dist_barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_up)
    run(n)
    t1.record(s_down)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    ms = dist_max(ms, world)
    h2d = sum(t.numel() * t.element_size() for t in (x_cpu, g_cpu, w_cpu))
    d2h = sum(o.numel() * o.element_size() for o in outs[0])
    value = sum(part_bytes().values()) * world / (ms * 1e-3) / 1e9
    return {"value": round(value, 2), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "path": "pinned host -> cudaMemcpyAsync -> quest_* C-ABI calls -> pinned host, "
                    "two buffer sets, upload / kernels / download on three streams"}


# ---------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def oracle_legs(rows_x=256, rows_w=88, gemm_rows=16):
    """Runs the oracle on a bounded row sample of each leg of one step. Returns the seconds
    each leg took and the rows it covered, per leg: the activation legs (quantize, trust
    backward, operand quantize of X) on rows_x rows, the weight operand quantize on rows_w
    rows, and the GEMM (with its dequantisation) on gemm_rows output rows against all
    NW weight rows."""
    import oracle
    from bit_quantization_aware_blockwise_b200 import inputs
    x = inputs.to_f64(inputs.activation_input(rows=rows_x))
    g = inputs.to_f64(inputs.grad_input(rows=rows_x))
    w = inputs.to_f64(inputs.weight_up(rows=rows_w))
    t0 = time.perf_counter()
    o = oracle.quantize(x, bits=BITS, had=HB)
    oracle.trust_bwd(g, o["mask"], had=HB)
    ox = oracle.quantize(x, bits=BITS, had=HB, rms_group=C)
    t1 = time.perf_counter()
    ow = oracle.quantize(w, bits=BITS, had=HB, rms_group=C)
    t2 = time.perf_counter()
    cx = (2 * ox["q"][:gemm_rows] + 1).astype(np.int8)
    cw = (2 * ow["q"] + 1).astype(np.int8)
    # the sampled weight rows' codes tiled to the full width: the cost is the triple loop
    cw_full = np.resize(cw, (NW, C))
    acc = oracle.gemm_i8(cx, cw_full)
    oracle.dequant_linear(acc, ox["scale"][:gemm_rows, 0], np.resize(ow["scale"][:, 0], NW))
    t3 = time.perf_counter()
    return {"act": (t1 - t0, rows_x, R), "weight": (t2 - t1, rows_w, NW), "gemm": (t3 - t2, gemm_rows, R)}


def _sample_text(rows_x, rows_w, gemm_rows, how):
    return (f"oracle on {rows_x} of {R} activation/gradient rows (quantize + trust backward + operand "
            f"quantize), {rows_w} of {NW} weight rows and {gemm_rows} of {R} GEMM output rows "
            f"({gemm_rows}x{NW}x{C}); each leg's time scaled to the full step by its sampled fraction; {how}")


def oracle_step_estimate(rows_x=256, rows_w=88, gemm_rows=16):
    """Seconds of one full step on one core, from a bounded sample of every leg; returns
    (seconds for a full step, bytes of a full step, seconds spent, description)."""
    legs = oracle_legs(rows_x, rows_w, gemm_rows)
    full = sum(t * total / rows for t, rows, total in legs.values())
    spent = sum(t for t, _, _ in legs.values())
    return full, sum(part_bytes().values()), spent, _sample_text(rows_x, rows_w, gemm_rows,
                                                                  "single-threaded C, fp64/int64")


def _oracle_shard(shape):
    legs = oracle_legs(*shape)
    return {k: v[0] for k, v in legs.items()}


def oracle_all_cores(rows_x, rows_w, gemm_rows):
    """The same legs split into row shards over every host core (one spawned process per
    core, the oracle itself unchanged); each leg's rate is n shards over the mean shard
    time. Returns (seconds for a full step, bytes of a full step, wall seconds, cores)."""
    import multiprocessing as mp
    n = max(1, os.cpu_count() or 1)
    shard = (max(1, rows_x // n), max(1, rows_w // n), max(1, gemm_rows // n))
    with mp.get_context("spawn").Pool(n) as pool:
        pool.map(_oracle_shard, [(2, 2, 1)] * n)          # start-up and imports, untimed
        t0 = time.perf_counter()
        res = pool.map(_oracle_shard, [shard] * n)
        wall = time.perf_counter() - t0
    rows = {"act": (shard[0], R), "weight": (shard[1], NW), "gemm": (shard[2], R)}
    full = 0.0
    for k, (r, total) in rows.items():
        t_mean = sum(d[k] for d in res) / n
        full += total / (n * r / t_mean)
    return full, sum(part_bytes().values()), wall, n


def cpu_baseline(args):
    import oracle
    oracle.build()
    # the full activation and weight legs and a 512-row block of the GEMM: about 10-20 s
    # of single-threaded CPU work
    full, nbytes, spent, sample = oracle_step_estimate(rows_x=R, rows_w=NW, gemm_rows=512)
    out = {"value": round(nbytes / full / 1e9, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": sample, "seconds": round(spent, 3), "seconds_per_full_step": round(full, 3)}
    full_n, bytes_n, wall_n, n = oracle_all_cores(R, NW, 512)
    out["all_cores"] = {"value": round(bytes_n / full_n / 1e9, 5), "unit": "GB/s", "cores": n,
                        "seconds": round(wall_n, 3), "seconds_per_full_step": round(full_n, 3),
                        "sample": "the same legs split into row shards, one spawned process per core"}
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    times, nb, sample = [], 0, ""
    if args.warmup > 0:
        oracle_step_estimate(rows_x=64, rows_w=22, gemm_rows=4)
    for _ in range(args.steps):
        full, nb, _, sample = oracle_step_estimate(rows_x=64, rows_w=22, gemm_rows=4)
        times.append(full)
    ms = 1e3 * sum(times) / len(times)
    value = nb / (ms * 1e-3) / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64/int64 (CPU oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "bits": BITS, "had_block": HB,
                   "note": "each step runs a bounded row sample of every leg of the workload and "
                           "scales each leg's time to the full step (ms_per_step is that estimate)"},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def _timed(f, flush, stream, warmup=10, reps=50):
    """Median and p10 (us) of `reps` launches of f, L2 flushed before each (untimed)."""
    import statistics
    import torch
    for _ in range(warmup):
        f()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        f()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    ts.sort()
    return statistics.median(ts), ts[len(ts) // 10]


def _graph_us(make_launch, sets, stream, n=20):
    """One CUDA graph of n launches cycling over `sets` buffer sets; us per launch."""
    import torch
    for k in range(len(sets)):
        make_launch(sets[k])()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            make_launch(sets[i % len(sets)])()
    g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(10):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3 / n)
    del g
    return sorted(ts)[len(ts) // 2]


def run_configs(args):
    """Kernel timings for every workload configuration of the hot path (not the
    bench line): median and p10 of 50 launches after 10 warm-ups, L2 flushed
    before each launch outside the events; the weight tensors also as a CUDA graph
    of 20 launches rotating over 16 buffer sets (> 3x L2)."""
    import torch
    import bit_quantization_aware_blockwise_b200 as q
    from bit_quantization_aware_blockwise_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)     # a non-default stream, so launches can be graph-captured
    torch.cuda.set_stream(stream)
    s = stream.cuda_stream
    peaks = load_peaks()
    flush = L2Flush(dev)
    rows = []

    def add(name, f, nbytes, unit_ops=None, extra=None, bf16=False, fp4=False):
        med, p10 = _timed(f, flush, stream)
        r = {"case": name, "median_us": round(med, 2), "p10_us": round(p10, 2), "bytes": nbytes,
             "gbs": round(nbytes / (med * 1e-6) / 1e9, 1)}
        r["frac_hbm_measured"] = round(r["gbs"] / peaks["hbm_gbs"], 4)
        r["frac_nominal_8tbs"] = round(r["gbs"] / NOMINAL_HBM_GBS, 4)
        if unit_ops and bf16:
            r["tflops"] = round(unit_ops / (med * 1e-6) / 1e12, 1)
            r["frac_bf16_peak"] = round(r["tflops"] / peaks["bf16_tflops"], 4)
        elif unit_ops:
            r["tops"] = round(unit_ops / (med * 1e-6) / 1e12, 1)
            r["frac_int8_peak"] = round(r["tops"] / (peaks["bf16_tflops"] * 2.0), 4)
            if fp4:   # nominal dense FP4 : bf16 ratio 9 : 2.25
                r["frac_fp4_peak"] = round(r["tops"] / (peaks["bf16_tflops"] * 4.0), 4)
        if extra:
            r.update(extra)
        rows.append(r)
        print(json.dumps(r), flush=True)

    def quant(x, bits, rms, code_mode, mask_mode, deq_dtype=None):
        rr, cc = x.shape
        codes = torch.empty(q.codes_bytes(rr, cc, bits, code_mode), dtype=torch.uint8, device=dev)
        scales = torch.empty(rr * (cc // rms), dtype=torch.float32, device=dev)
        mask = torch.empty(q.mask_bytes(rr, cc, mask_mode), dtype=torch.uint8, device=dev) \
            if mask_mode is not None else None
        deq = None
        if deq_dtype is not None:
            deq = torch.empty((rr, cc), dtype=torch.bfloat16 if deq_dtype == q.BF16 else torch.float32,
                              device=dev)
        xd = q.FP32 if x.dtype == torch.float32 else q.BF16
        f = lambda: q.quantize_fwd_raw(
            x.data_ptr(), xd, rr, cc, cc, bits, HB, rms, 1.0, code_mode, codes.data_ptr(), scales.data_ptr(),
            mask_mode if mask_mode is not None else 0, mask.data_ptr() if mask is not None else None,
            deq.data_ptr() if deq is not None else None, deq_dtype if deq is not None else 0, s)
        esz = x.element_size()
        e = rr * cc
        nbytes = esz * e + codes.numel() + (mask.numel() if mask is not None else 0) + 4 * scales.numel() \
            + (deq.numel() * deq.element_size() if deq is not None else 0)
        return f, nbytes, (codes, scales, mask)

    # calibration of the timing method (not paths of the library): an empty launch, and a
    # plain device copy of the byte counts of the weight, activation and twice-activation
    # quantizers (half read, half written)
    z = torch.empty(1, device=dev)
    add("comparison: empty launch (torch fill of one element)", lambda: z.fill_(1.0), 0)
    for mb in (30.6, 89.1, 178.2):
        n = int(mb * 1e6 / 4)
        src = torch.empty(n, dtype=torch.bfloat16, device=dev).normal_()
        dst = torch.empty_like(src)
        add(f"comparison: device copy of {mb} MB (torch copy_, {mb / 2} MB read + written)",
            lambda: dst.copy_(src), 4 * n)
        del src, dst
    # the fp32 256 x 512 N(0,1) tensor: int8 codes, fp32 dequant, byte mask
    x1 = inputs.smoke_input().to(dev)
    f, nb, _ = quant(x1, 4, HB, q.CODES_INT8, q.MASK_BYTES, q.FP32)
    add("quantize fp32 256x512 N(0,1) b4 int8 codes+fp32 deq+byte mask", f, nb)
    # the activations 16384 x 2048
    x2 = inputs.activation_input().to(dev)
    for bits in (1, 2, 3, 4, 8):
        f, nb, _ = quant(x2, bits, HB, q.CODES_PACKED, q.MASK_BITS)
        add(f"quantize activations 16384x2048 b{bits} codes+mask", f, nb)
    f, nb, _ = quant(x2, 4, HB, q.CODES_PACKED, q.MASK_BITS, q.BF16)
    add("quantize activations 16384x2048 b4 codes+mask+bf16 yhat", f, nb)
    # the weights, with the CUDA-graph batch over rotated buffers
    for wname, wt in (("W_up 5632x2048", inputs.weight_up()), ("W_down 2048x5632", inputs.weight_down())):
        w = wt.to(dev)
        for bits in (1, 4):
            f, nb, _ = quant(w, bits, HB, q.CODES_PACKED, q.MASK_BITS)
            sets = [quant(w.clone(), bits, HB, q.CODES_PACKED, q.MASK_BITS)[0] for _ in range(16)]
            g_us = _graph_us(lambda fn: fn, sets, stream)
            add(f"quantize {wname} b{bits} codes+mask", f, nb,
                extra={"graph_us_per_launch": round(g_us, 2),
                       "graph_gbs": round(nb / (g_us * 1e-6) / 1e9, 1)})
            del sets
    # trust backward of the 16384 x 2048 gradient with the activations' b = 4 mask
    fq, _, (codes, scales, mask) = quant(x2, 4, HB, q.CODES_PACKED, q.MASK_BITS)
    fq()
    g = inputs.grad_input().to(dev)
    gi = torch.empty_like(g)
    f = lambda: q.trust_bwd_raw(g.data_ptr(), mask.data_ptr(), q.MASK_BITS, R, C, HB, gi.data_ptr(), s)
    add("trust backward 16384x2048", f, 4 * R * C + R * C // 8)
    # the linear layer's operand codes (one RMS per row) and the layer
    fx, nbx, (cx, sx, _) = quant(x2, 4, C, q.CODES_GEMM_OPERAND, None)
    add("operand quantize X 16384x2048 (row RMS)", fx, nbx)
    w = inputs.weight_up().to(dev)
    fw, nbw, (cw, sw, _) = quant(w, 4, C, q.CODES_GEMM_OPERAND, None)
    add("operand quantize W_up 5632x2048 (row RMS)", fw, nbw)
    fx(); fw()
    y = torch.empty((R, NW), dtype=torch.bfloat16, device=dev)
    f = lambda: q.w4a4_linear_raw(cx.data_ptr(), sx.data_ptr(), cw.data_ptr(), sw.data_ptr(), R, NW, C,
                                  y.data_ptr(), None, s)
    add("W4A4 linear 16384x5632x2048", f, R * C + NW * C + 4 * (R + NW) + 2 * R * NW, unit_ops=GEMM_OPS)
    # the 1-bit path: b = 1 operand codes (c in {-1, +1}) through the same GEMM
    fx1, nbx1, (cx1, sx1, _) = quant(x2, 1, C, q.CODES_GEMM_OPERAND, None)
    fw1, nbw1, (cw1, sw1, _) = quant(w, 1, C, q.CODES_GEMM_OPERAND, None)
    add("W1A1 operand quantize X 16384x2048 b1 (row RMS)", fx1, nbx1)
    fx1(); fw1()
    f = lambda: q.w4a4_linear_raw(cx1.data_ptr(), sx1.data_ptr(), cw1.data_ptr(), sw1.data_ptr(), R, NW, C,
                                  y.data_ptr(), None, s)
    add("W1A1 linear 16384x5632x2048 (+-1 codes)", f, R * C + NW * C + 4 * (R + NW) + 2 * R * NW,
        unit_ops=GEMM_OPS)
    # per-128-group scales on both operands: E4M3 operand codes and the grouped layer
    E4 = q.CODES_GEMM_OPERAND_E4M3
    fxg, nbxg, (cxg, sxg, _) = quant(x2, 4, HB, E4, None)
    fwg, nbwg, (cwg, swg, _) = quant(w, 4, HB, E4, None)
    add("grouped operand quantize X 16384x2048 b4 E4M3 (RMS per 128-group)", fxg, nbxg)
    fxg(); fwg()
    G = C // HB
    f = lambda: q.w4a4_linear_grouped_raw(cxg.data_ptr(), sxg.data_ptr(), cwg.data_ptr(), swg.data_ptr(),
                                          R, NW, C, HB, y.data_ptr(), None, s)
    add("grouped linear 16384x5632x2048 (E4M3 codes, scales per 128-group)", f,
        R * C + NW * C + 4 * G * (R + NW) + 2 * R * NW, unit_ops=GEMM_OPS)
    # the FP4 (E2M1) grid: packed codes + mask per 128-group, int8 c = 2Q operands
    # (one RMS per row) and the same int8 layer on them
    F4, F4OP = q.CODES_FP4_PACKED, q.CODES_FP4_OPERAND
    f, nb, _ = quant(x2, 4, HB, F4, q.MASK_BITS)
    add("FP4 quantize 16384x2048 E2M1 codes+mask (RMS per 128-group)", f, nb)
    fx4, nbx4, (cx4, sx4, _) = quant(x2, 4, C, F4OP, None)
    fw4, nbw4, (cw4, sw4, _) = quant(w, 4, C, F4OP, None)
    add("FP4 operand quantize X 16384x2048 c=2Q (row RMS)", fx4, nbx4)
    add("FP4 operand quantize W_up 5632x2048 c=2Q (row RMS)", fw4, nbw4)
    fx4(); fw4()
    f = lambda: q.w4a4_linear_raw(cx4.data_ptr(), sx4.data_ptr(), cw4.data_ptr(), sw4.data_ptr(), R, NW, C,
                                  y.data_ptr(), None, s)
    add("FP4 linear 16384x5632x2048 (c=2Q codes, int8 tensor cores)", f,
        R * C + NW * C + 4 * (R + NW) + 2 * R * NW, unit_ops=GEMM_OPS)
    # the same layer on the block-scaled FP4 tensor cores: packed E2M1 codes, one RMS per row
    fxp, nbxp, (cxp, sxp, _) = quant(x2, 4, C, F4, None)
    fwp, nbwp, (cwp, swp, _) = quant(w, 4, C, F4, None)
    add("FP4 packed quantize X 16384x2048 E2M1 (row RMS)", fxp, nbxp)
    fxp(); fwp()
    f = lambda: q.fp4_linear_raw(cxp.data_ptr(), sxp.data_ptr(), cwp.data_ptr(), swp.data_ptr(), R, NW, C,
                                 y.data_ptr(), None, s)
    add("FP4 linear 16384x5632x2048 (packed E2M1, block-scaled FP4 tensor cores)", f,
        R * C // 2 + NW * C // 2 + 4 * (R + NW) + 2 * R * NW, unit_ops=GEMM_OPS, fp4=True)
    # the 2:4-sparse format: W_up quantized with pruning (one RMS per row), the layer
    # with the sparse weights on the sparse tensor cores against X's operand codes;
    # TOPS count the logical (dense-equivalent) 2 M N K
    wsp = {"codes": torch.empty((NW, C // 2), dtype=torch.int8, device=dev),
           "meta": torch.empty((NW, C // 8), dtype=torch.uint8, device=dev),
           "scales": torch.empty(NW, dtype=torch.float32, device=dev)}
    f = lambda: q.quantize_sparse24_raw(w.data_ptr(), NW, C, 4, HB, C, 1.0, wsp["codes"].data_ptr(),
                                        wsp["meta"].data_ptr(), wsp["scales"].data_ptr(), None, None, s)
    add("2:4-sparse quantize W_up 5632x2048 b4 (row RMS, survivors + metadata)", f,
        2 * NW * C + NW * C // 2 + NW * C // 8 + 4 * NW)
    f()
    fx(); q.device_status()
    f = lambda: q.w4a4_linear_sparse24_raw(cx.data_ptr(), sx.data_ptr(), wsp["codes"].data_ptr(),
                                           wsp["meta"].data_ptr(), wsp["scales"].data_ptr(), R, NW, C,
                                           y.data_ptr(), None, s)
    add("2:4-sparse W4A4 linear 16384x5632x2048 (sparse tensor cores, logical ops)", f,
        R * C + NW * C // 2 + NW * C // 8 + 4 * (R + NW) + 2 * R * NW, unit_ops=GEMM_OPS)
    # the input gradient of the layer with the trust backward fused into the bf16
    # product: w_hat from the weight quantizer's bf16 dequant, laid out [K, N] by the
    # library's transpose, X's trust mask from the trust backward case above
    fwq, _, _ = quant(w, 4, C, q.CODES_GEMM_OPERAND, None)
    w_hat = torch.empty((NW, C), dtype=torch.bfloat16, device=dev)
    cwq = torch.empty(NW * C, dtype=torch.uint8, device=dev)
    swq = torch.empty(NW, dtype=torch.float32, device=dev)
    q.quantize_fwd_raw(w.data_ptr(), q.BF16, NW, C, C, 4, HB, C, 1.0, q.CODES_GEMM_OPERAND, cwq.data_ptr(),
                       swq.data_ptr(), 0, None, w_hat.data_ptr(), q.BF16, s)
    wt = torch.empty((C, NW), dtype=torch.bfloat16, device=dev)
    f = lambda: q.transpose_bf16_raw(w_hat.data_ptr(), NW, C, wt.data_ptr(), s)
    add("transpose w_hat 5632x2048 bf16 (operand layout of the fused backward)", f, 4 * NW * C)
    f()
    gyl = inputs.layer_output_grad().to(dev)
    gx = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
    f = lambda: q.trust_bwd_linear_raw(gyl.data_ptr(), wt.data_ptr(), mask.data_ptr(), R, NW, C, HB,
                                       gx.data_ptr(), s)
    add("fused input gradient 16384x5632->2048 (bf16 tcgen05, trust backward in the epilogue)", f,
        2 * R * NW + 2 * C * NW + R * C // 8 + 2 * R * C, unit_ops=GEMM_OPS, bf16=True)
    # comparison only (not a path of the library): the same result unfused, torch's
    # cuBLAS bf16 product writing G to HBM, then the trust backward kernel reading it
    G = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
    gx2 = torch.empty_like(gx)

    def unfused():
        torch.matmul(gyl, w_hat, out=G)
        q.trust_bwd_raw(G.data_ptr(), mask.data_ptr(), q.MASK_BITS, R, C, HB, gx2.data_ptr(), s)
    add("comparison: cuBLAS bf16 product then trust backward (unfused, G through HBM)", unfused,
        2 * R * NW + 2 * C * NW + R * C // 8 + 2 * R * C, unit_ops=GEMM_OPS, bf16=True)
    # the QAT forward on dequantised operands: X and W_up quantized with RMS per 128-group
    # and bf16 yhat, then the bf16 layer (the per-group-scaled product on yhat)
    xh = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
    wh = torch.empty((NW, C), dtype=torch.bfloat16, device=dev)
    for src, dst in ((x2, xh), (w, wh)):
        rr = src.shape[0]
        cq = torch.empty(rr * C, dtype=torch.uint8, device=dev)
        sq = torch.empty(rr * (C // HB), dtype=torch.float32, device=dev)
        q.quantize_fwd_raw(src.data_ptr(), q.BF16, rr, C, C, 4, HB, HB, 1.0, q.CODES_INT8, cq.data_ptr(),
                           sq.data_ptr(), 0, None, dst.data_ptr(), q.BF16, s)
    f = lambda: q.linear_bf16_raw(xh.data_ptr(), wh.data_ptr(), R, NW, C, y.data_ptr(), s)
    add("QAT forward linear on bf16 yhat 16384x5632x2048 (RMS per 128-group)", f,
        2 * R * C + 2 * NW * C + 2 * R * NW, unit_ops=GEMM_OPS, bf16=True)
    y2 = torch.empty_like(y)
    f = lambda: torch.matmul(xh, wh.t(), out=y2)
    add("comparison: cuBLAS bf16 product on the same yhat", f, 2 * R * C + 2 * NW * C + 2 * R * NW,
        unit_ops=GEMM_OPS, bf16=True)
    gemm_tops = next(r["tops"] for r in rows if r["case"].startswith("W4A4 linear"))
    q.device_status()
    probe = mma_probe(dev, gemm_tops)
    for r in rows:   # int8 layers against the measured int8 MMA rate too
        if "tops" in r and "frac_fp4_peak" not in r and "tflops" not in r:
            r["frac_int8_probe"] = round(r["tops"] / probe["tops"], 4)
    fp4_tops = next(r["tops"] for r in rows if "block-scaled FP4" in r["case"])
    probe4 = mma_probe(dev, fp4_tops, fp4=True)
    probe4["note"] = "timed alone after the configs; the FP4 layer's fraction stays of 4 x the measured bf16 peak"
    sp_row = next(r for r in rows if r["case"].startswith("2:4-sparse W4A4 linear"))
    probe_sp = mma_probe(dev, sp_row["tops"], sparse=True)
    probe_sp["note"] = "2:4-sparse kind::i8, metadata resident in TMEM, dense-equivalent ops"
    sp_row["frac_sparse_probe"] = probe_sp["gemm_frac_of_probe"]
    probe_sp_cp = mma_probe(dev, None, sparse=True, cp_every=2)
    probe_sp_cp["note"] = "the same with a tcgen05.cp of metadata before every second MMA"
    probe_pair = mma_probe(dev, gemm_tops, pair=True)
    probe_pair["note"] = "cta_group::2 kind::i8 (M 256 per CTA pair), the instruction form of the int8 layers"
    probe_bf = mma_probe(dev, None, bf16=True)
    probe_bf["note"] = "kind::f16 bf16, measured the same way: the denominator for cuBLAS and the f3 kernels"
    for r in rows:
        if "tflops" in r:
            r["frac_bf16_probe"] = round(r["tflops"] / probe_bf["tops"], 4)
    print(json.dumps({"configs": rows, "int8_mma_probe": probe, "fp4_mma_probe": probe4,
                      "sparse_mma_probe": probe_sp, "sparse_mma_probe_cp2": probe_sp_cp,
                      "int8_pair_mma_probe": probe_pair, "bf16_mma_probe": probe_bf, "peaks": peaks}), flush=True)


def run_profile_kernels(args):
    """One launch of every kernel on a case sized for an ncu capture: inputs larger
    than L2 (32768 x 2048 bf16 = 134 MB) but a few hundred MB in all."""
    import torch
    import bit_quantization_aware_blockwise_b200 as q
    from bit_quantization_aware_blockwise_b200 import inputs
    rows = args.profile_rows
    dev = torch.device("cuda", 0)
    x = inputs.activations(rows, C, seed=1).to(dev)
    g = inputs.upstream_grad(rows, C, seed=4).to(dev)
    a = torch.from_numpy(inputs.gemm_codes(4096, C, seed=31)).to(dev)
    b = torch.from_numpy(inputs.gemm_codes(NW, C, seed=32)).to(dev)
    sa = torch.from_numpy(inputs.positive_scales(4096, 33)).to(dev)
    sb = torch.from_numpy(inputs.positive_scales(NW, 34)).to(dev)
    torch.cuda.synchronize()
    out = q.quantize_fwd(x, BITS, mask_mode=q.MASK_BITS)                               # 1
    gi = q.trust_bwd(g, out["mask"])                                                   # 2
    w_up = inputs.weight_up().to(dev)
    op, _ = q.quantize_operands(x, w_up, BITS, HB, q.CODES_GEMM_OPERAND)                 # 3
    y = q.w4a4_linear(a, sa, b, sb)                                                    # 4
    a8, b8 = a.float().to(torch.float8_e4m3fn), b.float().to(torch.float8_e4m3fn)
    sag = sa[:, None].repeat(1, C // HB).contiguous()
    sbg = sb[:, None].repeat(1, C // HB).contiguous()
    yg = q.w4a4_linear_grouped(a8, sag, b8, sbg)                                       # 5
    f4 = q.quantize_fwd(x, 4, code_mode=q.CODES_FP4_PACKED, mask_mode=q.MASK_BITS)    # 6
    gyl = inputs.upstream_grad(8192, NW, seed=5).to(dev)
    wt = q.transpose_bf16(inputs.weight_up().to(dev))                                  # 7
    gx = q.trust_bwd_linear(gyl, wt, out["mask"][: 8192 * C // 8])                     # 8
    yf = q.linear_bf16(x[:8192], w_up)                                                 # 9
    pa4 = torch.from_numpy(inputs.fp4_codes(8192, 2048, seed=35)).to(dev)
    pw4 = torch.from_numpy(inputs.fp4_codes(NW, 2048, seed=36)).to(dev)
    y4 = q.fp4_linear(pa4, sa.repeat(2), pw4, sb, 2048)                                # 10
    wsp = q.quantize_sparse24(w_up, 4, rms_group=C, mask=False)                        # 11
    ysp = q.w4a4_linear_sparse24(a, sa, wsp["codes"], wsp["meta"], wsp["scales"])      # 12
    torch.cuda.synchronize()
    q.device_status()
    print(json.dumps({"profile_kernels": "ok", "rows": rows, "checksum": [
        float(out["scales"].sum()), float(gi.float().abs().sum()), float(op["scales"].sum()),
        float(y.float().abs().sum()), float(yg.float().abs().sum()), float(f4["scales"].sum()),
        float(gx.float().abs().sum()), float(yf.float().abs().sum()), float(y4.float().abs().sum()),
        float(ysp.float().abs().sum())]}))


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 1000 for the B200 arm, 20 for the CPU oracle arm)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-kernels", action="store_true",
                    help="launch each kernel once on an ncu-sized case and exit")
    ap.add_argument("--profile-rows", type=int, default=32768)
    ap.add_argument("--no-probe", action="store_true", help="skip the int8 tensor-core peak probe")
    ap.add_argument("--configs", action="store_true",
                    help="time every workload configuration (median / p10 per kernel) and exit")
    args = ap.parse_args()
    if args.steps is None:
        # the oracle arm samples each step on the host cores (about half a second a step)
        args.steps = 1000 if args.impl == "b200" else 20
    if args.profile_kernels:
        run_profile_kernels(args)
        return
    if args.configs:
        run_configs(args)
        return
    if args.warmup < 3 and args.impl == "b200":
        args.warmup = 3
    world, rank, local = (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                          int(os.environ.get("LOCAL_RANK", "0")))
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_b200(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of per-token-group activation quantization on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pqg_quant call over the workload: load, optional SiLU-and-mul,
group absmax, scale, quantize and scale store, all in one kernel.  The default
workload is the flat quantization of a DeepSeek-V3 hidden state: bf16
[8192, 7168] with outliers and all-zero groups, G = 128, E4M3 codes and UE8M0
scales in the packed column-major layout.  Inputs are synthetic and seeded.
They are resident in HBM before timing starts, and several buffer sets rotate so
that each step's buffers have left the 126 MB L2 before they are reused.

Timing: each sample times exactly K steps with CUDA events on the launching
stream, between a barrier and a synchronize on both sides; the K launches are
queued behind a short device-side sleep issued before the start event, so the
host's launch cost stays outside the interval.  At least 10 samples and about
100 ms of timed work are taken; ``value`` comes from the median sample (the
slowest rank's, sample by sample), with the fastest and slowest beside it.

Rank 0 prints one JSON line.  ``value`` is effective HBM GB/s: the algorithmic
bytes (input read, codes and scales written) of all ranks' steps divided by the
slowest rank's device time.  Under torchrun each rank runs an independent
replica on its own GPU (weak scaling, no data-path collective).  NCCL is only
used for the barrier and the max over ranks of the timed interval.

``--impl reference`` times the CPU oracle on bounded samples of the same
workload instead, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "per-token-group quant effective HBM GB/s (% of 8 TB/s) and µs/call at M=1"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def workloads():
    from precision_activation_quantization_b200 import inputs
    return {
        "flat_hidden": lambda: inputs.flat_hidden(),
        "flat_hidden_fp32": lambda: inputs.flat_hidden(layout="row", scale_fmt="fp32").with_(
            name="flat_8192x7168_fp32_row"),
        "per_token": lambda: inputs.flat_hidden(layout="row", scale_fmt="fp32").with_(
            group=7168, name="per_token_8192x7168"),
        "mxfp4": lambda: inputs.mxfp4(),
        "nvfp4": lambda: inputs.nvfp4(),
        "fused": lambda: inputs.fused(),
        "fused_7168": lambda: inputs.fused(M=4096, K=7168),
        "masked": lambda: inputs.masked(),
        "masked_decode": lambda: inputs.masked(decode=True),
        "varlen": lambda: inputs.varlen(),
        "sweep_65536_bf16_e4m3_g128": lambda: inputs.sweep(65536),
        "sweep_65536_fp16_int8_g32": lambda: inputs.sweep(65536, in_dtype="fp16",
                                                          out_dtype="int8", group=32),
    }


def describe(w) -> dict:
    shape = [w.E, w.M, 2 * w.K if w.fused else w.K] if w.E > 1 else \
        [w.M, 2 * w.K if w.fused else w.K]
    d = {"workload": w.name, "input_shape": shape, "in_dtype": w.in_dtype,
         "out_dtype": w.out_dtype, "group": w.group,
         "scales": f"{w.scale_fmt} {dict(row='row-major', col='column-major TMA-aligned', packed='UE8M0-packed column-major', tile128x4='128x4 tiled')[w.layout]}",
         "fused_silu_mul": w.fused, "rows_quantized": w.rows,
         "algorithmic_bytes_per_step": w.algorithmic_bytes()}
    if w.masked_m is not None:
        d["masked"] = {"experts": w.E, "M_max": w.M, "sum_masked_m": w.rows,
                       "expected_m": w.expected_m}
    if w.global_scale is not None:
        d["global_scale"] = w.global_scale
    if w.seg_indptr is not None:
        d["varlen"] = {"segments": w.segments, "packed_rows": w.M, "tokens": w.rows,
                       "segment_alignment_rows": 128, "expected_m": w.expected_m}
    return d


def make_call(w, dev, M=None):
    """The C entry point for ``w`` with every argument but the buffers bound:
    call(in_ptr, out_ptr, scales_ptr, stream_handle) -> status.  NVFP4 goes
    through pqg_quant_nvfp4 with its global scale in device memory."""
    import torch
    from precision_activation_quantization_b200 import pqg
    M = w.M if M is None else M
    E = w.E if M == w.M else 1
    if w.seg_indptr is not None:
        # varlen: the workload's segments, or one segment of all M rows
        full = M == w.M
        ip = torch.from_numpy(np.asarray(w.seg_indptr if full else [0, M], np.int32)).to(dev)
        ln = (torch.from_numpy(np.asarray(w.seg_lens, np.int32)).to(dev)
              if full and w.seg_lens is not None else None)
        n_seg, em = ip.numel() - 1, (w.expected_m if full else 0)

        def call(a, b, c, sh):
            return pqg.pqg_quant_varlen(a, b, c, None, M, n_seg, w.K, w.group,
                                        pqg.IN_DTYPES[w.in_dtype], pqg.OUT_DTYPES[w.out_dtype],
                                        pqg.SCALE_FMTS[w.scale_fmt], pqg.LAYOUTS[w.layout],
                                        int(w.fused), ip.data_ptr(),
                                        None if ln is None else ln.data_ptr(), em, sh)
        call.keep = (ip, ln)
        return call
    mm = None if (w.masked_m is None or E == 1 and M != w.M) else \
        torch.from_numpy(w.masked_m).to(dev)
    mm_ptr = None if mm is None else mm.data_ptr()
    em = w.expected_m if mm is not None else 0
    if w.scale_fmt == "e4m3":
        gsc = torch.tensor([w.global_scale], dtype=torch.float32, device=dev)

        def call(a, b, c, sh):
            return pqg.pqg_quant_nvfp4(a, b, c, gsc.data_ptr(), M, E, w.K,
                                       pqg.IN_DTYPES[w.in_dtype], pqg.LAYOUTS[w.layout],
                                       int(w.fused), mm_ptr, em, sh)
        call.keep = (gsc, mm)
        return call

    def call(a, b, c, sh):
        return pqg.pqg_quant(a, b, c, M, E, w.K, w.group, pqg.IN_DTYPES[w.in_dtype],
                             pqg.OUT_DTYPES[w.out_dtype], pqg.SCALE_FMTS[w.scale_fmt],
                             pqg.LAYOUTS[w.layout], int(w.fused), mm_ptr, em, sh)
    call.keep = (mm,)
    return call


def kernel_of(w) -> str:
    """Which kernel a workload runs: "row" (per-token, G = K) or "strip"."""
    return "row" if w.group == w.K and w.group not in (16, 32, 64, 128) else "strip"


_C_TOKENS = re.compile(r'("(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\')|//[^\n]*|/\*.*?\*/',
                       re.DOTALL)


def code_only(text: str) -> str:
    """C/C++ source without its comments, blank lines and trailing blanks
    (string and character literals kept), so that editing a comment leaves the
    digest below unchanged."""
    text = _C_TOKENS.sub(lambda m: m.group(1) or "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def source_digest(kernel: str = "strip") -> str:
    """sha256 over the code of the CUDA sources a kernel is built from (the
    strip kernel does not include the per-token row kernel's file), to tell
    whether stored ncu counters still apply."""
    csrc = os.path.join(ROOT, "precision_activation_quantization_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(csrc)):
        if kernel == "strip" and f == "pqg_row_kernel.cuh":
            continue
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + code_only(fh.read()).encode())
    return h.hexdigest()


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def stored_traffic(name: str, kernel: str = "strip"):
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get(name)
        if rec and rec.get("source_sha256") == source_digest(kernel):
            return rec["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def max_over_ranks(value: float, device, world: int) -> float:
    """The largest ``value`` over all ranks (the slowest rank's time)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def max_over_ranks_all(values, device, world: int):
    """Element-wise max over ranks of a list of per-sample times."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(bytes_per_step: int, steps: int, ms: float, world: int) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's interval."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


# --------------------------------------------------------------------------
# Clock sampling (NVML, polled during the timed region)
# --------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nvml = pynvml
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        n = self._nvml
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                r = get_reasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "NVML polled every ~2 ms during the timed region"}


# --------------------------------------------------------------------------
# The reference arm: the CPU oracle
# --------------------------------------------------------------------------

def run_reference(args, w) -> dict:
    import concurrent.futures as cf
    cores = os.cpu_count() or 1
    rows = min(64, w.M)
    blocks = _oracle_blocks(w, rows)
    per_step = cores                     # one 64-row block per core per step

    def step(i, ex):
        chunk = [blocks[(i * per_step + k) % len(blocks)] for k in range(per_step)]
        return sum(ex.map(lambda b: _oracle_block(w, b), chunk)), sum(b[2] for b in chunk)

    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        for i in range(args.warmup):
            step(i, ex)
        total_bytes = total_rows = 0
        t0 = time.perf_counter()
        for i in range(args.steps):
            b, n = step(args.warmup + i, ex)
            total_bytes += b
            total_rows += n
        dt = time.perf_counter() - t0
    gbs = total_bytes / dt / 1e9
    sample = (f"{per_step} blocks of {rows} rows of {w.name} per step (cycled), one per host "
              f"thread, oracle C at -O2 as it stands")
    return {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": describe(w), "tokens_per_s": total_rows / dt,
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _oracle_blocks(w, rows: int):
    """(expert, first row, rows) blocks covering the workload's live rows."""
    if w.seg_indptr is not None:
        # varlen: the token rows of each (well-formed) segment of the one buffer
        lens = (np.diff(w.seg_indptr) if w.seg_lens is None else w.seg_lens)
        return [(0, int(w.seg_indptr[e]) + m0, min(rows, int(lens[e]) - m0))
                for e in range(w.segments) for m0 in range(0, int(lens[e]), rows)]
    live = [w.M if w.masked_m is None else int(np.clip(w.masked_m[e], 0, w.M))
            for e in range(w.E)]
    return [(e, m0, min(rows, live[e] - m0)) for e in range(w.E)
            for m0 in range(0, live[e], rows)]


def _oracle_block(w, blk):
    """Run the oracle, as it stands, on one block of rows; returns its bytes."""
    import oracle
    e, m0, n = blk
    sub = w.with_(x=w.x[e:e + 1, m0:m0 + n], M=n, E=1, masked_m=None, seg_indptr=None,
                  seg_lens=None)
    oracle.quant(sub.x, M=n, K=w.K, group=w.group, in_dtype=w.in_dtype, out_dtype=w.out_dtype,
                 scale_fmt=w.scale_fmt, layout=w.layout, fused=w.fused,
                 global_scale=w.global_scale)
    return sub.algorithmic_bytes()


def cpu_baseline(w, budget_s: float = 10.0) -> dict:
    """The oracle as it stands on the whole workload (masked: the live rows only):
    row blocks spread over every host core (the C oracle releases the GIL), then
    one thread, each for about ``budget_s`` seconds."""
    import concurrent.futures as cf
    cores = os.cpu_count() or 1
    blocks = _oracle_blocks(w, max(1, -(-w.M // (4 * cores))))

    def timed(workers):
        reps, t0 = 0, time.perf_counter()
        with cf.ThreadPoolExecutor(max_workers=workers) as ex:
            while True:
                list(ex.map(lambda b: _oracle_block(w, b), blocks))
                reps += 1
                dt = time.perf_counter() - t0
                if dt >= budget_s or reps >= 50:
                    return reps * w.algorithmic_bytes() / dt / 1e9, reps, dt

    par, reps_p, dt_p = timed(cores)
    one, reps_1, dt_1 = timed(1)
    return {"value": par, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"the whole {w.name} workload in {len(blocks)} row blocks over {cores} "
                      f"thread(s), {reps_p} time(s) in {dt_p:.1f} s",
            "single_thread": {"value": one, "unit": "GB/s", "cores": 1,
                              "sample": f"the same blocks on one thread, {reps_1} time(s) "
                                        f"in {dt_1:.1f} s"}}


# --------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------

def run_ours(args, w, rank: int, world: int, local_rank: int) -> dict | None:
    import torch
    import torch.distributed as dist
    from precision_activation_quantization_b200 import pqg

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    dt = torch.float16 if w.in_dtype == "fp16" else torch.bfloat16
    x0 = torch.from_numpy(np.ascontiguousarray(w.x).view(np.int16)).view(dt).to(dev)
    nbytes = pqg.pqg_scales_bytes(w.E, w.M, w.K, w.group, pqg.SCALE_FMTS[w.scale_fmt],
                                  pqg.LAYOUTS[w.layout])
    n_out = w.E * w.M * (w.K // 2 if w.out_dtype == "e2m1" else w.K)
    footprint = x0.numel() * 2 + n_out + nbytes
    sets = max(1, min(8, -(-4 * L2_BYTES // footprint)))
    xs = [x0] + [x0.clone() for _ in range(sets - 1)]
    outs = [torch.empty(n_out, dtype=torch.uint8, device=dev) for _ in range(sets)]
    scs = [torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev) for _ in range(sets)]
    call = make_call(w, dev)
    ptrs = [(xs[i].data_ptr(), outs[i].data_ptr(), scs[i].data_ptr()) for i in range(sets)]

    def launch(i):
        a, b, c = ptrs[i % sets]
        st = call(a, b, c, sh)
        if st != pqg.PQG_OK:
            raise pqg.PqgError(st)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    graph = None
    if args.graph:
        # the K timed steps captured once as a CUDA graph (host launch cost out
        # of the timed region); warm-up steps run eagerly before capture
        stream = torch.cuda.Stream(dev)
        sh = stream.cuda_stream
    t_host = time.perf_counter()
    for i in range(args.warmup):
        launch(i)
    host_us = (time.perf_counter() - t_host) * 1e6 / max(args.warmup, 1)
    if args.graph:
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        captured0 = pqg.pqg_launch_count()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(args.steps):
                launch(args.warmup + i)
        captured = pqg.pqg_launch_count() - captured0
    # Each sample times exactly K steps between a barrier + synchronize on
    # both sides.  Stream launches are queued behind a short device-side sleep
    # issued before the start event, so that the host's launch cost is not
    # inside the timed interval (the sleep covers the time the host needs to
    # queue the K launches).
    sleep_cycles = int(min(1.5 * args.steps * host_us + 20.0, 50e3) * 2e3)   # ~2 GHz

    def sample():
        barrier()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            if graph is None:
                torch.cuda._sleep(sleep_cycles)
            start.record(stream)
            if graph is not None:
                # replay on the capture stream, where the events are recorded
                graph.replay()
            else:
                for i in range(args.steps):
                    launch(args.warmup + i)
            end.record(stream)
        end.synchronize()
        barrier()
        return start.elapsed_time(end)

    launches0 = pqg.pqg_launch_count()
    with ClockSampler(dev.index) as clocks:
        first = max_over_ranks(sample(), dev, world)
        # at least 10 samples and at least ~100 ms of timed GPU work in total
        n_samples = args.samples or int(min(max(10, -(-100.0 // max(first, 1e-3))), 2000))
        times = [sample() for _ in range(n_samples - 1)]
    launches = (captured if graph is not None
                else (pqg.pqg_launch_count() - launches0) // n_samples)
    del graph
    per_sample = max_over_ranks_all([first] + times, dev, world)
    ms = statistics.median(per_sample)
    ms_step = ms / args.steps
    bytes_step = w.algorithmic_bytes()
    value = job_throughput(bytes_step, args.steps, ms, world)
    timing = {"samples": n_samples, "steps_per_sample": args.steps,
              "ms_per_sample": {"median": ms, "min": min(per_sample), "max": max(per_sample)},
              "value_min": job_throughput(bytes_step, args.steps, max(per_sample), world),
              "value_max": job_throughput(bytes_step, args.steps, min(per_sample), world),
              "method": ("each sample is the K timed steps between a barrier + synchronize on "
                         "both sides, timed with CUDA events on the launching stream "
                         + ("(one CUDA-graph replay)" if args.graph else
                            "(launches queued behind a device-side sleep issued before the "
                            "start event)")
                         + "; value = median sample, max over ranks per sample")}

    lat = e2e = None
    if not args.kernel_only:
        # latency at M = 1 (same configuration, one row)
        lat = latency_m1(w, dev) if rank == 0 else None
        # end to end: pinned host input -> device -> quantize -> codes/scales back
        e2e = end_to_end(args, w, dev, stream, x0, outs[0], scs[0], call, world)
    small_m = (latency_table(dev) if rank == 0 and w.name.startswith("sweep")
               and not args.kernel_only else None)

    del xs, outs, scs
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    peak, peak_src = hbm_peak()
    achieved = bytes_step / (ms_step * 1e-3) / 1e9
    traffic = stored_traffic(w.name, kernel_of(w))
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": dict(describe(w), launch="cuda-graph replay" if args.graph else "stream",
                       l2=f"{sets} rotating buffer sets ({sets * footprint / 1e6:.0f} MB "
                                       f"> 4 x 126 MB L2); each step reads a set last used "
                                       f"{sets - 1} steps earlier",
                       parallelism=f"{world} independent replica(s), no data-path collective"),
        "pct_of_8tbs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "tokens_per_s": world * w.rows * args.steps / (ms * 1e-3),
        "us_per_call_m1": lat,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": traffic,
                     "algorithmic_bytes_per_launch": bytes_step,
                     "kernel": ("pqg::row_quant_kernel" if kernel_of(w) == "row"
                                else "pqg::quant_kernel") + " (one launch per step)"},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "timing": timing,
    }
    if w.name.startswith("sweep") and not args.kernel_only:
        line["us_per_call_small_m"] = {
            "K": 4096, "scales": "fp32 row-major", "rows": small_m,
            "note": "graph = 200 launches in a CUDA graph, device time per call; stream = 200 "
                    "back-to-back launches from Python"}
    if world == 1 and not args.no_cpu_baseline and not args.kernel_only:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def latency(w, dev, M: int = 1) -> dict:
    """µs per call of ``w``'s variant on M rows: CUDA-graph replays (device time
    per call) and back-to-back stream launches from Python."""
    import torch
    from precision_activation_quantization_b200 import pqg
    width = 2 * w.K if w.fused else w.K
    x = torch.zeros((M, width), dtype=torch.bfloat16 if w.in_dtype == "bf16" else torch.float16,
                    device=dev)
    x.normal_()
    out = torch.empty(M * (w.K // 2 if w.out_dtype == "e2m1" else w.K), dtype=torch.uint8,
                      device=dev)
    nb = pqg.pqg_scales_bytes(1, M, w.K, w.group, pqg.SCALE_FMTS[w.scale_fmt],
                              pqg.LAYOUTS[w.layout])
    sc = torch.empty(nb, dtype=torch.uint8, device=dev)
    call = make_call(w, dev, M=M)
    a = (x.data_ptr(), out.data_ptr(), sc.data_ptr())
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for _ in range(10):
            call(*a, s.cuda_stream)
        n = 200
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(n):
                call(*a, s.cuda_stream)
        g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
        e1.synchronize()
        graph_us = e0.elapsed_time(e1) * 1e3 / (reps * n)
        e0.record(s)
        for _ in range(n):
            call(*a, s.cuda_stream)
        e1.record(s)
        e1.synchronize()
        stream_us = e0.elapsed_time(e1) * 1e3 / n
    del g
    return {"graph": graph_us, "stream": stream_us}


def latency_m1(w, dev) -> dict:
    """µs per call at M = 1 (one row of the workload's shape and variant)."""
    return dict(latency(w, dev, 1),
                note="1 x K row, same variant; graph = 200 launches captured in a CUDA graph "
                     "(device time per call); stream = 200 back-to-back launches from Python")


SMALL_M = (1, 16, 128, 1024)


def latency_table(dev) -> list:
    """µs per call of the dtype/size sweep's variants (bf16 and fp16, G = 32, 64
    and 128, INT8 and E4M3 codes with fp32 row-major scales, K = 4096) at the
    small row counts, where a call is latency-bound."""
    from precision_activation_quantization_b200 import inputs
    rows = []
    for in_dtype in ("bf16", "fp16"):
        for G in (32, 64, 128):
            for out_dtype in ("int8", "e4m3"):
                w = inputs.sweep(1, in_dtype=in_dtype, group=G, out_dtype=out_dtype)
                for M in SMALL_M:
                    rows.append(dict(in_dtype=in_dtype, group=G, out_dtype=out_dtype, M=M,
                                     **latency(w, dev, M)))
    return rows


def end_to_end(args, w, dev, stream, x_dev, out_dev, sc_dev, call, world) -> dict:
    """Same metric through the public API with host buffers: every step copies its
    input from pinned host memory, quantizes, and reads codes and scales back.

    Steps are pipelined the way a caller with host buffers would run them: the
    input copy of step i+1 (its own stream) overlaps the kernel and the output
    copy of step i (two more streams) over two device buffer sets; events order
    each buffer's reuse.  The timed region runs from the first input copy to
    the last output copy."""
    import torch
    import torch.distributed as dist
    from precision_activation_quantization_b200 import pqg
    x_host = torch.from_numpy(np.ascontiguousarray(w.x).view(np.int16)).view(x_dev.dtype)
    x_host = x_host.reshape(x_dev.shape).pin_memory()
    xs = [x_dev, torch.empty_like(x_dev)]
    outs = [out_dev, torch.empty_like(out_dev)]
    scs = [sc_dev, torch.empty_like(sc_dev)]
    out_hosts = [torch.empty(out_dev.shape, dtype=torch.uint8).pin_memory() for _ in range(2)]
    sc_hosts = [torch.empty(sc_dev.shape, dtype=torch.uint8).pin_memory() for _ in range(2)]
    steps = max(1, min(args.steps, 50))
    s_in, s_k, s_out = torch.cuda.Stream(dev), stream, torch.cuda.Stream(dev)

    def run(n):
        ev_k = [None] * n
        ev_out = [None] * n
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_k[i - 2])           # the kernel of step i-2 read xs[j]
                xs[j].copy_(x_host, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            s_k.wait_event(ev_in)
            if i >= 2:
                s_k.wait_event(ev_out[i - 2])              # outs[j] of step i-2 was read back
            st = call(xs[j].data_ptr(), outs[j].data_ptr(), scs[j].data_ptr(), s_k.cuda_stream)
            if st != pqg.PQG_OK:
                raise pqg.PqgError(st)
            ev_k[i] = torch.cuda.Event()
            ev_k[i].record(s_k)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_k[i])
                out_hosts[j].copy_(outs[j], non_blocking=True)
                sc_hosts[j].copy_(scs[j], non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(s_out)
        return ev_out[-1]

    run(2)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_k.wait_event(e0)
    s_out.wait_event(e0)
    last = run(steps)
    s_out.wait_event(last)
    e1.record(s_out)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), dev, world)
    return {"value": job_throughput(w.algorithmic_bytes(), steps, ms, world), "unit": "GB/s",
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": out_hosts[0].numel() + sc_hosts[0].numel(),
            "steps": steps, "ms_per_step": ms / steps,
            "pipeline": "input copy, kernel and output copy on three streams over two "
                        "device buffer sets"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="flat_hidden", choices=sorted(workloads()))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--samples", type=int, default=0,
                    help="timed samples of K steps each (default: at least 10 and ~100 ms)")
    ap.add_argument("--graph", action="store_true",
                    help="replay the K timed steps from one CUDA graph (launch-bound workloads)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the kernel loop only (no M=1 latency, e2e or CPU baseline); "
                         "used for profiler captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        w = workloads()[args.workload]()
        print(json.dumps(run_reference(args, w)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        w = workloads()[args.workload]()
        line = run_ours(args, w, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

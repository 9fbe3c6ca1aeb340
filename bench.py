#!/usr/bin/env python
"""Decode-attention throughput of libcalibq on synthetic InternVL-2.5-shaped
visual KV caches (1-bit CalibQuant: post-scaled, calibrated GQA attention over
packed codes).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--bits B] [--path octet|canonical]

One step = one decode-attention call (one layer) over a batch whose cache was
quantized beforehand (cache fill, timed separately and reported as
"cache_fill"). Prints ONE JSON line on rank 0. Multi-GPU runs (torchrun) give
every rank its own batch (weak scaling, no collective on the data path); the
step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch
from threadpoolctl import threadpool_limits

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_attention_cq_b200 import calibq as cq  # noqa: E402
from decode_attention_cq_b200 import synth  # noqa: E402

METRIC = "1-bit decode-attention tokens/s and achieved HBM GB/s (n=8192), % of roofline"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
FALLBACK_HBM_GBS = 6650.0
CALIB = (True, 0.8, 0.9)
KERNEL_SOURCES = {"k_decode_tc": "decode_tc.cu", "k_decode_row": "decode_row.cu", "k_decode_mma": "decode_mma.cu",
                  "k_decode_octet": "decode_octet.cu", "k_decode_ring": "decode_ring.cu",
                  "k_scores + k_softmax_v + k_merge": "decode_generic.cu"}


def decode_kernel_source(kernel: str) -> str:
    """Source file of a decode kernel named by cq_decode_kernel_name."""
    return "decode_attention_cq_b200/csrc/" + KERNEL_SOURCES[kernel]


def algorithmic_bytes(B, Hq, Hkv, n, d, bits, dsize=2):
    """Bytes one decode step must move at least: K and V codes, per-channel
    alpha/step of K and V, the queries and the output."""
    codes = 2 * B * Hkv * n * d * bits // 8
    stats = 4 * B * Hkv * d * dsize
    qo = 2 * B * Hq * d * dsize
    return codes + stats + qo


def cache_fill_bytes(B, Hkv, n, d, bits, dsize=2):
    """One read of K and V (the minimum: the statistics and the codes both need
    every element, and the single-read fill serves the second pass from L2) +
    writes of the codes and the statistics."""
    x = 2 * B * Hkv * n * d * dsize
    return x + 2 * B * Hkv * n * d * bits // 8 + 4 * B * Hkv * d * dsize


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel: str, workload: str, bits: int):
    """DRAM bytes per launch from the committed ncu summaries, if one was taken
    on this workload and bit width and the kernel source has not changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    src = decode_kernel_source(kernel)
    digest = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    with open(p) as f:
        records = json.load(f)["records"]
    for rec in records:
        if (rec.get("source") == src and rec.get("workload") == workload and rec.get("bits") == bits
                and rec.get("source_sha256_16") == digest):
            return rec
    return None


class ClockSampler:
    """Polls SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x1: "gpu_idle", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _poll(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def _sample(self):
        if self._nv is None:
            return
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        self._t = threading.Thread(target=self._poll, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join()
        if not self.samples:
            self._sample()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml, polled during the timed region"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[args.workload]
    B = args.batch or w.batch
    n, bits = w.n, args.bits
    layouts = ((cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V) if args.path == "octet"
               else (cq.LAYOUT_CANONICAL, cq.LAYOUT_CANONICAL))
    q, k, v = synth.make_case(B, w.hq, w.hkv, n, w.d, w.dtype, w.outliers, w.seed + 1000 * rank, device)
    torch.cuda.synchronize()

    # ---- cache fill (a1-a2): quantize K and V once; timed separately
    ws = torch.empty(cq.cq_quantize_kv_workspace_size(B, w.hkv, n, w.d), dtype=torch.uint8, device=device)
    kq = cq.cq_quantize_kv(k, bits, layouts[0], workspace=ws)
    vq = cq.cq_quantize_kv(v, bits, layouts[1], workspace=ws)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    def fill():
        cq.cq_quantize_kv(k, bits, layouts[0], out=kq, workspace=ws)
        cq.cq_quantize_kv(v, bits, layouts[1], out=vq, workspace=ws)

    fill_graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(fill_graph, capture_error_mode="relaxed"):
        fill()
    fill_ms = []
    for it in range(4):
        flush.fill_(it)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fill_graph.replay()
        e1.record(stream)
        e1.synchronize()
        if it:
            fill_ms.append(e0.elapsed_time(e1))
    del fill_graph, k, v
    torch.cuda.empty_cache()

    out = torch.empty_like(q)
    n_text = args.text
    if n_text:  # mixed cache: full-precision text tokens after the quantized visual ones
        if args.path != "octet":
            raise SystemExit("--text needs the octet layouts")
        gt = torch.Generator(device=device)
        gt.manual_seed(w.seed + 7 + 1000 * rank)
        k_text = synth.make_cache(B, w.hkv, n_text, w.d, w.dtype, 0, gt, device)
        v_text = synth.make_cache(B, w.hkv, n_text, w.d, w.dtype, 0, gt, device)
        dws = torch.empty(cq.cq_decode_attn_mixed_workspace_size(B, w.hq, w.d), dtype=torch.uint8, device=device)
    else:
        dws_n = cq.cq_decode_attn_workspace_size(layouts[0], layouts[1], B, w.hq, w.hkv, n, w.d, bits)
        dws = torch.empty(dws_n, dtype=torch.uint8, device=device) if dws_n else None
    launches_per_step = cq.cq_decode_launch_count(layouts[0], layouts[1], B, w.hq, w.hkv, n, w.d, bits, n_text)

    def decode(qq):
        if n_text:
            cq.cq_decode_attn_mixed(qq, kq, vq, k_text, v_text, calib=CALIB, out=out, workspace=dws)
        else:
            cq.cq_decode_attn(qq, kq, vq, calib=CALIB, out=out, workspace=dws)

    def step():
        decode(q)

    for it in range(args.warmup):
        flush.fill_(it & 255)
        step()
    torch.cuda.synchronize()

    # Host cost of one API call (validation + launch), measured while the GPU
    # is kept busy so that the host never waits for it.
    busy = torch.empty(1 << 30, dtype=torch.uint8, device=device)
    busy.fill_(1)
    h0 = time.perf_counter()
    for _ in range(20):
        step()
    host_us = (time.perf_counter() - h0) / 20 * 1e6
    del busy
    torch.cuda.synchronize()

    # The decode step is replayed from a CUDA graph so that the device time of
    # a step does not include host launch overhead (reported above).
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        step()
    torch.cuda.synchronize()
    for it in range(3):
        flush.fill_(it)
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region: K steps, L2 flushed between steps (outside the events)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_wall0 = time.perf_counter()
        for it in range(args.steps):
            flush.fill_((it * 7) & 255)
            starts[it].record(stream)
            graph.replay()
            ends[it].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall0
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    mean_ms = max_over_ranks(sum(step_ms) / len(step_ms), world, device)
    total_tokens = B * world  # one new token per sequence per step
    value = total_tokens / (mean_ms * 1e-3)

    # ---- end to end through the public API with host buffers
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_dev = torch.empty_like(q)
    e2e_ms = []
    for it in range(args.warmup + args.steps):
        flush.fill_(it & 255)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        q_dev.copy_(q_host, non_blocking=True)
        decode(q_dev)
        out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if it >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_mean = max_over_ranks(sum(e2e_ms) / len(e2e_ms), world, device)

    peak, peak_src = measured_peaks()
    dsize = 2 if w.dtype == "f16" else 4
    alg = algorithmic_bytes(B, w.hq, w.hkv, n, w.d, bits, dsize) + 2 * B * w.hkv * n_text * w.d * dsize
    kernel_ms = sum(step_ms) / len(step_ms)  # the step's launches (one on the plain octet path)
    achieved = alg / (kernel_ms * 1e-3) / 1e9
    kernel = cq.cq_decode_kernel_name(*layouts, B, w.hq, w.hkv, n, w.d, bits)
    trec = None if n_text else traffic_record(kernel, args.workload, bits)
    fill_mean = sum(fill_ms) / len(fill_ms)
    fill_alg = cache_fill_bytes(B, w.hkv, n, w.d, bits)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": mean_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u%d codes, int8 tensor-core products, f32 softmax, f16 I/O" % bits if args.path == "octet"
        else "u%d codes, f32 math, f16 I/O" % bits,
        "data": "synthetic (seeded InternVL-2.5-shaped K/V caches, no dataset or checkpoint)",
        "config": {"workload": args.workload, "batch_per_gpu": B, "global_batch": B * world,
                   "q_heads": w.hq, "kv_heads": w.hkv, "head_dim": w.d, "n_tokens": n, "bits": bits,
                   "layout": args.path, "text_tokens": n_text,
                   "calibration": {"tau_lo": CALIB[1], "tau_hi": CALIB[2]},
                   "l2": "flushed (256 MB write) between timed steps",
                   "parallelism": f"dp{world} (independent sequences per GPU)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": None if trec is None else trec["dram_bytes_per_launch"],
                     "algorithmic_bytes_per_launch": alg,
                     "kernel": kernel + ((" (text tokens in the same launch)" if kernel == "k_decode_row"
                                          else " (partial) + k_text_merge_mma") if n_text else
                                         (" + split-row launch (2-CTA clusters)"
                                          if kernel == "k_decode_row" and launches_per_step == 2 else ""))},
        "cache_fill": {"ms": fill_mean, "algorithmic_bytes": fill_alg,
                       "achieved_gbs": fill_alg / (fill_mean * 1e-3) / 1e9,
                       "frac": fill_alg / (fill_mean * 1e-3) / 1e9 / peak},
        "e2e": {"value": total_tokens / (e2e_mean * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": q.numel() * q.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size()},
        "gpu_launches": launches_per_step * args.steps,
        "host_overhead_us_per_call": host_us,
        "step_timing": "CUDA events around a CUDA-graph replay of one cq_decode_attn call",
        "clocks": clocks.summary(),
        "wall_s_timed_region": t_wall,
    }
    return line


def run_oracle_sample(w, rows: int, seed: int):
    """Times the fp64 CPU oracle's decode (given its own quantized cache) on
    `rows` (batch, kv-head) rows of workload w; returns (seconds, rows)."""
    import oracle
    from oracle import calibquant as oc
    q, k, v = synth.make_case(1, 4, 1, w.n, w.d, w.dtype, w.outliers, seed, "cpu")
    f = lambda t: t.to(torch.float64).numpy()
    q, k, v = f(q), f(k), f(v)
    kq = oracle.quantize_cache(k, 1, w.dtype)
    vq = oracle.quantize_cache(v, 1, w.dtype)
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):  # the baseline is stated as one core
        _oracle_rows(oc, q, kq, vq, rows)
    return time.perf_counter() - t0, rows


def _oracle_rows(oc, q, kq, vq, rows):
    for _ in range(rows):
        kh = oc.dequantize(kq["codes"], kq["alpha"], kq["scale"])
        vh = oc.dequantize(vq["codes"], vq["alpha"], vq["scale"])
        x = oc.scores_dequantized(q, kh)
        p = oc.softmax(oc.calibrate(x, CALIB[1], CALIB[2]))
        oc.attend_dequantized(p, vh)


def cpu_baseline(w):
    secs, rows = 0.0, 0
    while secs < 10.0 and rows < 400:  # about ten seconds of CPU work
        s, r = run_oracle_sample(w, rows=8, seed=99 + rows)
        secs += s
        rows += r
    seqs = rows / w.hkv  # a sequence has Hkv (batch, kv-head) rows
    return {"value": seqs / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} (sequence, kv-head) rows of {args_global.workload} "
                      f"(4 query heads x n={w.n} each), fp64 numpy, decode given the oracle's own "
                      f"quantized cache; {secs:.1f} s"}


def _oracle_timed_task(task):
    """One worker of the all-cores oracle baseline: builds its inputs, waits for
    the common start time, then decodes whole rows until the common end time;
    returns the rows it finished in the window."""
    wname, seed, start, span = task
    from oracle import calibquant as oc
    import oracle
    w = synth.WORKLOADS[wname]
    q, k, v = synth.make_case(1, 4, 1, w.n, w.d, w.dtype, w.outliers, seed, "cpu")
    f = lambda t: t.to(torch.float64).numpy()
    q, k, v = f(q), f(k), f(v)
    kq = oracle.quantize_cache(k, 1, w.dtype)
    vq = oracle.quantize_cache(v, 1, w.dtype)
    rows = 0
    with threadpool_limits(limits=1):
        while time.time() < start:
            time.sleep(0.01)
        while time.time() < start + span:
            _oracle_rows(oc, q, kq, vq, 1)
            rows += 1
    return rows


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_all_cores(w, wname: str, span: float = 10.0):
    """The oracle on every host core at once (one single-threaded process per
    core, at most 32): rows finished by all processes in a common window."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    nproc = os.cpu_count() or 1
    workers = max(1, min(nproc, 32))
    start = time.time() + 45.0  # spawn, imports and inputs finish before the window opens
    try:  # a worker that dies raises here instead of leaving the bench waiting
        with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
            futs = [ex.submit(_oracle_timed_task, (wname, 500 + i, start, span)) for i in range(workers)]
            rows = sum(f.result(timeout=120 + span) for f in futs)
    except Exception as e:  # noqa: BLE001 -- a baseline, reported as missing rather than failing the bench
        return {"value": None, "unit": "tokens/s", "cores": workers, "nproc": nproc, "kind": "oracle",
                "error": f"{type(e).__name__}: {e}"[:200]}
    seqs = rows / w.hkv
    return {"value": seqs / span, "unit": "tokens/s", "cores": workers, "nproc": nproc, "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{rows} (sequence, kv-head) rows of {wname} decoded by {workers} single-threaded "
                      f"processes in a common {span:.0f} s window (fp64 numpy)"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    times = []
    for it in range(args.warmup + args.steps):
        secs, rows = run_oracle_sample(w, rows=1, seed=it)
        if it >= args.warmup:
            times.append(secs)
    mean = sum(times) / len(times)
    value = (1 / w.hkv) / mean
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded InternVL-2.5-shaped K/V caches)",
        "config": {"workload": args.workload, "bits": 1, "step": "one (sequence, kv-head) row"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"one (sequence, kv-head) row per step, n={w.n}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


args_global = None


BUDGET_LAYERS, BUDGET_N = 32, 3328  # full InternVL-2.5-8B decode step at n = 3328


def budget_batches(budget_gb: float, hkv: int = 8, d: int = 128):
    """Largest batch whose KV cache fits the budget (GB = 1e9 bytes, cache only):
    1-bit codes plus f16 alpha / step of K and V, versus an f16 cache."""
    per_seq_1bit = BUDGET_LAYERS * hkv * (2 * BUDGET_N * d // 8 + 4 * d * 2)
    per_seq_f16 = BUDGET_LAYERS * hkv * 2 * BUDGET_N * d * 2
    return int(budget_gb * 1e9 // per_seq_1bit), int(budget_gb * 1e9 // per_seq_f16), per_seq_1bit, per_seq_f16


def _time_graph(step, steps: int, warmup: int) -> float:
    """Mean ms of one captured step (all layers), CUDA events on the capture stream."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step()
        for _ in range(warmup):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(s)
        for _ in range(steps):
            g.replay()
        e1.record(s)
        e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del g
    return ms


def _time_flushed(step, steps: int, warmup: int, flush) -> float:
    """Mean ms of one step replayed from a CUDA graph, CUDA events on the
    launching stream around each replay, the L2 flushed (outside the events)
    before every timed replay."""
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(warmup):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    for it in range(warmup):
        flush.fill_(it & 255)
        g.replay()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for it in range(steps):
        flush.fill_((it * 7) & 255)
        starts[it].record(stream)
        g.replay()
        ends[it].record(stream)
    torch.cuda.synchronize()
    del g
    return sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps


def run_bit_sweep(args):
    """Bit-width sweep at bitsweep_n8192_b16 (batch 16, 32 / 8 heads, d = 128,
    n = 8192, the caches quantized by the library at each b): one JSON line
    per b in {1, 2, 4, 8} with the step time of one cq_decode_attn call,
    tokens/s, GB/s of algorithmic bytes and the fraction of the measured copy
    bandwidth. (The output error of each b against the fp64 oracle is reported
    by tests/bitsweep_error_report.py on the same seeded inputs.)"""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS["bitsweep_n8192_b16"]
    q, k, v = synth.make_workload(w, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peak, peak_src = measured_peaks()
    K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V
    for bits in (1, 2, 4, 8):
        kq = cq.cq_quantize_kv(k, bits, K)
        vq = cq.cq_quantize_kv(v, bits, V)
        out = torch.empty_like(q)

        def step():
            cq.cq_decode_attn(q, kq, vq, calib=CALIB, out=out)

        ms = _time_flushed(step, min(args.steps, 200), args.warmup, flush)
        alg = algorithmic_bytes(w.batch, w.hq, w.hkv, w.n, w.d, bits)
        gbs = alg / (ms * 1e-3) / 1e9
        print(json.dumps({
            "metric": "decode-attention tokens/s and achieved HBM GB/s per bit width (n=8192, batch 16)",
            "bits": bits, "value": w.batch / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "higher_is_better": True, "data": "synthetic (seeded InternVL-2.5-shaped K/V caches)",
            "config": {"workload": "bitsweep_n8192_b16", "batch": w.batch, "q_heads": w.hq, "kv_heads": w.hkv,
                       "head_dim": w.d, "n_tokens": w.n, "layout": "octet",
                       "calibration": {"tau_lo": CALIB[1], "tau_hi": CALIB[2]},
                       "l2": "flushed (256 MB write) between timed steps"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_source": peak_src, "algorithmic_bytes_per_launch": alg},
            "kernel": cq.cq_decode_kernel_name(K, V, w.batch, w.hq, w.hkv, w.n, w.d, bits),
            "gpu_launches_per_step": cq.cq_decode_launch_count(K, V, w.batch, w.hq, w.hkv, w.n, w.d, bits)}),
            flush=True)
        del kq, vq, out
        torch.cuda.empty_cache()


def run_budget(args):
    """Memory-budget sweep: a full 32-layer decode step (32 / 8 heads, d = 128,
    n = 3328) with the largest batch whose KV cache fits each budget, 1-bit
    cache through libcalibq against an f16 cache through PyTorch's fused
    attention (scaled_dot_product_attention, the comparison arm). Every layer
    has its own buffers (the working set is far above L2). Inputs are random:
    the step time does not depend on the values. One JSON line per budget."""
    dev = torch.device("cuda", 0)
    hq, hkv, d, n = 32, 8, 128, BUDGET_N
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    for budget in args.budgets:
        b1, b16, per1, per16 = budget_batches(budget, hkv, d)
        rb = cq.cq_codes_bytes(cq.LAYOUT_OCTET_K, 1, 1, n, d, 1)  # == the OCTET_V row at n = 3328
        layers = []
        for _ in range(BUDGET_LAYERS):
            codes = [torch.randint(0, 256, (b1, hkv, rb), dtype=torch.uint8, device=dev, generator=gen)
                     for _ in range(2)]
            stats = [torch.rand(b1, hkv, d, device=dev, generator=gen).half() + 0.5 for _ in range(4)]
            kq = cq.QuantizedCache(codes[0], stats[0] - 1.0, stats[1], cq.LAYOUT_OCTET_K, 1, n)
            vq = cq.QuantizedCache(codes[1], stats[2] - 1.0, stats[3], cq.LAYOUT_OCTET_V, 1, n)
            q = torch.randn(b1, hq, d, device=dev, generator=gen).half()
            layers.append((q, kq, vq, torch.empty_like(q)))
        kernel = cq.cq_decode_kernel_name(cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, b1, hq, hkv, n, d, 1)

        def step1():
            for q, kq, vq, out in layers:
                cq.cq_decode_attn(q, kq, vq, calib=CALIB, out=out)

        steps = min(args.steps, 20)  # a 32-layer step is milliseconds long
        ms1 = _time_graph(step1, steps, args.warmup)
        bytes1 = BUDGET_LAYERS * algorithmic_bytes(b1, hq, hkv, n, d, 1)
        del layers, step1
        torch.cuda.empty_cache()
        layers16 = []
        for _ in range(BUDGET_LAYERS):
            k = torch.randn(b16, hkv, n, d, device=dev, generator=gen).half()
            v = torch.randn(b16, hkv, n, d, device=dev, generator=gen).half()
            q = torch.randn(b16, hq, 1, d, device=dev, generator=gen).half()
            layers16.append((q, k, v))

        def step16():
            for q, k, v in layers16:
                torch.nn.functional.scaled_dot_product_attention(q, k, v, enable_gqa=True)

        ms16 = _time_graph(step16, steps, args.warmup)
        bytes16 = BUDGET_LAYERS * (2 * b16 * hkv * n * d * 2 + 2 * b16 * hq * d * 2)
        del layers16, step16
        torch.cuda.empty_cache()
        tps1, tps16 = b1 / (ms1 * 1e-3), b16 / (ms16 * 1e-3)
        print(json.dumps({
            "metric": "decode-step tokens/s under a KV-cache memory budget (32 layers, n=3328)",
            "budget_gb": budget, "data": "synthetic (random codes, statistics and f16 caches)",
            "config": {"workload": "budget_n3328_32layers", "layers": BUDGET_LAYERS, "q_heads": hq, "kv_heads": hkv,
                       "head_dim": d, "n_tokens": n, "cache_bytes_per_sequence": {"1bit": per1, "f16": per16}},
            "calibquant_1bit": {"batch": b1, "ms_per_step": ms1, "tokens_per_s": tps1, "kernel": kernel,
                                "achieved_gbs": bytes1 / (ms1 * 1e-3) / 1e9},
            "f16_cache": {"batch": b16, "ms_per_step": ms16, "tokens_per_s": tps16,
                          "kernel": "torch scaled_dot_product_attention (enable_gqa)",
                          "achieved_gbs": bytes16 / (ms16 * 1e-3) / 1e9},
            "speedup": tps1 / tps16}), flush=True)


def main():
    global args_global
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="internvl8b_n8192_b64", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--bits", type=int, default=1)
    ap.add_argument("--path", choices=["octet", "canonical"], default="octet")
    ap.add_argument("--text", type=int, default=0,
                    help="full-precision text tokens after the quantized ones (mixed cache)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--budget-sweep", action="store_true",
                    help="32-layer decode step under KV-cache budgets, 1-bit vs f16 cache (one line per budget)")
    ap.add_argument("--budgets", type=float, nargs="+", default=[5, 10, 20, 30])
    ap.add_argument("--bit-sweep", action="store_true",
                    help="bit widths 1, 2, 4, 8 at bitsweep_n8192_b16 (one line per width)")
    args = ap.parse_args()
    args_global = args
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.budget_sweep:
        run_budget(args)
        return
    if args.bit_sweep:
        run_bit_sweep(args)
        return
    world, rank, local = dist_setup()
    if args.impl == "reference":
        line = run_reference(args, world, rank)
    else:
        line = run_ours(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(synth.WORKLOADS[args.workload])
            line["cpu_baseline"]["nproc"] = os.cpu_count() or 1
            line["cpu_baseline"]["cpu_model"] = cpu_model()
            line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(synth.WORKLOADS[args.workload], args.workload)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python3
"""Benchmark: NVFP4 sparse MLA decode on B200.

One step = one decode launch of the hot path (list compaction, row gather,
on-chip NVFP4 unpack, QK^T, online softmax, PV, split merge) over the
35-token x 64-head workload: 35 query tokens from 35 requests, each request
with a 140,000-row context in a shared paged NVFP4 cache (4.9M rows), 2048
indexer-selected rows per token.  The staged FP8 comparison path and the
append kernel are timed in the same run and reported beside the headline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
(the reference arm for this build) on a bounded sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 sparse MLA decode µs/launch & TFLOP/s, % of roofline (1×B200)"
FLOP_PER_ROW_HEAD = 2 * 576 + 2 * 512          # QK^T + PV per (token, head, valid row)
ROW_BYTES = 352
N_SETS = 8                                      # rotating index/query sets
L2_BYTES = 126 * 2 ** 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip staged/append/e2e/cpu legs")
    ap.add_argument("--workload", default="decode35x64",
                    choices=["decode35x64", "sweep", "padded", "prefill", "tiny", "paged", "fp8", "indexer",
                             "blhnc", "plans", "all-others"],
                    help="decode35x64 (default) prints the one result line; the others time the remaining "
                         "workloads and print one line per shape")
    ap.add_argument("--ctx", type=int, default=140_000,
                    help="context rows per request of the decode35x64 leg (smaller values give a small case "
                         "of the same kernel, e.g. for a profiler capture)")
    ap.add_argument("--layers", type=int, default=64,
                    help="layers of the request converted by --workload blhnc")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="time the K launches replayed from a captured CUDA graph (default) or issued one by one")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, torch_device: int, period: float = 0.01):
        self.samples = []
        self.period = period
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            p = torch.cuda.get_device_properties(torch_device)
            bus = getattr(p, "pci_bus_id", None)
            if bus is not None:  # match the CUDA device to its NVML handle by PCI location
                bus_id = "%08X:%02X:%02X.0" % (getattr(p, "pci_domain_id", 0), bus, getattr(p, "pci_device_id", 0))
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus_id.encode())
                except Exception:  # noqa: BLE001
                    self.h = None
            if self.h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                ids = [v for v in vis.split(",") if v.strip()]
                idx = int(ids[torch_device]) if ids and ids[torch_device].strip().isdigit() else torch_device
                self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvml unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "sampled during the timed region"
        if not inside:  # region shorter than one period: take the samples nearest to it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = sorted(v for k, v in self.REASONS.items() if bits & k and v != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "note": note}


def code_fingerprint(path: str) -> str:
    """sha256 of a C/CUDA source with comments and whitespace removed, so a
    comment edit keeps the fingerprint and any code change alters it."""
    import re
    src = open(path, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()


def kernel_traffic(kernel_file: str):
    """DRAM bytes per launch from a committed ncu summary, valid only while
    the kernel code is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_code_sha256") != code_fingerprint(kernel_file):
        return None
    return d.get("dram_bytes_per_launch")


def workload_stats(indices_sets, T, H):
    """Valid rows per launch and algorithmic bytes / FLOP of one launch."""
    import torch
    valid = [int(((ix >= 0)).sum().item()) for ix in indices_sets]
    rows = statistics.mean(valid)
    flop = FLOP_PER_ROW_HEAD * H * rows
    bytes_ = ROW_BYTES * rows + T * indices_sets[0].shape[1] * 4 + T * H * (576 * 2 + 512 * 2 + 4)
    return rows, flop, bytes_


def oracle_passes(w, seconds: float):
    """Time the CPU oracle over all of w's tokens, repeating whole passes
    until about `seconds` of CPU time have run; returns (FLOP per second,
    passes, seconds, threads)."""
    import oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from harness import oracle_inputs
    qn, qr, rows, remap, _ = oracle_inputs(w, list(range(w.T)))
    flop = FLOP_PER_ROW_HEAD * w.H * int((remap >= 0).sum())
    passes, t_all = 0, 0.0
    while passes == 0 or t_all < seconds:
        t0 = time.perf_counter()
        oracle.sparse_mla(qn, qr, rows, remap, w.sm_scale)
        t_all += time.perf_counter() - t0
        passes += 1
    return flop * passes / t_all, passes, t_all, oracle.max_threads()


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of every rank's value (the job is as slow as its slowest
    replica); every rank takes the same collective step."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as tdist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flop_per_launch: float, ms_total: float, steps: int, world: int) -> float:
    """Whole-job throughput: every rank ran `steps` launches of the same work,
    timed as the slowest rank's `ms_total`."""
    return flop_per_launch * steps * world / (ms_total * 1e-3) / 1e12


def reference_arm(args, rank, world):
    """CPU oracle on host cores, rank 0 only, bounded sample of the workload."""
    if rank != 0:
        return
    import torch
    from nvfp4_sparse_mla_decode_b200 import synth
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = synth.decode35(dev)
    # one step = whole passes of the oracle over all 35 tokens for ~10 s
    if args.warmup > 0:
        oracle_passes(w, 0.0)
    rates, passes, secs, cores = [], 0, 0.0, 0
    for _ in range(min(args.steps, 3)):
        r, n, t, cores = oracle_passes(w, 10.0)
        rates.append(r)
        passes += n
        secs += t
    tflops = statistics.median(rates) / 1e12
    sec = secs / max(1, len(rates))
    sample = ("%d passes over all %d tokens of decode35x64 (H=64, 2048 valid rows each) in %d steps of ~10 s, "
              "FP64 oracle incl. row dequantization" % (passes, w.T, len(rates)))
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": len(rates), "warmup": 1 if args.warmup > 0 else 0, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode35x64", "T": w.T, "H": w.H, "topk": 2048, "ctx_rows": 140000,
                   "sample": "all tokens, repeated passes"},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_other_workload(name, w, nv, synth, args):
    """One JSON line for a non-default workload: single launches with a cold
    L2 (a buffer twice the L2 size is written before each), timed with CUDA
    events on the launching stream around the decode alone; median of 20."""
    import torch
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    cache = build_cache(w)
    rows, flop, alg_bytes = workload_stats([w.indices], w.T, w.H)
    topk = w.indices.shape[1]
    out = torch.empty(w.T, w.H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(w.T, w.H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(w.T, w.H, topk)), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out=out, lse=lse, workspace=ws,
                  dev_status=status)
    times = []
    for _ in range(20):
        flush.fill_(1)
        e0.record(stream)
        nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out=out, lse=lse, workspace=ws,
                  dev_status=status)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    us = statistics.median(times)
    peaks, _ = measured_peaks()
    t_roof = max(flop / (float(peaks["bf16_tflops"]) * 1e12), alg_bytes / (float(peaks["hbm_gbs"]) * 1e9))
    line = {"metric": METRIC, "workload": name, "T": w.T, "H": w.H, "topk": topk,
            "valid_rows_per_launch": rows, "splits": nv.num_splits(w.T, w.H, topk), "us_per_launch": us,
            "tflops": flop / (us * 1e-6) / 1e12, "gathered_gbs": rows * ROW_BYTES / (us * 1e-6) / 1e9,
            "roofline_us": t_roof * 1e6, "frac_of_roofline": t_roof / (us * 1e-6),
            "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}
    del cache, flush
    torch.cuda.empty_cache()
    return line


def config_workloads(synth):
    """The parity configurations other than the headline launch, as
    (name, workload factory) pairs: the tiny case, the H=128 decode sweep at
    every token count, the padded-list stress and the 4000-token prefill."""
    items = [("tiny1x16", lambda: synth.tiny("cuda"))]
    for T in (1, 8, 32, 64, 128, 256):
        items.append(("sweep%dx128" % T, lambda T=T: synth.sweep("cuda", T)))
    items.append(("padded256x64", lambda: synth.padded("cuda")))
    items.append(("prefill4000x64", lambda: synth.append_prefill("cuda")))
    return items


def time_paged(nv, synth, args):
    """decode35x64 with request-local positions and block tables (the
    translation inside the launch) against the same lists as slot ids: single
    launches with a cold L2, median of 20 each."""
    import torch
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    w = synth.decode35("cuda")
    cache = build_cache(w)
    table = synth.block_table(w)
    pos = w.positions.contiguous()
    out = torch.empty(w.T, w.H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(w.T, w.H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(w.T, w.H)), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    calls = {
        "slot_ids": lambda: nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out=out, lse=lse,
                                      workspace=ws, dev_status=status),
        "positions_block_table": lambda: nv.decode_paged(w.q_nope, w.q_rope, cache, pos, table, synth.PAGE_SIZE,
                                                         w.sm_scale, out=out, lse=lse, workspace=ws,
                                                         dev_status=status),
    }
    res = {}
    for name, fn in calls.items():
        for _ in range(3):
            fn()
        times = []
        for _ in range(20):
            flush.fill_(1)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
        res[name] = statistics.median(times)
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    print(json.dumps({"metric": METRIC, "workload": "decode35x64 paged", "T": w.T, "H": w.H,
                      "us_per_launch_slot_ids": res["slot_ids"],
                      "us_per_launch_positions_block_table": res["positions_block_table"],
                      "translation_overhead_us": res["positions_block_table"] - res["slot_ids"],
                      "page_size": synth.PAGE_SIZE, "table_stride": int(table.shape[1]),
                      "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}),
          flush=True)
    del cache, flush
    torch.cuda.empty_cache()


def cold_median_us(fn, flush, n=20):
    """Median device time (us) of fn() over n launches, each after writing a
    buffer larger than L2; CUDA events on the current stream."""
    import torch
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        fn()
    times = []
    for _ in range(n):
        flush.fill_(1)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    return statistics.median(times)


def time_fp8(nv, synth, args):
    """decode35x64 over the 576-byte E4M3 row cache (the row before NVFP4)
    against the 352-byte NVFP4 cache and the staged path, plus both append
    kernels on the 4000 prefill rows: single launches, L2 flushed, median
    of 20 each."""
    import torch
    from nvfp4_sparse_mla_decode_b200.cache import build_cache, build_fp8_cache
    w = synth.decode35("cuda")
    cache = build_cache(w)
    fcache = build_fp8_cache(w)
    rows, flop, _ = workload_stats([w.indices], w.T, w.H)
    out = torch.empty(w.T, w.H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(w.T, w.H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(w.T, w.H)), dtype=torch.uint8, device="cuda")
    staging = torch.empty(nv.staging_size(w.T), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    kw = dict(out=out, lse=lse, workspace=ws, dev_status=status)
    us = {
        "nvfp4_cache": cold_median_us(lambda: nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, **kw),
                                      flush),
        "fp8_cache": cold_median_us(lambda: nv.fp8_decode(w.q_nope, w.q_rope, fcache, w.indices, w.sm_scale,
                                                          **kw), flush),
        "staged": cold_median_us(lambda: nv.staged_decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale,
                                                          staging=staging, **kw), flush),
    }
    del cache, fcache, staging
    torch.cuda.empty_cache()
    wa = synth.append_prefill("cuda")
    a_us = {}
    for name, rb, fn in (("nvfp4", nv.ROW_BYTES, nv.kv_append), ("fp8", nv.STAGED_ROW_BYTES, nv.fp8_kv_append)):
        ac = torch.zeros(wa.num_slots, rb, dtype=torch.uint8, device="cuda")
        a_us[name] = cold_median_us(lambda: fn(wa.new_lat, wa.new_rope, wa.new_slots, ac, status), flush)
        del ac
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    peaks, _ = measured_peaks()
    line = {"metric": METRIC, "workload": "decode35x64 fp8 rows", "T": w.T, "H": w.H,
            "valid_rows_per_launch": rows,
            "us_per_launch": us,
            "tflops": {k: flop / (v * 1e-6) / 1e12 for k, v in us.items()},
            "gathered_gbs": {"nvfp4_cache": rows * nv.ROW_BYTES / (us["nvfp4_cache"] * 1e-6) / 1e9,
                             "fp8_cache": rows * nv.STAGED_ROW_BYTES / (us["fp8_cache"] * 1e-6) / 1e9},
            "rows_per_gb": {"nvfp4": 1e9 / nv.ROW_BYTES, "fp8": 1e9 / nv.STAGED_ROW_BYTES},
            "capacity_ratio": nv.STAGED_ROW_BYTES / nv.ROW_BYTES,
            "append_4000_rows_us": a_us,
            "append_gbs": {"nvfp4": wa.T * (1152 + 352 + 4) / (a_us["nvfp4"] * 1e-6) / 1e9,
                           "fp8": wa.T * (1152 + 576 + 4) / (a_us["fp8"] * 1e-6) / 1e9},
            "hbm_peak_gbs": float(peaks["hbm_gbs"]),
            "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}
    print(json.dumps(line), flush=True)
    del flush
    torch.cuda.empty_cache()


def time_indexer(nv, synth, args):
    """The sparse indexer on 35 requests of 140,000 positions (page 64): the
    score kernel, the top-k kernel and both in one call, single launches with
    L2 flushed, median of 20 each; then the indexer followed by the paged
    decode over its lists."""
    import math
    import torch
    T, ctx, page = 35, 140_000, synth.PAGE_SIZE
    w = synth.decode35("cuda")
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    cache = build_cache(w)
    table = synth.block_table(w)
    keys = synth.indexer_keys(w.num_slots, 1, "cuda")
    q, wt = synth.indexer_queries(T, 1, "cuda")
    lens = torch.tensor(w.ctx_lens, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stride = nv.indexer_score_stride(ctx)
    scores = torch.empty(T, stride, dtype=torch.float32, device="cuda")
    pos = torch.empty(T, 2048, dtype=torch.int32, device="cuda")
    ws_i = torch.zeros(nv.lib().nvfp4mla_indexer_workspace_size(T, ctx), dtype=torch.uint8, device="cuda")
    ws_k = torch.zeros(max(256, nv.lib().nvfp4mla_indexer_topk_workspace_size(T)), dtype=torch.uint8,
                       device="cuda")
    out = torch.empty(T, w.H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(T, w.H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(T, w.H)), dtype=torch.uint8, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    def scores_only():
        nv.indexer_scores(q, wt, keys, table, page, lens, ctx, scores=scores, dev_status=status)

    def topk_only():
        nv.indexer_topk(scores, lens, ctx, 2048, positions=pos, workspace=ws_k, dev_status=status)

    def indexer():
        nv.sparse_indexer(q, wt, keys, table, page, lens, ctx, positions=pos, workspace=ws_i, dev_status=status)

    def indexer_then_decode():
        indexer()
        nv.decode_paged(w.q_nope, w.q_rope, cache, pos, table, page, w.sm_scale, out=out, lse=lse, workspace=ws,
                        dev_status=status)

    us = {"scores": cold_median_us(scores_only, flush)}
    scores_only()
    us["topk"] = cold_median_us(topk_only, flush)
    us["indexer"] = cold_median_us(indexer, flush)
    us["indexer_then_decode"] = cold_median_us(indexer_then_decode, flush)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    peaks, _ = measured_peaks()
    positions = T * ctx
    pages = T * math.ceil(ctx / page)
    # algorithmic bytes of the score kernel: keys, table entries, q, w, scores written
    score_bytes = positions * 128 + pages * 4 + T * 64 * (128 + 4) + positions * 4
    flop = 2.0 * positions * 64 * 128
    line = {"metric": METRIC, "workload": "indexer35x140000", "T": T, "ctx": ctx, "page_size": page,
            "index_heads": 64, "index_dim": 128, "topk": 2048, "us_per_launch": us,
            "score_kernel_gbs": score_bytes / (us["scores"] * 1e-6) / 1e9,
            "score_kernel_frac_of_hbm": score_bytes / (us["scores"] * 1e-6) / 1e9 / float(peaks["hbm_gbs"]),
            "score_kernel_alg_bytes": score_bytes, "score_kernel_tflops_fp8": flop / (us["scores"] * 1e-6) / 1e12,
            "hbm_peak_gbs": float(peaks["hbm_gbs"]),
            "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}
    print(json.dumps(line), flush=True)
    del cache, keys, flush
    torch.cuda.empty_cache()


def time_blhnc(nv, synth, args):
    """The block-major layout conversion for one 200,000-position request
    (page 64, 352-byte rows) over --layers layers (64 by default, a
    representative depth; the pages give none): per-layer caches ->
    block-major cache with blocks a
    sixteenth of the size, and back; single launches with L2 flushed, median
    of 20; plus the descriptor counts of moving that request."""
    import numpy as np
    import torch
    L, N, C, sub, ctx = args.layers, synth.PAGE_SIZE, 352, 16, 200_000
    nb = (ctx + N - 1) // N
    num_blocks = nb + 64
    rng = np.random.default_rng(5)
    # the request's blocks: runs of 8 consecutive blocks in random order
    supers = rng.permutation(num_blocks // 8)
    ids = (supers[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)[:nb].astype(np.int32)
    # block-major ids: a packed transfer buffer, and a cache whose free
    # blocks also come in runs of 8
    packed = np.arange(nb * sub, dtype=np.int32)
    nsup = (nb * sub + 7) // 8 + 8
    frag = (rng.permutation(nsup)[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)[:nb * sub].astype(np.int32)
    g = torch.Generator(device="cuda").manual_seed(5)
    caches = [torch.randint(0, 256, (num_blocks, N, C), generator=g, device="cuda", dtype=torch.int32)
              .to(torch.uint8) for _ in range(L)]
    out = torch.empty(nsup * 8, L, N // sub, C, dtype=torch.uint8, device="cuda")
    ptrs = torch.tensor([c.data_ptr() for c in caches], dtype=torch.int64, device="cuda")
    ids_d = torch.from_numpy(ids).cuda()
    frag_d = torch.from_numpy(frag).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    us = {
        "to_block_major": cold_median_us(lambda: nv.blhnc_convert(caches, ids_d, frag_d, out, sub, True, ptrs,
                                                                  status), flush),
        "back": cold_median_us(lambda: nv.blhnc_convert(caches, ids_d, frag_d, out, sub, False, ptrs, status),
                               flush),
    }
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    peaks, _ = measured_peaks()
    moved = 2 * nb * N * L * C  # every byte read once and written once
    line = {"metric": METRIC, "workload": "blhnc200000x%dlayers" % L, "positions": ctx, "layers": L, "block_size": N,
            "block_major_block_size": N // sub, "row_bytes": C, "us_per_launch": us,
            "gbs": {k: moved / (v * 1e-6) / 1e9 for k, v in us.items()},
            "frac_of_hbm": {k: moved / (v * 1e-6) / 1e9 / float(peaks["hbm_gbs"]) for k, v in us.items()},
            "bytes_moved": moved,
            "descriptors": {"per_layer_layout": nv.copy_descriptors(ids, L),
                            "block_major_fragmented": nv.copy_descriptors(frag),
                            "block_major_packed": nv.copy_descriptors(packed)},
            "hbm_peak_gbs": float(peaks["hbm_gbs"]),
            "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}
    print(json.dumps(line), flush=True)
    del caches, out, flush
    torch.cuda.empty_cache()


def time_plans(nv, synth, args):
    """Small batches under each head-group width (nvfp4mla_tuning with
    heads_per_cta fixed, the split count left automatic): one line per
    shape, cold single launches (L2 flushed before each, median of 20),
    preallocated outputs and workspaces, 140,000-row contexts."""
    import torch
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    for H in (64, 128):
        for T in (1, 2, 4, 8):
            w = synth.per_request("cuda", [140_000] * T, H, seed=5 + T, name="plans")
            cache = build_cache(w)
            out = torch.empty(T, H, 512, dtype=torch.float16, device="cuda")
            lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
            res = {}
            for hg in (64, 32, 16):
                tuning = nv.Tuning(splits=0, heads_per_cta=hg)
                wsz = nv.workspace_size(T, H, 2048, tuning)
                ws = torch.zeros(max(1, wsz), dtype=torch.uint8, device="cuda")
                S = 1 if wsz == 0 else (wsz - 4096) // (T * H * 514 * 4)

                def fn():
                    nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out=out, lse=lse, workspace=ws,
                              tuning=tuning)
                res["hg%d" % hg] = {"splits": S, "ctas": T * (H // hg) * S, "us_per_launch": cold_median_us(fn, flush)}
            ws = torch.zeros(max(1, nv.workspace_size(T, H)), dtype=torch.uint8, device="cuda")

            def fn_auto():
                nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out=out, lse=lse, workspace=ws)
            auto = {"splits": nv.num_splits(T, H), "us_per_launch": cold_median_us(fn_auto, flush)}
            print(json.dumps({"metric": METRIC, "workload": "plans T=%d H=%d" % (T, H), "T": T, "H": H,
                              "by_heads_per_cta": res, "automatic": auto,
                              "timing": "single launch, L2 flushed before it, median of 20", "data": "synthetic"}),
                  flush=True)
            del cache
            torch.cuda.empty_cache()


def other_workloads(args):
    import torch
    import nvfp4_sparse_mla_decode_b200 as nv
    from nvfp4_sparse_mla_decode_b200 import synth
    assert torch.cuda.is_available(), "bench.py needs a CUDA GPU"
    nv.lib()
    names = (["tiny", "sweep", "padded", "prefill", "paged", "fp8", "indexer", "blhnc", "plans"]
             if args.workload == "all-others" else [args.workload])
    for name in names:
        if name == "plans":
            time_plans(nv, synth, args)
        if name == "blhnc":
            time_blhnc(nv, synth, args)
        if name == "indexer":
            time_indexer(nv, synth, args)
        if name == "paged":
            time_paged(nv, synth, args)
        if name == "fp8":
            time_fp8(nv, synth, args)
        for cname, make in config_workloads(synth):
            if (name == "tiny" and cname.startswith("tiny")) or (name == "sweep" and cname.startswith("sweep")) or \
                    (name == "padded" and cname.startswith("padded")) or (name == "prefill" and cname.startswith("prefill")):
                print(json.dumps(time_other_workload(cname, make(), nv, synth, args)), flush=True)


def graph_us(fns, n):
    """Device time per call (us) of the callables in fns, captured once in a
    CUDA graph (one call each) and replayed until n calls have run; CUDA
    events on the launching stream around the replays."""
    import torch
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for fn in fns:
            fn()
    g.replay()
    torch.cuda.synchronize()
    reps = max(1, n // len(fns))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * len(fns))
    del g
    return us


def staged_leg(nv, w, cache, sets, rows, flop, native_us, peak_bw, args):
    """The staged FP8 path on the same rotating sets, each step timed alone
    and both together, every figure from CUDA-graph replays like the native
    launch: step 1 writes the E4M3 rows of the valid entries to HBM, step 2
    runs attention over them."""
    import torch
    T, H, topk = w.T, w.H, sets[0][0].shape[1]
    staging = torch.empty(nv.staging_size(T, topk), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(T, H, topk)), dtype=torch.uint8, device="cuda")
    n = max(80, min(4000, args.steps // 4))
    stage = [lambda ix=ix: nv.staged_stage(cache, ix, staging) for ix, _, _ in sets]
    attend = [lambda ix=ix, qn=qn, qr=qr: nv.staged_attend(qn, qr, cache.shape[0], ix, staging, w.sm_scale, out=out,
                                                           lse=lse, workspace=ws) for ix, qn, qr in sets]
    both = [lambda ix=ix, qn=qn, qr=qr: nv.staged_decode(qn, qr, cache, ix, w.sm_scale, out=out, lse=lse,
                                                         staging=staging, workspace=ws) for ix, qn, qr in sets]
    for f in both:
        f()
    us_stage, us_attend, us_both = graph_us(stage, n), graph_us(attend, n), graph_us(both, n)
    stage_bytes = rows * (ROW_BYTES + nv.STAGED_ROW_BYTES) + T * topk * 4
    del staging
    return {"us_per_launch": us_both, "tflops": flop / (us_both * 1e-6) / 1e12, "native_speedup": us_both / native_us,
            "stage_us": us_stage, "stage_gbs": stage_bytes / (us_stage * 1e-6) / 1e9,
            "stage_frac_of_hbm": stage_bytes / (us_stage * 1e-6) / 1e9 / peak_bw, "stage_bytes": stage_bytes,
            "attend_us": us_attend, "attend_tflops": flop / (us_attend * 1e-6) / 1e12, "launches": 2,
            "staging_bytes": nv.staging_size(T, topk), "timing": "CUDA graph replays, %d calls each" % n}


N_E2E_STREAMS = 4


def e2e_leg(nv, w, cache, sets, flop, world, args):
    """End to end through the host-buffer C-ABI call: each step copies its
    queries and lists from pinned host memory, decodes, and copies out and
    lse back; consecutive steps rotate over N_E2E_STREAMS streams (each with
    its own device buffers and workspace), so the uploads of later steps, the
    kernels and the downloads of earlier steps overlap.  Device time from the
    first copy to the last result."""
    import torch
    T, H, topk = w.T, w.H, sets[0][0].shape[1]
    h_sets = [(ix.cpu().pin_memory(), qn.cpu().pin_memory(), qr.cpu().pin_memory()) for ix, qn, qr in sets]
    streams = [torch.cuda.Stream() for _ in range(N_E2E_STREAMS)]
    bufs = []
    for _ in streams:
        bufs.append(dict(d_q_nope=torch.empty_like(sets[0][1]), d_q_rope=torch.empty_like(sets[0][2]),
                         d_indices=torch.empty_like(sets[0][0]),
                         d_out=torch.empty(T, H, 512, dtype=torch.float16, device="cuda"),
                         d_lse=torch.empty(T, H, dtype=torch.float32, device="cuda"),
                         h_out=torch.empty(T, H, 512, dtype=torch.float16).pin_memory(),
                         h_lse=torch.empty(T, H, dtype=torch.float32).pin_memory(),
                         workspace=torch.zeros(max(1, nv.workspace_size(T, H, topk)), dtype=torch.uint8,
                                               device="cuda")))

    def step(k):
        b = bufs[k % N_E2E_STREAMS]
        ix, qn, qr = h_sets[k % len(h_sets)]
        nv.decode_host(qn, qr, ix, b["h_out"], b["h_lse"], b["d_q_nope"], b["d_q_rope"], b["d_indices"], b["d_out"],
                       b["d_lse"], cache, w.sm_scale, workspace=b["workspace"], stream=streams[k % N_E2E_STREAMS])

    for k in range(6):
        step(k)
    torch.cuda.synchronize()
    ne = max(40, min(2000, args.steps // 10))
    cur = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s in streams:
        s.wait_stream(cur)
    for k in range(ne):
        step(k)
    for s in streams:
        cur.wait_stream(s)
    e1.record(cur)
    torch.cuda.synchronize()
    eus = e0.elapsed_time(e1) * 1e3 / ne
    h2d = sets[0][0].numel() * 4 + sets[0][1].numel() * 2 + sets[0][2].numel() * 2
    d2h = T * H * 512 * 2 + T * H * 4
    return {"value": flop / (eus * 1e-6) / 1e12 * world, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "us_per_step": eus, "copies_declared": True,
            "api": "nvfp4_sparse_mla_decode_host (pinned host in/out, copies inside the call)",
            "overlap": "%d streams, one set of device buffers each" % N_E2E_STREAMS}


def configs_leg(nv, synth, args):
    """Every other parity configuration, timed as single launches with L2
    flushed before each (median of 20): us/launch, TFLOP/s, gathered GB/s and
    the fraction of the roofline at the measured peaks."""
    import torch
    res = {}
    for name, make in config_workloads(synth):
        r = time_other_workload(name, make(), nv, synth, args)
        res[name] = {k: r[k] for k in ("T", "H", "valid_rows_per_launch", "splits", "us_per_launch", "tflops",
                                        "gathered_gbs", "roofline_us", "frac_of_roofline")}
        torch.cuda.empty_cache()
    return res


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    if args.workload != "decode35x64":
        return other_workloads(args) if rank == 0 else None

    import torch
    import torch.distributed as tdist
    import nvfp4_sparse_mla_decode_b200 as nv
    from nvfp4_sparse_mla_decode_b200 import synth

    assert torch.cuda.is_available(), "bench.py needs a CUDA GPU"
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    nv.lib()  # fails loudly if the library is missing

    # ------------------------------------------------------------ workload
    w = synth.decode35("cuda", seed=1 + 1000 * rank, ctx=args.ctx)
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    t_build = time.perf_counter()
    cache = build_cache(w)
    torch.cuda.synchronize()
    t_build = time.perf_counter() - t_build
    sets = [(w.indices, w.q_nope, w.q_rope)] + [synth.redraw(w, 100 + k + 1000 * rank) for k in range(N_SETS - 1)]
    rows, flop, alg_bytes = workload_stats([s[0] for s in sets], w.T, w.H)
    T, H, topk = w.T, w.H, 2048
    out = torch.empty(T, H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(1, nv.workspace_size(T, H, topk)), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    launches_per_step = 1  # the split merge runs inside the decode kernel

    def step(k):
        ix, qn, qr = sets[k % N_SETS]
        nv.decode(qn, qr, cache, ix, w.sm_scale, out=out, lse=lse, workspace=ws, dev_status=status)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()

    # The K timed launches: a CUDA graph holding one launch per rotating set,
    # replayed K // N_SETS times, then the K % N_SETS remaining launches --
    # exactly K launches of the same kernel on the same stream.
    graph = None
    if args.launch == "graph":
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for k in range(N_SETS):
                step(k)
        graph.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()

    def timed_launches(n):
        if graph is None:
            for k in range(n):
                step(k)
            return
        for _ in range(n // N_SETS):
            graph.replay()
        for k in range(n % N_SETS):
            step(k)

    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        tdist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.perf_counter()
    e0.record(stream)
    timed_launches(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    if world > 1:
        tdist.barrier()
    sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    sec_per = ms * 1e-3 / args.steps
    tflops = job_tflops(flop, ms, args.steps, world)
    us = sec_per * 1e6
    peaks, peak_kind = measured_peaks()
    peak_tf = float(peaks["bf16_tflops"])    # FP16 and BF16 share the nominal dense rate
    peak_bw = float(peaks["hbm_gbs"])
    t_roof = max(flop / (peak_tf * 1e12), alg_bytes / (peak_bw * 1e9))
    clocks = sampler.summary(h0, h1)
    # for reference: the same launches issued one by one from the host
    n_stream = min(args.steps, 2000)
    torch.cuda.synchronize()
    e0.record(stream)
    for k in range(n_stream):
        step(k)
    e1.record(stream)
    torch.cuda.synchronize()
    stream_us = e0.elapsed_time(e1) * 1e3 / n_stream

    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": "decode35x64", "T": T, "H": H, "topk": topk, "ctx_rows": args.ctx,
                   "cache_rows": w.num_slots, "valid_rows_per_launch": rows, "splits": nv.num_splits(T, H, topk),
                   "l2": "inputs larger than L2: %d rotating index/query sets, %.0f MB gathered per cycle > %d MB L2"
                         % (N_SETS, N_SETS * rows * ROW_BYTES / 1e6, L2_BYTES >> 20),
                   "parallelism": "replicas" if world > 1 else "single",
                   "launch": "cuda_graph" if graph is not None else "stream"},
        "us_per_launch": us,
        "us_per_launch_stream_issued": stream_us,
        "gathered_gbs": rows * ROW_BYTES / sec_per / 1e9,
        "alg_bytes_per_launch": alg_bytes, "alg_flop_per_launch": flop,
        "roofline": {"bound": "tensor", "achieved": flop / sec_per / 1e12, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": (flop / sec_per / 1e12) / peak_tf,
                     "traffic": kernel_traffic(os.path.join(ROOT, "nvfp4_sparse_mla_decode_b200", "csrc", "decode_nvfp4.cu")),
                     "peak_source": "%s bf16_tflops (burst) from MEASURED_PEAKS.json" % peak_kind
                                    if peak_kind == "measured" else "fallback 1590 TFLOP/s",
                     "roofline_us": t_roof * 1e6, "frac_of_roofline_time": t_roof / sec_per,
                     "mem_bound_us": alg_bytes / (peak_bw * 1e9) * 1e6, "hbm_peak_gbs": peak_bw},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cache_build_s": t_build,
    }

    if not args.no_extras:
        line["staged_fp8"] = staged_leg(nv, w, cache, sets, rows, flop, us, peak_bw, args)
        line["e2e"] = e2e_leg(nv, w, cache, sets, flop, world, args)
        # ----------------------------------------------------------- append
        wa = synth.append_prefill("cuda")
        acache = torch.zeros(wa.num_slots, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        for _ in range(3):
            nv.kv_append(wa.new_lat, wa.new_rope, wa.new_slots, acache)
        ta = []
        for _ in range(20):
            flush.fill_(1)
            e0.record(stream)
            nv.kv_append(wa.new_lat, wa.new_rope, wa.new_slots, acache)
            e1.record(stream)
            torch.cuda.synchronize()
            ta.append(e0.elapsed_time(e1) * 1e3)
        aus = statistics.median(ta)
        abytes = wa.T * (1152 + 352 + 4)
        line["append"] = {"rows": wa.T, "us_per_launch": aus, "gbs": abytes / (aus * 1e-6) / 1e9,
                          "frac_of_hbm": abytes / (aus * 1e-6) / 1e9 / peak_bw, "l2": "flushed before each launch"}
        del acache, flush
        # ---------------------------------------------------- cpu baseline
        if rank == 0:
            try:
                rate, passes, secs, cores = oracle_passes(w, 10.0)
                line["cpu_baseline"] = {
                    "value": rate / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                    "sample": "%d passes over all %d tokens of decode35x64 (H=64, 2048 rows each), FP64 oracle "
                              "incl. row dequantization, %.1f s" % (passes, T, secs)}
            except Exception as e:  # noqa: BLE001
                line["cpu_baseline"] = {"value": None, "unit": "TFLOP/s", "cores": None, "kind": "oracle",
                                        "sample": "oracle unavailable: %s" % e}
    if not args.no_extras and rank == 0:
        line["configs"] = configs_leg(nv, synth, args)
        line["configs_timing"] = "single launch per config, L2 flushed before it, median of 20"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Throughput of MLA latent-KV decode on B200: one step = mla_decode_plan +
mla_decode + mla_combine over one batch of the workload (default: V3 shapes,
B=64, H=128, ragged KV lengths 1k-32k).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C3] [--impl reference]

Prints one JSON line (rank 0). Under torchrun (N > 1) every rank decodes its
own copy of the batch (replicas: the path has no cross-GPU exchange), so the
job's KV-tokens/s is N x the batch over the slowest rank's time.

The CPU float64 oracle is timed here as a reported baseline (``cpu_baseline``
and ``--impl reference``) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_latent_kv_26_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MLA decode KV-tokens/s and achieved TB/s / TFLOP/s as fraction of roofline"
UNIT = "KV-tokens/s"
BYTES_PER_TOKEN = 576 * 2       # one cached row: c_kv[512] + k_pe[64], bf16
FLOPS_PER_ROW_TOKEN = 2 * (576 + 512)  # QK^T over 576 + PV over 512, multiply-add = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- accounting


def accounting(inp: dict, row_bytes: int = BYTES_PER_TOKEN) -> dict:
    """Algorithmic work of one step (no split partials, no re-reads); a cached
    row is ``row_bytes`` (1152 bf16, 656 in the fp8 cache format)."""
    lens = [int(x) for x in inp["seq_lens"]]
    B, Sq, H, topk = inp["batch"], inp["q_len"], inp["heads"], inp["topk"]
    kv_tokens = 0          # distinct cache rows read per sequence
    row_tokens = 0         # sum over (b, i) of visible tokens; x H for score rows
    table_bytes = 0
    for b, L in enumerate(lens):
        if topk > 0:
            idx = inp["indices"][b]
            uniq = int(torch.unique(idx[idx >= 0]).numel())
            kv_tokens += uniq
            row_tokens += int((idx >= 0).sum())
            table_bytes += idx.numel() * 4 + uniq * 4
        else:
            per_q = [max(L - Sq + i + 1, 0) if inp["causal"] else L for i in range(Sq)]
            kv_tokens += max(per_q) if per_q else 0
            row_tokens += sum(per_q)
            table_bytes += ((max(per_q) + 63) // 64) * 4
    rows = B * Sq * H
    bytes_ = kv_tokens * row_bytes + rows * 576 * 2 + rows * 512 * 2 + rows * 4 + table_bytes + B * 4
    flops = row_tokens * H * FLOPS_PER_ROW_TOKEN
    return {"kv_tokens": kv_tokens, "row_tokens": row_tokens, "bytes": bytes_, "flops": flops,
            "h2d_bytes": rows * 576 * 2 + inp["block_table"].numel() * 4 + B * 4 +
            (inp["indices"].numel() * 4 if inp["indices"] is not None else 0),
            "d2h_bytes": rows * 512 * 2 + rows * 4}


L2_NOMINAL_BYTES = 126 * 1024 * 1024  # B200 L2, used when no device is visible (CPU reference arm)


def l2_bytes_of(dev=None) -> int:
    if dev is not None:
        return int(torch.cuda.get_device_properties(dev).L2_cache_size)
    if torch.cuda.is_available():
        return int(torch.cuda.get_device_properties(0).L2_cache_size)
    return L2_NOMINAL_BYTES


def decode_config(inp: dict, acc: dict, n_gpus: int, l2_bytes: int, cache: str = "bf16") -> dict:
    """The ``config`` object of the decode line; both arms print the same one."""
    w = inp["workload"]
    flush = acc["bytes"] < 2 * l2_bytes
    name = f"{w.key} {w.name}" + ("" if cache == "bf16" else " fp8-cache (656 B per token)")
    return {"workload": name, "batch": w.batch, "q_len": w.q_len, "heads": w.heads,
            "kv_len": f"{w.len_lo}..{w.len_hi}" + (f" top{w.topk}" if w.topk else ""),
            "kv_tokens_per_step": acc["kv_tokens"], "bytes_per_step": acc["bytes"],
            "flops_per_step": acc["flops"], "seed": w.seed,
            "l2": (f"{acc['bytes'] / 1e6:.0f} MB read per step, within 2x L2 ({l2_bytes / 1e6:.0f} MB): "
                   f"L2 flushed by a {2 * l2_bytes / 1e6:.0f} MB write before every timed step")
            if flush else f"inputs larger than 2x L2 ({acc['bytes'] / 1e6:.0f} MB read per step), no flush",
            "parallelism": f"replicas x{n_gpus}"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(files) -> str:
    """First 16 hex digits of the sha256 of the kernel's source files, in order."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "mla_latent_kv_26_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from
    profiles/traffic.json, if that capture was taken on the current kernel
    source; else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f).get(f"{kernel}/{workload}")
    except (OSError, ValueError):
        return None
    if not entry or entry.get("source_sha") != source_sha(entry["sources"]):
        return None
    return int(entry["dram_bytes_per_launch"])


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device: int, interval_s: float = 0.01):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        self.interval = interval_s
        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # no NVML: report it
            self.nv = None
            self.error = f"nvml unavailable: {e}"

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = int(self._get_reasons(self.h))
                self.samples.append(mhz)
                self.reasons |= r
            except Exception as e:
                self.error = str(e)
            time.sleep(self.interval)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.error or "no samples"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle arm


def oracle_sample(inp: dict, budget_s: float):
    """Time the float64 oracle on whole sequences of the batch until the budget
    is used; returns (kv_tokens, seconds, sequences)."""
    import oracle

    t0 = time.perf_counter()
    toks, done = 0, 0
    order = list(range(inp["batch"]))
    for b in order:
        oracle.mla_decode(inp["q"], inp["cache"], inp["block_table"], inp["seq_lens"], causal=inp["causal"],
                          indices=inp["indices"], batches=[b])
        L = int(inp["seq_lens"][b])
        toks += min(inp["topk"], L) if inp["topk"] else L
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return toks, time.perf_counter() - t0, done


def run_reference(args, inp, rank, row_bytes=BYTES_PER_TOKEN):
    if rank != 0:
        return
    if inp["cache"].dtype == torch.uint8:
        import oracle

        inp = dict(inp, cache=oracle.dequantize_cache(inp["cache"]))  # what a decode over the fp8 cache computes with
    torch.set_num_threads(os.cpu_count() or 1)
    # each step: the oracle on a bounded slice (two sequences) of the batch
    per_step = []
    toks_total, secs_total = 0, 0.0
    order = list(range(inp["batch"]))
    for s in range(args.warmup + args.steps):
        import oracle

        bs = [order[(2 * s) % len(order)], order[(2 * s + 1) % len(order)]]
        t0 = time.perf_counter()
        oracle.mla_decode(inp["q"], inp["cache"], inp["block_table"], inp["seq_lens"], causal=inp["causal"],
                          indices=inp["indices"], batches=bs)
        dt = time.perf_counter() - t0
        toks = sum(min(inp["topk"], int(inp["seq_lens"][b])) if inp["topk"] else int(inp["seq_lens"][b]) for b in bs)
        if s >= args.warmup:
            toks_total += toks
            secs_total += dt
            per_step.append(dt)
    value = toks_total / secs_total if secs_total > 0 else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs_total / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(inp, accounting(inp, row_bytes), args.gpus, l2_bytes_of(), args.cache),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": "float64 CPU oracle, two whole sequences of the batch per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ranks


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of per-rank timings over all ranks (the job is as
    slow as its slowest rank); identity for a single process."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_value(world: int, kv_tokens: int, ms_per_step: float) -> float:
    """Whole-job KV tokens per second: every rank decodes its own replica of
    the step's batch, timed by the slowest rank."""
    return world * kv_tokens / (ms_per_step / 1e3)


# ---------------------------------------------------------------- cache insert (--op insert)

INSERT_METRIC = "MLA latent-cache insert tokens/s (kv_norm + RoPE + paged write) and achieved GB/s vs HBM roofline"
INSERT_UNIT = "tokens/s"


def insert_accounting(d: dict) -> dict:
    """Algorithmic bytes of one insert: per token its input row (1152 B), its
    cache row (1152 B), sequence id and position (8 B); per distinct position
    one cos/sin row (256 B); per distinct (sequence, page) one block-table
    entry; the weight once."""
    n = int(d["kv"].shape[0])
    pos = d["positions"].to(torch.int64)
    pages = torch.unique(d["seq_ids"].to(torch.int64) * (1 << 32) + pos // 64).numel()
    bytes_ = n * (2 * 576 * 2 + 8) + torch.unique(pos).numel() * 256 + pages * 4 + 1024
    return {"tokens": n, "bytes": int(bytes_), "h2d_bytes": n * (576 * 2 + 8), "d2h_bytes": 4}


def insert_oracle_sample(d: dict, budget_s: float):
    """The oracle's insert on the tokens of sequence 0 (one page, 64 tokens, per
    call; wrapping round to its start) until the budget is used; returns
    (tokens, seconds)."""
    import oracle

    t0, done = time.perf_counter(), 0
    n0 = int((d["seq_ids"] == 0).sum())
    while time.perf_counter() - t0 < budget_s:
        i = done % n0
        k = min(64 - i % 64, n0 - i)
        base = (i // 64) * 64
        page = int(d["block_table"][0, i // 64])
        oracle.cache_insert(d["cache"][page:page + 1], torch.zeros(1, 1, dtype=torch.int32),
                            torch.zeros(k, dtype=torch.int32), d["positions"][i:i + k] - base, d["kv"][i:i + k],
                            d["weight"], 1e-6, d["cos"][base:], d["sin"][base:])
        done += k
    return done, time.perf_counter() - t0


def run_insert_bench(args, world, rank, local):
    from mla_latent_kv_26_b200.workloads import insert_inputs

    B, T = args.insert_batch, args.insert_tokens
    d = insert_inputs(lens=[T] * B, new_tokens=[T] * B, seed=5)
    acc = insert_accounting(d)
    name = f"insert-b{B}-prefill{T}"
    cfg = {"workload": f"{name}: {B} sequences x {T} new tokens (positions 0..{T - 1}), 576-wide rows",
           "tokens_per_step": acc["tokens"], "bytes_per_step": acc["bytes"]}
    if args.impl == "reference":
        if rank != 0:
            return
        torch.set_num_threads(os.cpu_count() or 1)
        secs, toks = 0.0, 0
        for s in range(args.warmup + args.steps):
            n, dt = insert_oracle_sample(d, 0.5)
            if s >= args.warmup:
                toks, secs = toks + n, secs + dt
        v = toks / secs
        print(json.dumps({
            "impl": "reference", "metric": INSERT_METRIC, "value": v, "unit": INSERT_UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": v, "unit": INSERT_UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
                             "sample": "float64 oracle insert, about 0.5 s of tokens of sequence 0 per step"},
            "e2e": {"value": v, "unit": INSERT_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return

    import torch.distributed as dist

    from mla_latent_kv_26_b200.decoder import cache_insert

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(kv, seq, pos, st):
        cache_insert(kv, g["weight"], g["cos"], g["sin"], seq, pos, g["block_table"], g["cache"], error_word=err,
                     stream=st)

    # Steady state, no L2 flush: a step reads and writes more than the L2
    # holds, and back-to-back steps each pay for the write-back of the rows
    # the previous one left dirty in L2 (a flush by writing a large buffer
    # would instead charge the step with the flush buffer's write-back).
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    for _ in range(args.warmup):
        step(g["kv"], g["seq_ids"], g["positions"], stream)
    torch.cuda.synchronize(dev)
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local, interval_s=0.002)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    with sampler:
        e0.record(stream)
        for i in range(K):
            step(g["kv"], g["seq_ids"], g["positions"], stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier(device_ids=[local])
    (ms,) = max_over_ranks([e0.elapsed_time(e1) / K], world, dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"insert flagged bad tokens: {int(err.item()):#x}")

    # end to end: the new rows, sequence ids and positions copied in from
    # pinned host memory every step, the error word read back
    host = {k: d[k].pin_memory() for k in ("kv", "seq_ids", "positions")}
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    host_err = torch.zeros(1, dtype=torch.int32).pin_memory()
    K2 = max(3, min(K, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K2):
        for k, v in host.items():
            dev_in[k].copy_(v, non_blocking=True)
        step(dev_in["kv"], dev_in["seq_ids"], dev_in["positions"], stream)
        host_err.copy_(err, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / K2], world, dev)

    peaks, peak_src = load_peaks()
    gbs = acc["bytes"] / (ms / 1e3) / 1e9
    line = {
        "metric": INSERT_METRIC, "value": world * acc["tokens"] / (ms / 1e3), "unit": INSERT_UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(cfg, l2=f"no flush: {acc['bytes'] / 1e6:.0f} MB moved per step against a {l2 / 1e6:.0f} MB "
                                f"L2; back-to-back steps, each paying the previous one's write-backs",
                       parallelism=f"replicas x{world}"),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "kernel": "mla_insert_kernel",
                     "traffic": profiled_traffic("mla_insert_kernel", f"prefill{B}x{T}"),
                     "peak_source": peak_src},
        "e2e": {"value": world * acc["tokens"] / (e2e_ms / 1e3), "unit": INSERT_UNIT,
                "h2d_bytes_per_step": acc["h2d_bytes"], "d2h_bytes_per_step": acc["d2h_bytes"], "ms_per_step": e2e_ms},
        "gpu_launches": K,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1:
        torch.set_num_threads(os.cpu_count() or 1)
        n, secs = insert_oracle_sample(d, args.cpu_budget)
        line["cpu_baseline"] = {"value": n / secs, "unit": INSERT_UNIT, "cores": torch.get_num_threads(),
                                "kind": "oracle",
                                "sample": f"{n} tokens of sequence 0 (wrapping round), float64, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- absorb / un-absorb (--op absorb)

ABSORB_METRIC = "MLA absorb + un-absorb projection tokens/s (W_UK^T q_nope, W_UV o_lat) and achieved GB/s vs HBM roofline"


def absorb_accounting(T: int, H: int) -> dict:
    """Algorithmic bytes of one absorb + un-absorb pass: both weight halves
    once, q [T,H,192] and q_abs [T,H,576] (absorb), o_lat [T,H,512] and out
    [T,H,128] (un-absorb)."""
    w = H * 128 * 512 * 2
    absorb = w + T * H * (192 + 576) * 2
    unabsorb = w + T * H * (512 + 128) * 2
    flops = 2 * T * H * 128 * 512 * 2
    return {"absorb": absorb, "unabsorb": unabsorb, "bytes": absorb + unabsorb, "flops": flops,
            "h2d_bytes": T * H * (192 + 512) * 2, "d2h_bytes": T * H * (576 + 128) * 2}


def absorb_oracle_sample(d: dict, budget_s: float):
    import oracle

    t0, done = time.perf_counter(), 0
    w_uk, w_uv = d["wkv_b"][:, :128, :], d["wkv_b"][:, 128:, :]
    while time.perf_counter() - t0 < budget_s:
        t = done % d["tokens"]
        oracle.absorb_query(d["q"][t, :, :128], w_uk)
        oracle.unabsorb_output(d["o_lat"][t], w_uv)
        done += 1
    return done, time.perf_counter() - t0


def run_absorb_bench(args, world, rank, local):
    from mla_latent_kv_26_b200.workloads import absorb_inputs

    T, H = args.absorb_tokens, 128
    d = absorb_inputs(tokens=T, heads=H, seed=6)
    acc = absorb_accounting(T, H)
    cfg = {"workload": f"absorb-t{T}-h{H}: {T} decode tokens x {H} heads, wkv_b [H,256,512] bf16",
           "tokens_per_step": T, "bytes_per_step": acc["bytes"], "flops_per_step": acc["flops"]}
    if args.impl == "reference":
        if rank != 0:
            return
        torch.set_num_threads(os.cpu_count() or 1)
        toks, secs = 0, 0.0
        for s in range(args.warmup + args.steps):
            n, dt = absorb_oracle_sample(d, 0.2)
            if s >= args.warmup:
                toks, secs = toks + n, secs + dt
        v = toks / secs
        print(json.dumps({
            "impl": "reference", "metric": ABSORB_METRIC, "value": v, "unit": INSERT_UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": v, "unit": INSERT_UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
                             "sample": "float64 oracle projections, about 0.2 s of tokens per step"},
            "e2e": {"value": v, "unit": INSERT_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return

    import torch.distributed as dist

    from mla_latent_kv_26_b200.decoder import absorb_query, unabsorb_output

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    q_abs = torch.empty(T, H, 576, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # The weights (33.5 MB) fit in L2: before every timed step the L2 is
    # flushed by READING a buffer twice its size, which leaves it full of clean
    # lines (a flush by writing would charge the step with the write-back of
    # the flush buffer's dirty lines).
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.ones(2 * l2 // 4, dtype=torch.float32, device=dev)
    sink = torch.empty(1, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        absorb_query(g["q"], g["wkv_b"], q_abs, error_word=err)
        unabsorb_output(g["o_lat"], g["wkv_b"], out, error_word=err)
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(K)]
    sampler = ClockSampler(local, interval_s=0.002)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    with sampler:
        for i in range(K):
            torch.sum(flush_buf, dim=0, out=sink)
            ev[i][0].record(stream)
            absorb_query(g["q"], g["wkv_b"], q_abs, error_word=err)
            ev[i][1].record(stream)
            unabsorb_output(g["o_lat"], g["wkv_b"], out, error_word=err)
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier(device_ids=[local])
    a_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    u_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    ms = sum(e[0].elapsed_time(e[2]) for e in ev) / K
    ms, a_ms, u_ms = max_over_ranks([ms, a_ms, u_ms], world, dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item()):#x}")

    # end to end: q and o_lat from pinned host memory, q_abs and out back, every step
    hq, ho = d["q"].pin_memory(), d["o_lat"].pin_memory()
    hqa = torch.empty(T, H, 576, dtype=torch.bfloat16).pin_memory()
    hout = torch.empty(T, H, 128, dtype=torch.bfloat16).pin_memory()
    dq, do = torch.empty_like(g["q"]), torch.empty_like(g["o_lat"])
    K2 = max(3, min(K, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K2):
        dq.copy_(hq, non_blocking=True)
        do.copy_(ho, non_blocking=True)
        absorb_query(dq, g["wkv_b"], q_abs, error_word=err)
        unabsorb_output(do, g["wkv_b"], out, error_word=err)
        hqa.copy_(q_abs, non_blocking=True)
        hout.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / K2], world, dev)

    peaks, peak_src = load_peaks()
    gbs = acc["bytes"] / (ms / 1e3) / 1e9
    a_gbs = acc["absorb"] / (a_ms / 1e3) / 1e9
    u_gbs = acc["unabsorb"] / (u_ms / 1e3) / 1e9
    line = {
        "metric": ABSORB_METRIC, "value": world * T / (ms / 1e3), "unit": INSERT_UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict(cfg, l2=f"L2 flushed before every timed step by reading a {2 * l2 / 1e6:.0f} MB buffer",
                       parallelism=f"replicas x{world}"),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "kernel": "mla_absorb_q_kernel + mla_unabsorb_o_kernel", "peak_source": peak_src,
                     "absorb_us": a_ms * 1e3, "absorb_frac": a_gbs / peaks["hbm_gbs"],
                     "unabsorb_us": u_ms * 1e3, "unabsorb_frac": u_gbs / peaks["hbm_gbs"],
                     "tflop_per_s": acc["flops"] / (ms / 1e3) / 1e12},
        "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": INSERT_UNIT, "h2d_bytes_per_step": acc["h2d_bytes"],
                "d2h_bytes_per_step": acc["d2h_bytes"], "ms_per_step": e2e_ms},
        "gpu_launches": 2 * K,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1:
        torch.set_num_threads(os.cpu_count() or 1)
        n, secs = absorb_oracle_sample(d, args.cpu_budget)
        line["cpu_baseline"] = {"value": n / secs, "unit": INSERT_UNIT, "cores": torch.get_num_threads(),
                                "kind": "oracle", "sample": f"{n} tokens (absorb + un-absorb), float64, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- indexer + top-k (--op indexer)

INDEXER_METRIC = ("sparse-attention indexer keys/s (fp8 index scores + exact top-k) and achieved GB/s vs HBM "
                  "roofline")
INDEXER_UNIT = "keys/s"


def indexer_accounting(b: int, m: int, h: int, n: int, k: int) -> dict:
    """Algorithmic bytes: the scores kernel reads q, q_s, k and k_s once and
    writes the scores; the top-k reads the scores and writes the positions."""
    scores = b * m * h * 128 + 4 * b * m * h + b * n * 128 + 4 * b * n + 4 * b * m * n
    topk = 4 * b * m * n + 4 * b * m * k
    flops = 2 * b * m * h * n * 128
    return {"scores": scores, "topk": topk, "bytes": scores + topk, "flops": flops, "keys": b * m * n,
            "h2d_bytes": b * m * h * (128 + 4), "d2h_bytes": 4 * b * m * k}


def indexer_oracle_sample(d: dict, k: int, budget_s: float):
    """The oracle's scores and top-k for whole query rows until the budget is
    used; returns (keys scored, seconds)."""
    import oracle

    t0, done, r = time.perf_counter(), 0, 0
    while time.perf_counter() - t0 < budget_s:
        b = r % d["batch"]
        sc = oracle.index_scores(d["q"][b:b + 1], d["q_s"][b:b + 1], d["k"][b:b + 1], d["k_s"][b:b + 1])
        oracle.topk_positions(sc.view(-1, d["num_keys"]), k)
        done += d["q_len"] * d["num_keys"]
        r += 1
    return done, time.perf_counter() - t0


def run_indexer_bench(args, world, rank, local):
    from mla_latent_kv_26_b200.workloads import indexer_inputs

    b, m, h, n, K = 16, 1, 64, 131072, 2048
    d = indexer_inputs(batch=b, q_len=m, heads=h, num_keys=n, seed=8)
    acc = indexer_accounting(b, m, h, n, K)
    cfg = {"workload": f"indexer-b{b}-m{m}-h{h}-n{n}-top{K}: fp8 index scores of {n} keys for {b} sequences, "
                       f"{h} index heads of 128, then the top {K} positions per query",
           "keys_per_step": acc["keys"], "bytes_per_step": acc["bytes"], "flops_per_step": acc["flops"],
           "l2": f"inputs larger than 2x L2 ({acc['bytes'] / 1e6:.0f} MB moved per step), no flush",
           "parallelism": f"replicas x{args.gpus if args.impl == 'reference' else world}"}
    if args.impl == "reference":
        if rank != 0:
            return
        torch.set_num_threads(os.cpu_count() or 1)
        keys, secs = 0, 0.0
        for s in range(args.warmup + args.steps):
            kk, dt = indexer_oracle_sample(d, K, 0.3)
            if s >= args.warmup:
                keys, secs = keys + kk, secs + dt
        v = keys / secs
        print(json.dumps({
            "impl": "reference", "metric": INDEXER_METRIC, "value": v, "unit": INDEXER_UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": v, "unit": INDEXER_UNIT, "cores": torch.get_num_threads(), "kind": "oracle",
                             "sample": "float64 oracle scores + top-k of whole query rows, about 0.3 s per step"},
            "e2e": {"value": v, "unit": INDEXER_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return

    import torch.distributed as dist

    from mla_latent_kv_26_b200 import binding as Bd

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    g = {key: (v.to(dev) if isinstance(v, torch.Tensor) else v) for key, v in d.items()}
    scores = torch.empty(b, m, n, dtype=torch.float32, device=dev)
    idx = torch.empty(b * m, K, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lens = torch.full((b * m,), n, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sdesc = Bd.make_index_desc(batch=b, q_len=m, num_heads=h, num_keys=n)
    tdesc = Bd.make_topk_desc(rows=b * m, num_keys=n, k=K)

    def step(q, q_s, ev=None, st=stream):
        if ev is not None:
            ev[0].record(st)
        Bd.check(Bd.mla_index_scores(sdesc, q, q_s, g["k"], g["k_s"], scores, err, st), "mla_index_scores")
        if ev is not None:
            ev[1].record(st)
        Bd.check(Bd.mla_topk(tdesc, scores, lens, idx, st), "mla_topk")
        if ev is not None:
            ev[2].record(st)

    for _ in range(args.warmup):
        step(g["q"], g["q_s"])
    torch.cuda.synchronize(dev)
    K_steps = args.steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(K_steps)]
    sampler = ClockSampler(local, interval_s=0.002)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize(dev)
    with sampler:
        for i in range(K_steps):
            step(g["q"], g["q_s"], ev[i])
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier(device_ids=[local])
    s_ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    t_ms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    ms = sum(e[0].elapsed_time(e[2]) for e in ev) / K_steps
    ms, s_ms, t_ms = max_over_ranks([ms, s_ms, t_ms], world, dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item()):#x}")

    # end to end: the step's queries and weights in from pinned host memory,
    # the chosen positions back, every step (the key cache stays resident)
    hq, hqs = d["q"].pin_memory(), d["q_s"].pin_memory()
    hidx = torch.empty(b * m, K, dtype=torch.int32).pin_memory()
    dq, dqs = torch.empty_like(g["q"]), torch.empty_like(g["q_s"])
    K2 = max(3, min(K_steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K2):
        dq.copy_(hq, non_blocking=True)
        dqs.copy_(hqs, non_blocking=True)
        step(dq, dqs)
        hidx.copy_(idx, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / K2], world, dev)

    peaks, peak_src = load_peaks()
    s_gbs = acc["scores"] / (s_ms / 1e3) / 1e9
    t_gbs = acc["topk"] / (t_ms / 1e3) / 1e9
    line = {
        "metric": INDEXER_METRIC, "value": world * acc["keys"] / (ms / 1e3), "unit": INDEXER_UNIT, "n_gpus": world,
        "steps": K_steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 in, f32 accumulate", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "hbm", "achieved": s_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": s_gbs / peaks["hbm_gbs"], "kernel": "mla_index_kernel",
                     "traffic": profiled_traffic("mla_index_kernel", f"b{b}n{n}"), "peak_source": peak_src,
                     "scores_us": s_ms * 1e3, "topk_us": t_ms * 1e3, "topk_gbs": t_gbs,
                     "tflop_per_s": acc["flops"] / (s_ms / 1e3) / 1e12},
        "e2e": {"value": world * acc["keys"] / (e2e_ms / 1e3), "unit": INDEXER_UNIT,
                "h2d_bytes_per_step": acc["h2d_bytes"], "d2h_bytes_per_step": acc["d2h_bytes"], "ms_per_step": e2e_ms},
        "gpu_launches": 2 * K_steps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1:
        torch.set_num_threads(os.cpu_count() or 1)
        kk, secs = indexer_oracle_sample(d, K, args.cpu_budget)
        line["cpu_baseline"] = {"value": kk / secs, "unit": INDEXER_UNIT, "cores": torch.get_num_threads(),
                                "kind": "oracle", "sample": f"{kk} keys (whole query rows), float64, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------- GPU arm


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="C3", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="libmla", choices=["libmla", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--profile", action="store_true", help="kernel launches only (for ncu): no e2e/oracle/clocks")
    ap.add_argument("--num-sms", type=int, default=0)
    ap.add_argument("--e2e-lanes", type=int, default=4, help="decoders / streams the end-to-end steps rotate over")
    ap.add_argument("--op", default="decode", choices=["decode", "insert", "absorb", "indexer"],
                    help="decode: the decode step (default); insert: the latent-cache insert alone; "
                         "absorb: the absorb + un-absorb projections; indexer: fp8 index scores + top-k")
    ap.add_argument("--absorb-tokens", type=int, default=64, help="query tokens for --op absorb")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="decode: the latent cache format (fp8: e4m3 codes + per-token scale, 656 B per token)")
    ap.add_argument("--insert-batch", type=int, default=64)
    ap.add_argument("--insert-tokens", type=int, default=1024, help="new tokens per sequence for --op insert")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        args.gpus = world

    if args.op == "insert":
        run_insert_bench(args, world, rank, local)
        return
    if args.op == "absorb":
        run_absorb_bench(args, world, rank, local)
        return
    if args.op == "indexer":
        run_indexer_bench(args, world, rank, local)
        return

    inp = make_inputs(args.workload)
    row_bytes = BYTES_PER_TOKEN
    if args.cache == "fp8":
        from mla_latent_kv_26_b200.workloads import make_fp8_cache

        inp["cache"] = make_fp8_cache(inp)  # [pages, 64, 656] uint8 replaces the bf16 cache
        row_bytes = 656

    if args.impl == "reference":
        run_reference(args, inp, rank, row_bytes)
        return

    import torch.distributed as dist

    from mla_latent_kv_26_b200.decoder import decoder_for

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    acc = accounting(inp, row_bytes)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    dec = decoder_for(inp, num_sms=args.num_sms, device=dev)
    stream = torch.cuda.current_stream(dev)

    # ev: events recorded before plan, before decode, after decode, after combine
    def step(ev=None, st=None):
        st = stream if st is None else st
        if ev is not None:
            ev[0].record(st)
        dec.plan_step(g["seq_lens"], st)
        if ev is not None:
            ev[1].record(st)
        dec.decode_step(g["q"], g["cache"], g["block_table"], g["seq_lens"], g["indices"], st)
        if ev is not None:
            ev[2].record(st)
        dec.combine_step(st)
        if ev is not None:
            ev[3].record(st)

    # Inputs within twice the L2 size are flushed from L2 before every timed
    # step (a write of a buffer twice the L2 size, outside the step's events).
    l2_bytes = l2_bytes_of(dev)
    flush_l2 = acc["bytes"] < 2 * l2_bytes
    flush_buf = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) if flush_l2 else None

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, bits = dec.error(stream)
    if st != 0:
        raise RuntimeError(f"device error after warm-up: status {st} bits {bits:#x}")

    K = args.steps
    sampler = ClockSampler(local) if not args.profile else None

    # K timed steps. Every other step also records an event between every two
    # kernels (each such event adds a launch gap, so the other steps carry
    # none); those steps give each kernel's own time (median), in the same run
    # and thermal state as the headline.
    SAMPLE = 2
    sampled = [i for i in range(K) if i % SAMPLE == 0]
    kev = {i: tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for i in sampled}
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.__enter__()
    t_start.record(stream)
    for i in range(K):
        if flush_l2:
            flush_buf.fill_(i & 0xFF)
            sev[i][0].record(stream)
        step(kev.get(i))
        if flush_l2:
            sev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.__exit__(None, None, None)
    barrier()
    # with the L2 flush, the timed work is the sum of the steps' own intervals
    elapsed_ms = sum(a.elapsed_time(b) for a, b in sev) if flush_l2 else t_start.elapsed_time(t_end)
    plan_ms = statistics.median(e[0].elapsed_time(e[1]) for e in kev.values())
    decode_ms = statistics.median(e[1].elapsed_time(e[2]) for e in kev.values())
    combine_ms = statistics.median(e[2].elapsed_time(e[3]) for e in kev.values())
    elapsed_ms, decode_ms, plan_ms, combine_ms = max_over_ranks([elapsed_ms, decode_ms, plan_ms, combine_ms], world, dev)
    ms_per_step = elapsed_ms / K

    # 100 more steps, each with an event between every two kernels, right
    # after the timed region (not part of the headline): per-kernel medians of 100
    K100 = 100
    kev100 = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(K100)]
    barrier()
    for i in range(K100):
        if flush_l2:
            flush_buf.fill_(i & 0xFF)
        step(kev100[i])
    torch.cuda.synchronize(dev)
    barrier()
    med100 = [statistics.median(e[a].elapsed_time(e[a + 1]) for e in kev100) for a in range(3)]
    med100 = max_over_ranks(med100, world, dev)

    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": ms_per_step, "decode_ms": decode_ms}))
        if world > 1:
            dist.destroy_process_group()
        return

    # ---- end to end through the public API with pinned host buffers: every
    # step copies its inputs in and its output and LSE back. Consecutive steps
    # rotate over --e2e-lanes decoders on as many streams, so one step's
    # copies overlap the neighbouring steps' kernels (as a caller decoding
    # step after step would run it); each stream keeps its own device
    # buffers. A lane runs copy in -> kernels -> copy out in order, so with L
    # lanes a step costs at least (copy in + kernels + copy out) / L: two
    # lanes leave the step copy-bound on C3 (564 us against 401 us of
    # kernels), three make it kernel-bound (393 us); small workloads, whose
    # copies outweigh their kernels, still gain from a fourth (C5: 172, 109,
    # 89 us).
    host_in = {k: inp[k].pin_memory() for k in ("q", "block_table", "seq_lens")}
    if inp["indices"] is not None:
        host_in["indices"] = inp["indices"].pin_memory()
    lanes = []
    for li in range(max(1, args.e2e_lanes)):
        dl = dec if li == 0 else decoder_for(inp, num_sms=args.num_sms, device=dev)
        lanes.append({
            "dec": dl,
            "stream": torch.cuda.Stream(dev),
            "dev_in": {k: torch.empty_like(v, device=dev) for k, v in host_in.items()},
            "host_out": torch.empty(dl.out.shape, dtype=dl.out.dtype).pin_memory(),
            "host_lse": torch.empty(dl.lse.shape, dtype=dl.lse.dtype).pin_memory(),
        })

    def e2e_step(i):
        ln = lanes[i % len(lanes)]
        st, dl, din = ln["stream"], ln["dec"], ln["dev_in"]
        with torch.cuda.stream(st):
            for k, v in host_in.items():
                din[k].copy_(v, non_blocking=True)
            dl.plan_step(din["seq_lens"], st)
            dl.decode_step(din["q"], g["cache"], din["block_table"], din["seq_lens"], din.get("indices"), st)
            dl.combine_step(st)
            ln["host_out"].copy_(dl.out, non_blocking=True)
            ln["host_lse"].copy_(dl.lse, non_blocking=True)

    def lanes_wait(ev):
        for ln in lanes:
            ln["stream"].wait_event(ev)

    def join_lanes():
        for ln in lanes:
            stream.wait_stream(ln["stream"])

    torch.cuda.synchronize(dev)
    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    K2 = max(3, min(K, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    lanes_wait(e0)
    for i in range(K2):
        e2e_step(i)
    join_lanes()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / K2], world, dev)

    for ln in lanes:
        st, bits = ln["dec"].error(stream)
        if st != 0:
            raise RuntimeError(f"device error in timed region: status {st} bits {bits:#x}")

    # small inputs: the same step captured in a CUDA graph (launch overhead removed), L2 flushed before each replay
    graph_ms = None
    if flush_l2:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            step(st=side)  # warm the capture stream
            with torch.cuda.graph(graph, stream=side):
                step(st=side)
        stream.wait_stream(side)
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(K):
            flush_buf.fill_(i & 0xFF)
            gev[i][0].record(stream)
            graph.replay()
            gev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        (graph_ms,) = max_over_ranks([sum(a.elapsed_time(b) for a, b in gev) / K], world, dev)
        del graph

    peaks, peak_src = load_peaks()
    t_hbm = acc["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = acc["flops"] / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    dec_s = decode_ms / 1e3
    achieved_gbs = acc["bytes"] / dec_s / 1e9
    achieved_tf = acc["flops"] / dec_s / 1e12
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved_tf / peaks["bf16_tflops"]}
    roof["traffic"] = profiled_traffic("mla_decode_kernel", args.workload + ("" if args.cache == "bf16" else "-fp8"))
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst figures)" if peak_src == "measured" else peak_src
    roof["kernel"] = "mla_decode_kernel"
    roof["roofline_time_us"] = max(t_hbm, t_tc) * 1e6
    roof["kernel_time_us"] = decode_ms * 1e3
    roof["time_frac"] = max(t_hbm, t_tc) / dec_s
    roof["time_frac_step"] = max(t_hbm, t_tc) / (ms_per_step / 1e3)
    roof["tb_per_s"] = achieved_gbs / 1e3
    roof["tflop_per_s"] = achieved_tf
    roof["tensor_frac"] = achieved_tf / peaks["bf16_tflops"]

    value = job_value(world, acc["kv_tokens"], ms_per_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if args.cache == "bf16" else "bf16 (fp8 e4m3 cache expanded to bf16)", "data": "synthetic",
        "config": decode_config(inp, acc, world, l2_bytes, args.cache),
        "launch": {"decode_workers": dec.num_workers, "ctas_per_worker": 2},
        "roofline": roof,
        "e2e": {"value": job_value(world, acc["kv_tokens"], e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": acc["h2d_bytes"], "d2h_bytes_per_step": acc["d2h_bytes"],
                "ms_per_step": e2e_ms, "streams": len(lanes),
                "note": "plan + decode + combine through the C ABI, inputs from pinned host memory and out/lse "
                        f"back every step; consecutive steps rotate over {len(lanes)} decoders on as many streams"},
        "gpu_launches": 3 * K,
        "kernels_us": {"plan": plan_ms * 1e3, "decode": decode_ms * 1e3, "combine": combine_ms * 1e3,
                       "sampled_steps": len(kev), "statistic": "median of the sampled timed steps",
                       "median_of_100_after": {"plan": med100[0] * 1e3, "decode": med100[1] * 1e3,
                                               "combine": med100[2] * 1e3}},
        "graph_ms_per_step": graph_ms,
        "clocks": sampler.summary() if sampler else None,
    }
    if rank == 0 and world == 1:
        torch.set_num_threads(os.cpu_count() or 1)
        if inp["cache"].dtype == torch.uint8:
            import oracle

            inp = dict(inp, cache=oracle.dequantize_cache(inp["cache"]))
        toks, secs, nseq = oracle_sample(inp, args.cpu_budget)
        line["cpu_baseline"] = {"value": toks / secs, "unit": UNIT, "cores": torch.get_num_threads(),
                                "kind": "oracle",
                                "sample": f"{nseq} of {inp['batch']} sequences ({toks} KV tokens) of the same batch, "
                                          f"float64, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

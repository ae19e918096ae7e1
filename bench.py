#!/usr/bin/env python
"""Benchmark of the sparse FP8-KV MLA decode hot path on B200.

One step = the whole hot path over one batch of synthetic input:
scheduler metadata -> split-KV decode kernel -> PDL-chained combine, through
the library's public API (the C ABI via the Python binding).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the float64 CPU oracle, timed on host cores

Rank 0 prints one JSON line.  With N > 1 (launched by torch.distributed.run)
every rank runs its own independent replica of the workload (different
seeds, no data-path collective): requests are independent, so the path shards
with no exchange and the scaling is weak.  `value` is the FLOP of all ranks'
steps divided by the slowest rank's time.

Timing: W warm-up steps, then exactly K steps bracketed by a barrier and a
device synchronisation, timed with CUDA events on the launching stream.  The
inputs rotate over several independent copies (each with its own cache,
queries and indices) whose combined size exceeds the 126 MB L2, so a step's
gathered rows were not left in L2 by the previous steps.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import signal
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse FP8-KV MLA decode TFLOP/s (% of BF16 TC peak) and gathered-KV GB/s"
DQK, DV, ROW = 576, 512, 656


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_h128_b64_topk2048")
    ap.add_argument("--copies", type=int, default=4, help="independent input copies rotated over the steps")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the per-workload records of the other shapes and of the sparse-prefill entry")
    return ap.parse_args()


def host_cpu():
    """(logical cores, model name) of the host the CPU baseline runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 0, model


def valid_counts(idx: np.ndarray, seqlens: np.ndarray) -> np.ndarray:
    sl = np.asarray(seqlens, dtype=np.int64).reshape(-1, 1, 1)
    return ((idx >= 0) & (idx < sl)).sum(axis=-1)


def step_flops(h_q: int, valid: np.ndarray) -> float:
    """Algorithmic FLOP of one step: 2 * h_q * valid_topk * (576 + 512) summed over query tokens."""
    return float(2.0 * h_q * (DQK + DV) * valid.astype(np.float64).sum())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clock and throttle-reason samples (every 20 ms) around a timed region.

    `mark_start()` / `mark_end()` bracket the timed region; the summary keeps the
    samples whose timestamps fall inside it, widened by `pad_ms` on each side (a
    region of a few milliseconds is shorter than nvidia-smi's sampling period, and
    the warm-up right before it runs the same work)."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, pad_ms: float = 50.0):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.pad_ms = pad_ms
        self.t_start = None
        self.t_end = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "20", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def mark_start(self):
        self.t_start = datetime.datetime.now()

    def mark_end(self):
        self.t_end = datetime.datetime.now()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)   # let the sample after the region land
            self.proc.send_signal(signal.SIGTERM)
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    @staticmethod
    def parse(lines):
        rows = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        return rows

    def summarize(self, rows):
        window = f"timed region +- {self.pad_ms:.0f} ms"
        if self.t_start is not None and self.t_end is not None and rows and all(r[0] is not None for r in rows):
            pad = datetime.timedelta(milliseconds=self.pad_ms)
            rows = [r for r in rows if self.t_start - pad <= r[0] <= self.t_end + pad]
        else:
            window = "whole sampler run (timestamps unavailable)"
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        sm = [r[1] for r in rows]
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[2] for r in rows), "reasons": reasons,
                "samples": len(rows), "window": window}

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        with open(self.path) as f:
            rows = self.parse(f.readlines())
        os.remove(self.path)
        return self.summarize(rows)


# ---------------------------------------------------------------------------
# the reference arm: the float64 CPU oracle
# ---------------------------------------------------------------------------

def host_inputs(w):
    """Host copies of a workload for the oracle (cache rows from the oracle's own quantiser)."""
    import oracle
    from sparse_mla_decoding_b200 import workloads as W
    lay = W.layout(w)
    rows = lay.num_blocks * W.BLOCK
    cache = np.empty((rows, ROW), dtype=np.uint8)
    for start, lat, rope in W.cache_values(w, rows, chunk_rows=W.GEN_CHUNK_ROWS * 4):
        cache[start:start + lat.shape[0]] = oracle.quantize_tokens_bulk(lat, rope)
    W.poison(cache, W.unused_rows(lay))
    idx = W.indices(w, lay.seqlens)
    return dict(q=W.queries(w), cache=cache.reshape(lay.num_blocks, W.BLOCK, ROW), bt=lay.block_table,
                seqlens=lay.seqlens.astype(np.int32), idx=idx)


def cpu_oracle_sample(w, hi, budget_s: float, max_tokens=None):
    """Time the oracle (single-threaded, as it stands) on tokens until the budget is spent."""
    import oracle
    tokens = [(b, t) for b in range(w.batch) for t in range(w.s_q)]
    rng = np.random.default_rng(2024)
    order = rng.permutation(len(tokens))
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    for k in order:
        b, t = tokens[k]
        oracle.sparse_decode_token(hi["q"][b, t], hi["cache"], hi["bt"][b], int(hi["seqlens"][b]), hi["idx"][b, t])
        v = int(((hi["idx"][b, t] >= 0) & (hi["idx"][b, t] < hi["seqlens"][b])).sum())
        flops += 2.0 * w.h_q * (DQK + DV) * v
        done += 1
        if time.perf_counter() - t0 >= budget_s or (max_tokens and done >= max_tokens):
            break
    dt = time.perf_counter() - t0
    return flops, dt, done


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    hi = host_inputs(w)
    n_tok = w.batch * w.s_q
    per_step_budget = max(0.2, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, hi, per_step_budget / 4, max_tokens=1)
    tot_f, tot_t, tot_n = 0.0, 0.0, 0
    for _ in range(args.steps):
        f, t, n = cpu_oracle_sample(w, hi, per_step_budget)
        tot_f, tot_t, tot_n = tot_f + f, tot_t + t, tot_n + n
    tflops = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q, "topk": w.topk},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": 1, "host_cores": host_cpu()[0],
                         "cpu_model": host_cpu()[1], "kind": "oracle",
                         "sample": f"{tot_n} of {n_tok} query tokens per pass over {args.steps} steps "
                                   f"(single-threaded float64 C oracle)"},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def time_decode_calls(smla, torch, copies, metas, ws, outs, stream, steps):
    """Mean CUDA-event duration (ms) of `steps` decode calls over the rotating input copies.

    Each call is bracketed by its own pair of events on `stream`; the device is
    synchronised before and after the loop."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        d, (sm, ns) = copies[i % len(copies)], metas[i % len(metas)]
        evs[i][0].record(stream)
        smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns,
                                    workspace=ws, out=outs)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def make_device_copy(w, device, values="host"):
    """Generator values -> device tensors; the cache rows are written by the library's own KV writer.

    values="host" draws the cache values with the shared generator (the streams
    the tests use); values="device" draws the same distributions (N(0,1), the
    workload's outlier channels x8) with a seeded torch generator on the GPU,
    which is much faster for the multi-GB caches.  Queries, lengths, block
    tables and indices always come from the shared generator."""
    import torch
    import sparse_mla_decoding_b200 as smla
    from sparse_mla_decoding_b200 import workloads as W
    lay = W.layout(w)
    rows = lay.num_blocks * W.BLOCK
    cache = torch.empty((lay.num_blocks, W.BLOCK, ROW), dtype=torch.uint8, device=device)
    flat = cache.view(rows, ROW)
    if values == "host":
        for start, lat, rope in W.cache_values(w, rows, chunk_rows=W.GEN_CHUNK_ROWS * 4):
            n = lat.shape[0]
            dl = torch.from_numpy(lat.view(np.int16)).to(device).view(torch.bfloat16)
            dr = torch.from_numpy(rope.view(np.int16)).to(device).view(torch.bfloat16)
            smla.quantize_kv(dl, dr, flat[start:start + n])
    else:
        gen = torch.Generator(device=device)
        gen.manual_seed(int(w.seed) * 7919 + 11)
        ch = torch.from_numpy(W.outlier_channels(w)).to(device)
        step = 1 << 20
        for start in range(0, rows, step):
            n = min(step, rows - start)
            lat = torch.randn((n, DV), generator=gen, device=device)
            if ch.numel():
                lat[:, ch] *= w.outlier_factor
            rope = torch.randn((n, 64), generator=gen, device=device)
            smla.quantize_kv(lat.to(torch.bfloat16), rope.to(torch.bfloat16), flat[start:start + n])
    unused = torch.from_numpy(W.unused_rows(lay)).to(device)
    flat[unused] = torch.from_numpy(W.POISON_ROW).to(device)
    idx = W.indices(w, lay.seqlens)
    q = torch.from_numpy(W.queries(w).view(np.int16)).to(device).view(torch.bfloat16)
    return dict(q=q, kvcache=cache, block_table=torch.from_numpy(lay.block_table).to(device),
                cache_seqlens=torch.from_numpy(lay.seqlens.astype(np.int32)).to(device),
                indices=torch.from_numpy(idx).to(device), idx_host=idx, seqlens_host=lay.seqlens)


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one split-kernel
# launch from an ncu capture, per workload, with the hash of the split kernel's
# sources and build flags the capture was taken on (split_kernel_hash()).
# Reported only while they still match; the capture commands are in profiles/.
NCU_TRAFFIC = {
    "decode_h128_b64_topk2048": {
        "bytes": 107_896_320 + 3_602_944,
        "srchash": "f291856577637ecbceaccd3305e82dd35474fa43d80a3ac7043f775ae7eb292e"},
    "decode_h64_b128_sq2_topk2048": {
        "bytes": 397_131_264 + 13_732_096,
        "srchash": "f291856577637ecbceaccd3305e82dd35474fa43d80a3ac7043f775ae7eb292e"},
}

def split_kernel_hash():
    """Hash of the files the split kernel is compiled from (and of the build flags)."""
    import hashlib
    pkg = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sparse_mla_decoding_b200")
    h = hashlib.sha256()
    for rel in ("csrc/splitkv_mla.cu", "csrc/sm100.cuh", "csrc/splitkv_mla.h", "build.py"):
        h.update(rel.encode())
        with open(os.path.join(pkg, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload):
    rec = NCU_TRAFFIC.get(workload)
    if rec is None or rec["srchash"] != split_kernel_hash():
        return None
    return rec["bytes"]


def rank_seed(w, rank, copy):
    """Seed of input copy `copy` on rank `rank`: every rank and copy draws its own inputs."""
    return w.seed + 1000 * rank + 17 * copy


def reduce_over_ranks(times, work, device, world):
    """Whole-job numbers: the max of each time and the sum of each work count over ranks.

    Every rank calls it with the same list lengths, in the same order (NCCL on GPUs;
    the CPU tests run it over gloo)."""
    import torch
    t = torch.tensor([float(x) for x in times], dtype=torch.float64, device=device)
    s = torch.tensor([float(x) for x in work], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(s, op=dist.ReduceOp.SUM)
    return t.tolist(), s.tolist()


def roofline(peaks, h_q, per_launch_flops, per_launch_bytes, launch_ms):
    """Roofline of one launch: tensor-bound above the measured ridge, HBM-bound below it."""
    intensity = (2.0 * h_q * (DQK + DV)) / ROW
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity >= ridge:
        achieved = per_launch_flops / (launch_ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"]}
    achieved = per_launch_bytes / (launch_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"]}


def timed(fn, n, stream, flush=None):
    """Mean device time (ms) of fn() over n calls, with CUDA events on `stream`.

    Without `flush` the calls run back to back between two events; with it,
    every call is bracketed by its own events and flush() runs between calls,
    outside the timed intervals."""
    import torch
    if flush is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(n):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        flush()
        evs[i][0].record(stream)
        fn(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([x.elapsed_time(y) for x, y in evs]))


# How each extra record keeps a step's gathered rows from being served out of
# L2 by an earlier timed step, and how its cache values are drawn.
EXTRA_DECODE = (
    ("tiny_h16_b2_topk64", 1, "host", "flush",
     "one copy; L2 flushed (256 MB write) between individually timed calls"),
    ("decode_h64_b128_sq2_topk2048", 1, "device", None,
     "one copy: each step gathers 327 MB of rows from a 2.75 GB cache, both larger than the 126 MB L2"),
    ("longctx_varlen_h128_b32_topk2048", 4, "device", None,
     "inputs rotated over 4 independent copies (4 x 43 MB of rows per step, 4 x 1.5 GB caches) > 126 MB L2"),
    ("prefill_shaped_h128_sq4096_topk2048", 1, "device", None,
     "one copy: 604 MB of queries per step > 126 MB L2; the 43 MB cache itself is L2-resident by design "
     "(each step reads it 128 times over), so its GB/s are L2 reads"),
)


def decode_record(w, n_copies, values, mode, l2_note, args, device, rank, world, peaks):
    """The headline measurements (whole step, decode call, end to end) for one more workload."""
    import torch
    import sparse_mla_decoding_b200 as smla
    stream = torch.cuda.current_stream(device)
    copies = [make_device_copy(w.with_(seed=rank_seed(w, rank, c)), device, values) for c in range(n_copies)]
    torch.cuda.synchronize()
    flops = [step_flops(w.h_q, valid_counts(c["idx_host"], c["seqlens_host"])) for c in copies]
    valid = [float(valid_counts(c["idx_host"], c["seqlens_host"]).sum()) for c in copies]
    num_parts = smla.default_num_sm_parts(w.h_q, device)
    ws = smla.new_workspace(w.batch, w.s_q, w.h_q, w.topk, num_parts, device)
    outs = (torch.empty((w.batch, w.s_q, w.h_q, DV), dtype=torch.bfloat16, device=device),
            torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=device))
    metas = [smla.get_mla_metadata(c["cache_seqlens"], w.topk, w.h_q, num_parts, s_q=w.s_q) for c in copies]
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device) if mode == "flush" else None
    flush = (lambda: flush_buf.fill_(1)) if flush_buf is not None else None

    def step(i):
        d = copies[i % n_copies]
        sm, ns = smla.get_mla_metadata(d["cache_seqlens"], w.topk, w.h_q, num_parts, s_q=w.s_q)
        smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"],
                                    sm, ns, workspace=ws, out=outs)

    def call(i):
        d, (sm, ns) = copies[i % n_copies], metas[i % n_copies]
        smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"],
                                    sm, ns, workspace=ws, out=outs)

    host = [dict(q=c["q"].cpu().pin_memory(), indices=c["indices"].cpu().pin_memory(),
                 block_table=c["block_table"].cpu().pin_memory(), cache_seqlens=c["cache_seqlens"].cpu().pin_memory())
            for c in copies]
    dq, di = torch.empty_like(copies[0]["q"]), torch.empty_like(copies[0]["indices"])
    dsl = torch.empty_like(copies[0]["cache_seqlens"])
    dbt = [torch.empty_like(c["block_table"]) for c in copies]   # widths differ when lengths are drawn
    ho = torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory()
    hl = torch.empty(outs[1].shape, dtype=outs[1].dtype).pin_memory()
    h2d = int(np.mean([sum(h[k].numel() * h[k].element_size() for k in h) for h in host]))
    d2h = ho.numel() * 2 + hl.numel() * 4

    def e2e_step(i):
        h, c = host[i % n_copies], copies[i % n_copies]
        dq.copy_(h["q"], non_blocking=True)
        di.copy_(h["indices"], non_blocking=True)
        dbt[i % n_copies].copy_(h["block_table"], non_blocking=True)
        dsl.copy_(h["cache_seqlens"], non_blocking=True)
        sm, ns = smla.get_mla_metadata(dsl, w.topk, w.h_q, num_parts, s_q=w.s_q)
        o, l = smla.flash_mla_with_kvcache(dq, c["kvcache"], dbt[i % n_copies], dsl, di, sm, ns, workspace=ws,
                                           out=outs)
        ho.copy_(o, non_blocking=True)
        hl.copy_(l, non_blocking=True)

    steps = max(args.steps // 2, 8)
    for i in range(args.warmup):
        step(i)
        e2e_step(i)
    step_ms = timed(step, steps, stream, flush)
    call_ms = timed(call, steps, stream, flush)
    e2e_ms = timed(e2e_step, steps, stream, flush)
    status, raw = smla.get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word set during the {w.name} record: {raw:#x}")
    mean_f, mean_v = float(np.mean(flops)), float(np.mean(valid))
    (step_ms, call_ms, e2e_ms), (f_all, v_all) = reduce_over_ranks([step_ms, call_ms, e2e_ms], [mean_f, mean_v],
                                                                   device, world)
    rec = {"value": f_all / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms, "steps": steps,
           "gathered_kv_gbs": v_all * ROW / (step_ms * 1e-3) / 1e9,
           "roofline": dict(roofline(peaks, w.h_q, mean_f, mean_v * ROW, call_ms),
                            kernel="splitkv_mla_kernel + combine_kernel (one decode call)", kernel_ms=call_ms,
                            traffic=measured_traffic(w.name), peak_source=peaks["source"] + " (burst)"),
           "e2e": {"value": f_all / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                   "d2h_bytes_per_step": int(d2h)},
           "config": {"workload": w.name, "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q, "topk": w.topk,
                      "cache_values": "shared generator" if values == "host" else "seeded torch generator on the GPU",
                      "l2": l2_note}}
    del copies, host, ws, flush_buf
    torch.cuda.empty_cache()
    return rec


# Dense decode shapes (every cached token attended; the pages give no shapes
# for it): 64 requests of 8192 tokens, 128 heads, one new token, FP8 or BF16
# cache rows.  Each step gathers 344 MB (FP8) or 604 MB (BF16) of rows, both
# larger than the 126 MB L2, from one copy.
DENSE_RECORDS = (("dense_fp8_h128_b64_s8192", 0), ("dense_bf16_h128_b64_s8192", 1))


def dense_record(name, kv_format, args, device, rank, world, peaks):
    """Dense decode (metadata + split kernel + combine) on one paged cache."""
    import torch
    import sparse_mla_decoding_b200 as smla
    from sparse_mla_decoding_b200 import workloads as W
    w = W.Workload(name, batch=64, s_q=1, h_q=128, topk=1, seed=rank_seed(W.DECODE_H128, rank, 5 + kv_format),
                   seqlens=(8192,) * 64)
    stream = torch.cuda.current_stream(device)
    lay = W.layout(w)
    rows = lay.num_blocks * W.BLOCK
    gen = torch.Generator(device=device)
    gen.manual_seed(int(w.seed) * 131 + 7)
    if kv_format == 0:
        kv = torch.empty((lay.num_blocks, W.BLOCK, ROW), dtype=torch.uint8, device=device)
        flat = kv.view(rows, ROW)
        for start in range(0, rows, 1 << 20):
            n = min(1 << 20, rows - start)
            smla.quantize_kv(torch.randn((n, DV), generator=gen, device=device).to(torch.bfloat16),
                             torch.randn((n, 64), generator=gen, device=device).to(torch.bfloat16), flat[start:start + n])
        row_bytes = ROW
    else:
        kv = torch.randn((lay.num_blocks, W.BLOCK, DQK), generator=gen, device=device).to(torch.bfloat16)
        row_bytes = 2 * DQK
    q = torch.from_numpy(W.queries(w).view(np.int16)).to(device).view(torch.bfloat16)
    bt = torch.from_numpy(lay.block_table).to(device)
    sl = torch.from_numpy(lay.seqlens.astype(np.int32)).to(device)
    tokens = float(lay.seqlens.sum()) * w.s_q
    flops = 2.0 * w.h_q * (DQK + DV) * tokens
    parts = smla.default_num_sm_parts(w.h_q, device)
    ws = smla.new_workspace(w.batch, w.s_q, w.h_q, 1, parts, device)
    outs = (torch.empty((w.batch, w.s_q, w.h_q, DV), dtype=torch.bfloat16, device=device),
            torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=device))
    meta = smla.get_mla_metadata_dense(sl, w.h_q, s_q=w.s_q, causal=True, num_sm_parts=parts)

    def step(i):
        sm, ns, tp = smla.get_mla_metadata_dense(sl, w.h_q, s_q=w.s_q, causal=True, num_sm_parts=parts)
        smla.flash_mla_dense_with_kvcache(q, kv, bt, sl, sm, ns, tp, causal=True, workspace=ws, out=outs)

    def call(i):
        smla.flash_mla_dense_with_kvcache(q, kv, bt, sl, *meta, causal=True, workspace=ws, out=outs)

    for i in range(args.warmup):
        step(i)
    steps = max(args.steps // 2, 8)
    step_ms = timed(step, steps, stream)
    call_ms = timed(call, steps, stream)
    status, raw = smla.get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word set during the {name} record: {raw:#x}")
    (step_ms, call_ms), (f_all, b_all) = reduce_over_ranks([step_ms, call_ms], [flops, tokens * row_bytes], device,
                                                           world)
    rec = {"value": f_all / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": step_ms, "steps": steps,
           "gathered_kv_gbs": b_all / (step_ms * 1e-3) / 1e9,
           "roofline": dict(roofline(peaks, w.h_q, flops, tokens * row_bytes, call_ms) if kv_format == 0 else
                            _dense_bf16_roofline(peaks, flops, tokens * row_bytes, call_ms),
                            kernel="splitkv_mla_kernel + combine_kernel (one dense decode call)", kernel_ms=call_ms,
                            peak_source=peaks["source"] + " (burst)"),
           "config": {"api": "flash_mla_dense_with_kvcache", "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q,
                      "seqlen": 8192, "causal": True, "kv_row_bytes": row_bytes,
                      "cache_values": "seeded torch generator on the GPU",
                      "l2": f"one copy: {tokens * row_bytes / 1e6:.0f} MB of rows per step > 126 MB L2"}}
    del kv, ws, q
    torch.cuda.empty_cache()
    return rec


def _dense_bf16_roofline(peaks, flops, nbytes, ms):
    """BF16 rows carry 1152 bytes for 2 * 128 * 1088 flop: compare both roofs, report the binding one."""
    intensity = flops / nbytes
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity >= ridge:
        a = flops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / peaks["bf16_tflops"]}
    a = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": a / peaks["hbm_gbs"]}


def sparse_fwd_record(args, device, rank, world, peaks):
    """flash_mla_sparse_fwd on the prefill-shaped workload: 4096 query tokens over one flat FP8 cache."""
    import torch
    import sparse_mla_decoding_b200 as smla
    from sparse_mla_decoding_b200 import workloads as W
    w = W.BY_NAME["prefill_shaped_h128_sq4096_topk2048"].with_(seed=rank_seed(W.PREFILL_SHAPED, rank, 0))
    stream = torch.cuda.current_stream(device)
    d = make_device_copy(w, device, "device")
    s_kv = int(d["seqlens_host"][0])
    # the flat cache holds logical token i at row i
    pos = torch.arange(s_kv, device=device)
    rows = d["block_table"][0].long()[pos // W.BLOCK] * W.BLOCK + pos % W.BLOCK
    kv = d["kvcache"].view(-1, ROW).index_select(0, rows).contiguous()
    q = d["q"].view(w.s_q, w.h_q, DQK)
    idx = d["indices"].view(w.s_q, 1, w.topk)
    f = step_flops(w.h_q, valid_counts(d["idx_host"], d["seqlens_host"]))
    v = float(valid_counts(d["idx_host"], d["seqlens_host"]).sum())
    parts = smla.default_num_sm_parts(w.h_q, device)
    ws = smla.new_sparse_fwd_workspace(w.s_q, w.h_q, s_kv, w.topk, parts, device)
    outs = (torch.empty((w.s_q, w.h_q, DV), dtype=torch.bfloat16, device=device),
            torch.empty((w.s_q, w.h_q), dtype=torch.float32, device=device))

    def call(i):
        smla.flash_mla_sparse_fwd(q, kv, idx, num_sm_parts=parts, workspace=ws, out=outs)

    for i in range(args.warmup):
        call(i)
    steps = max(args.steps // 5, 4)
    ms = timed(call, steps, stream)
    status, raw = smla.get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word set during the sparse_fwd record: {raw:#x}")
    (ms,), (f_all, v_all) = reduce_over_ranks([ms], [f, v], device, world)
    rec = {"value": f_all / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "steps": steps,
           "gathered_kv_gbs_l2": v_all * ROW / (ms * 1e-3) / 1e9,
           "roofline": dict(roofline(peaks, w.h_q, f, v * ROW, ms),
                            kernel="flash_mla_sparse_fwd (set-up + metadata + split kernel + combine)",
                            peak_source=peaks["source"] + " (burst)"),
           "config": {"api": "flash_mla_sparse_fwd", "s_q": w.s_q, "h_q": w.h_q, "s_kv": s_kv, "topk": w.topk,
                      "indices": "causal, < 61440 + query position",
                      "l2": "604 MB of queries per call > 126 MB L2; the 43 MB cache is L2-resident by design"}}
    del d, kv, ws
    torch.cuda.empty_cache()
    return rec


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_mla_decoding_b200 as smla
    from sparse_mla_decoding_b200 import workloads as W

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    smla.lib()
    stream = torch.cuda.current_stream(device)

    # independent copies (weak scaling: every rank has its own seeds)
    copies = [make_device_copy(w.with_(seed=rank_seed(w, rank, c)), device) for c in range(args.copies)]
    torch.cuda.synchronize()
    flops_per_copy = [step_flops(w.h_q, valid_counts(c["idx_host"], c["seqlens_host"])) for c in copies]
    valid_per_copy = [float(valid_counts(c["idx_host"], c["seqlens_host"]).sum()) for c in copies]
    topk = w.topk
    num_parts = smla.default_num_sm_parts(w.h_q, device)
    ws = smla.new_workspace(w.batch, w.s_q, w.h_q, topk, num_parts, device)
    outs = (torch.empty((w.batch, w.s_q, w.h_q, DV), dtype=torch.bfloat16, device=device),
            torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=device))

    def step(c):
        d = copies[c]
        sm, ns = smla.get_mla_metadata(d["cache_seqlens"], topk, w.h_q, num_parts, s_q=w.s_q)
        return smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                           d["indices"], sm, ns, workspace=ws, out=outs)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i % args.copies)
    torch.cuda.synchronize()

    # ---- the timed region --------------------------------------------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        ev0.record(stream)
        for i in range(args.steps):
            step(i % args.copies)
        ev1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier()
    ms_total = ev0.elapsed_time(ev1)
    clocks = clk.summary()
    my_flops = sum(flops_per_copy[i % args.copies] for i in range(args.steps))
    my_valid = sum(valid_per_copy[i % args.copies] for i in range(args.steps))

    # ---- the decode call alone (split kernel + chained combine), for the roofline
    metas = [smla.get_mla_metadata(copies[c]["cache_seqlens"], topk, w.h_q, num_parts, s_q=w.s_q)
             for c in range(args.copies)]
    kern_ms = time_decode_calls(smla, torch, copies, metas, ws, outs, stream, args.steps)

    # ---- the same decode calls in the two-CTA cluster form (128 heads), for comparison
    cluster_form = None
    if w.h_q > 64:
        prev_form = smla.set_head_pair_form(True)
        try:
            time_decode_calls(smla, torch, copies, metas, ws, outs, stream, 3)   # warm-up of this form
            pair_ms = time_decode_calls(smla, torch, copies, metas, ws, outs, stream, args.steps)
            cluster_form = {"kernel_ms": pair_ms,
                            "decode_call_tflops": float(np.mean(flops_per_copy)) / (pair_ms * 1e-3) / 1e12,
                            "note": "smla_set_head_pair_form(1): each 128-head part as a two-CTA cluster sharing "
                                    "dequantised tiles; the default runs the two 64-head CTAs independently"}
        except Exception as e:   # a comparison only: never lose the bench line over it
            cluster_form = {"error": f"{type(e).__name__}: {e}"}
        finally:
            smla.set_head_pair_form(prev_form)

    # ---- end to end: pinned host inputs in, results out, every step --------
    e2e = None
    host = []
    for c in copies:
        host.append(dict(q=c["q"].cpu().pin_memory(), indices=c["indices"].cpu().pin_memory(),
                         block_table=c["block_table"].cpu().pin_memory(),
                         cache_seqlens=c["cache_seqlens"].cpu().pin_memory()))
    dq = torch.empty_like(copies[0]["q"])
    di = torch.empty_like(copies[0]["indices"])
    dbt = [torch.empty_like(c["block_table"]) for c in copies]
    dsl = torch.empty_like(copies[0]["cache_seqlens"])
    ho = torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory()
    hl = torch.empty(outs[1].shape, dtype=outs[1].dtype).pin_memory()
    h2d = (host[0]["q"].numel() * 2 + host[0]["indices"].numel() * 4 + host[0]["block_table"].numel() * 4 +
           host[0]["cache_seqlens"].numel() * 4)
    d2h = ho.numel() * 2 + hl.numel() * 4

    def e2e_step(c):
        h = host[c]
        dq.copy_(h["q"], non_blocking=True)
        di.copy_(h["indices"], non_blocking=True)
        dbt[c].copy_(h["block_table"], non_blocking=True)
        dsl.copy_(h["cache_seqlens"], non_blocking=True)
        sm, ns = smla.get_mla_metadata(dsl, topk, w.h_q, num_parts, s_q=w.s_q)
        o, l = smla.flash_mla_with_kvcache(dq, copies[c]["kvcache"], dbt[c], dsl, di, sm, ns, workspace=ws, out=outs)
        ho.copy_(o, non_blocking=True)
        hl.copy_(l, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i % args.copies)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i % args.copies)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)

    status, raw = smla.get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word set during the benchmark: {raw:#x}")

    # ---- reduce over ranks (max time, summed work) --------------------------
    (ms_total, e2e_ms, kern_ms), (tot_flops, tot_valid) = reduce_over_ranks(
        [ms_total, e2e_ms, kern_ms], [my_flops, my_valid], device, world)
    peaks = load_peaks()
    if rank != 0:
        # the other ranks take the same collective steps for the extra records
        if not args.no_extra_workloads:
            from sparse_mla_decoding_b200 import workloads as W
            for name, n_copies, values, mode, note in EXTRA_DECODE:
                if name != w.name:
                    decode_record(W.BY_NAME[name], n_copies, values, mode, note, args, device, rank, world, peaks)
            sparse_fwd_record(args, device, rank, world, peaks)
            for name, fmt in DENSE_RECORDS:
                dense_record(name, fmt, args, device, rank, world, peaks)
        return

    tflops = tot_flops / (ms_total * 1e-3) / 1e12
    gbs = tot_valid * ROW / (ms_total * 1e-3) / 1e9
    # roofline of the decode call on this rank: per-launch algorithmic work / average launch duration
    per_launch_flops = float(np.mean(flops_per_copy))
    per_launch_bytes = float(np.mean(valid_per_copy)) * ROW
    roof = roofline(peaks, w.h_q, per_launch_flops, per_launch_bytes, kern_ms)
    roof.update({"traffic": measured_traffic(w.name), "kernel": "splitkv_mla_kernel + combine_kernel (one decode call)",
                 "kernel_ms": kern_ms, "peak_source": peaks["source"] + " (burst)"})

    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "s_q": w.s_q, "h_q": w.h_q, "topk": w.topk,
                   "seqlen": int(copies[0]["seqlens_host"].max()), "kv_row_bytes": ROW, "num_sm_parts": num_parts,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs rotated over {args.copies} independent copies "
                         f"({args.copies} x {copies[0]['kvcache'].numel() / 1e6:.0f} MB cache) > 126 MB L2"},
        "gathered_kv_gbs": gbs,
        "pct_of_bf16_peak": 100.0 * tflops / world / peaks["bf16_tflops"],
        "roofline": roof,
        "e2e": {"value": tot_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if cluster_form is not None:
        line["cluster_form"] = cluster_form
    if world == 1 and not args.no_cpu_baseline:
        hi = host_inputs(w.with_(seed=w.seed))
        f, t, n = cpu_oracle_sample(w, hi, args.cpu_seconds)
        cores, model = host_cpu()
        line["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": 1, "host_cores": cores,
                                "cpu_model": model, "kind": "oracle",
                                "sample": f"{n} of {w.batch * w.s_q} query tokens of the same workload, "
                                          f"{t:.1f} s single-threaded float64 C oracle"}
    if not args.no_extra_workloads:
        from sparse_mla_decoding_b200 import workloads as W
        extra = {}
        for name, n_copies, values, mode, note in EXTRA_DECODE:
            if name == w.name:
                continue
            extra[name] = decode_record(W.BY_NAME[name], n_copies, values, mode, note, args, device, rank, world, peaks)
        extra["sparse_fwd_prefill_shaped_h128_sq4096_topk2048"] = sparse_fwd_record(args, device, rank, world, peaks)
        for name, fmt in DENSE_RECORDS:
            extra[name] = dense_record(name, fmt, args, device, rank, world, peaks)
        line["workloads"] = extra
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from sparse_mla_decoding_b200 import workloads as W
    w = W.BY_NAME[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

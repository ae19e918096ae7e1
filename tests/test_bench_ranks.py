"""Host-side logic of bench.py on CPU, no GPU: the multi-rank path over two gloo ranks,
the reference arm's rank gating and the clock sampler's window.

bench.py runs one process per GPU; on more than one rank the whole-job time is
the max over ranks and the work is summed, rank 0 alone prints, and every rank
draws its own inputs.  These tests run that logic over gloo with world size 2.
"""
import contextlib
import io
import json
import os
import socket
import sys
import tempfile
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: times (r + 1, 10 - r, 0.5 r), work (r + 1, 100)
        times, work = bench.reduce_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank], [rank + 1, 100], "cpu", world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"times": times, "work": work}, f)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    import torch.multiprocessing as mp

    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_main, args=(world, _free_port(), d), nprocs=world, join=True)
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(world)]
    for r in res:   # every rank ends with the same whole-job numbers
        assert r["times"] == [2.0, 10.0, 0.5]
        assert r["work"] == [3.0, 200.0]


def test_single_rank_reduction_is_identity():
    import bench

    times, work = bench.reduce_over_ranks([3.5, 1.0], [7, 8], "cpu", 1)
    assert times == [3.5, 1.0] and work == [7.0, 8.0]


def test_rank_seeds_are_distinct():
    import bench
    from sparse_mla_decoding_b200 import workloads as W

    w = W.BY_NAME["decode_h128_b64_topk2048"]
    seeds = {bench.rank_seed(w, r, c) for r in range(8) for c in range(4)}
    assert len(seeds) == 32


def test_reference_arm_prints_on_rank0_only():
    import bench
    from sparse_mla_decoding_b200 import workloads as W

    w = W.BY_NAME["tiny_h16_b2_topk64"]
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=2)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, w, rank=1, world=2)
    assert buf.getvalue() == ""
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, w, rank=0, world=2)
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_clock_sampler_keeps_samples_of_the_timed_region():
    import datetime

    import bench

    c = bench.ClockSampler(0, pad_ms=50.0)
    lines = [
        "2026/12/02 19:35:11.000, 0, 1000, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 19:35:12.100, 0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 19:35:12.200, 0, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 19:35:13.900, 0, 210, 1965, 100.0, 0x0, Not Active, Active, Not Active, Not Active",
        "garbage line",
    ]
    rows = c.parse(lines)
    assert len(rows) == 4
    c.t_start = datetime.datetime(2026, 12, 2, 19, 35, 12, 90000)
    c.t_end = datetime.datetime(2026, 12, 2, 19, 35, 12, 160000)
    s = c.summarize(rows)
    assert s["samples"] == 2 and s["sm_mhz"] == 1932.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and "timed region" in s["window"]


def test_clock_sampler_without_timestamps_uses_every_sample():
    import bench

    c = bench.ClockSampler(0)
    rows = c.parse(["n/a, 0, 1800, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active"])
    c.mark_start()
    c.mark_end()
    s = c.summarize(rows)
    assert s["samples"] == 1 and s["sm_mhz"] == 1800.0 and "whole sampler run" in s["window"]


def test_time_decode_calls_brackets_each_call_and_rotates_copies():
    """The roofline's decode-call timing (also used for the cluster-form comparison):
    one event pair per call on the given stream, copies and metadata rotated, the
    device synchronised around the loop, the mean of the per-call durations."""
    import bench

    log = []

    class Event:
        t = 0.0

        def __init__(self, enable_timing):
            assert enable_timing
            self.when = None

        def record(self, stream):
            assert stream == "s0"
            Event.t += 1.0
            self.when = Event.t
            log.append("rec")

        def elapsed_time(self, other):
            return other.when - self.when

    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(
        Event=Event, synchronize=lambda: log.append("sync")))

    class FakeLib:
        def flash_mla_with_kvcache(self, q, kv, bt, sl, idx, sm, ns, workspace, out):
            assert workspace == "ws" and out == "outs"
            log.append(("call", q, sm))
            Event.t += 2.0      # each call takes 2 units between its two records

    copies = [dict(q=f"q{c}", kvcache="kv", block_table="bt", cache_seqlens="sl", indices="idx") for c in range(3)]
    metas = [(f"sm{c}", "ns") for c in range(3)]
    ms = bench.time_decode_calls(FakeLib(), fake_torch, copies, metas, "ws", "outs", "s0", 5)
    assert ms == 3.0            # record, +2 for the call, record: 3 units per call
    calls = [e for e in log if isinstance(e, tuple)]
    assert [c[1] for c in calls] == ["q0", "q1", "q2", "q0", "q1"]
    assert [c[2] for c in calls] == ["sm0", "sm1", "sm2", "sm0", "sm1"]
    assert log[0] == "sync" and log[-1] == "sync" and log.count("rec") == 10

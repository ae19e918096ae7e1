"""Request sharding over devices, on the CPU (no GPU): the cost-balanced split,
reassembly of per-shard results in one process, and the one-process-per-device
form over two gloo ranks.  The decode itself is replaced by a stand-in call
whose output depends on every input of its request, so a request routed to the
wrong shard or copied back to the wrong place changes the result."""
import datetime
import json
import os
import socket
import sys
import tempfile

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_mla_decoding_b200 import sharding as S   # noqa: E402

H, SQ, TOPK = 4, 2, 8


def fake_inputs(batch, seed=0):
    g = torch.Generator().manual_seed(seed)
    return dict(q=torch.randn((batch, SQ, H, 576), generator=g).to(torch.bfloat16),
                kvcache=torch.zeros((1, 64, 656), dtype=torch.uint8),
                block_table=torch.randint(0, 100, (batch, 3), generator=g, dtype=torch.int32),
                cache_seqlens=torch.randint(1, 1000, (batch,), generator=g, dtype=torch.int32),
                indices=torch.randint(-1, 1000, (batch, SQ, TOPK), generator=g, dtype=torch.int32))


def fake_call(x, sched, scale):
    """Per-request stand-in for the decode: o and lse mix every per-request input."""
    sig = (x["block_table"].float().sum(1) + x["cache_seqlens"].float()).view(-1, 1, 1)
    o = (x["q"][..., :512].float() * 2 + x["indices"].float().sum(-1, keepdim=True).unsqueeze(-1) + sig.unsqueeze(-1))
    lse = x["q"].float().sum(-1) + sig
    return o.to(torch.bfloat16), lse


def fake_schedule(x):
    return None, None


def take(x, a, b):
    return {k: (v[a:b] if k != "kvcache" else v) for k, v in x.items()}


def test_split_covers_in_order_and_balances():
    rng = np.random.default_rng(3)
    for batch, parts in [(0, 3), (1, 4), (5, 5), (37, 4), (1000, 8)]:
        cost = rng.integers(1, 50, batch).astype(float)
        spans = S.split_requests(batch, parts, cost)
        assert len(spans) == parts
        assert spans[0][0] == 0 and spans[-1][1] == batch
        assert all(a <= b for a, b in spans) and all(spans[i][1] == spans[i + 1][0] for i in range(parts - 1))
        if batch:
            loads = [cost[a:b].sum() for a, b in spans]
            assert max(loads) <= cost.sum() / parts + cost.max() + 1e-9
    # equal costs split evenly
    assert S.split_requests(12, 4) == [(0, 3), (3, 6), (6, 9), (9, 12)]
    with pytest.raises(ValueError):
        S.split_requests(3, 2, [1.0, -1.0, 2.0])


def test_run_sharded_reassembles_in_request_order():
    batch = 11
    x = fake_inputs(batch, seed=1)
    o_ref, lse_ref = fake_call(x, None, None)
    devices = [torch.device("cpu")] * 3
    cost = x["cache_seqlens"].float().numpy()
    shards = S.shard_requests(batch, devices, cost)
    o, lse = S.run_sharded(shards, [take(x, s.start, s.end) for s in shards], torch.device("cpu"),
                           call=fake_call, schedule=fake_schedule)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, batch):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sparse_mla_decoding_b200 import sharding as S2
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = fake_inputs(batch, seed=2)          # every rank can build the batch; it keeps its own shard
        shards = S2.shard_requests(batch, [torch.device("cpu")] * world, x["cache_seqlens"].float().numpy())
        me = shards[rank]
        o, lse = S2.decode_on_ranks(take(x, me.start, me.end), me, batch, call=fake_call, schedule=fake_schedule)
        o_ref, lse_ref = fake_call(x, None, None)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"o_equal": bool(torch.equal(o, o_ref)), "lse_equal": bool(torch.equal(lse, lse_ref)),
                       "span": [me.start, me.end]}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("batch", [9, 1], ids=["uneven", "one_empty_shard"])
def test_decode_on_ranks_gloo_world2(batch):
    import torch.multiprocessing as mp
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_rank_main, args=(world, _free_port(), d, batch), nprocs=world, join=True)
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(world)]
    assert all(r["o_equal"] and r["lse_equal"] for r in res)
    assert res[0]["span"][0] == 0 and res[-1]["span"][1] == batch

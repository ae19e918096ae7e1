"""Request sharding of the sparse MLA decode over several GPUs.

Requests (batch entries, each with its own paged cache rows, block table,
length and index lists) are independent, so a batch shards over devices with
no exchange on the data path: every device runs the single-GPU decode on the
requests whose caches it holds, and only the results (o, lse) are brought
back together.  Two forms:

* one process, several devices (``shard_requests`` + ``run_sharded``): each
  shard runs on its device's current stream; the results are copied into
  the caller's output tensors on one device;
* one process per device under torch.distributed (``decode_on_ranks``): each
  rank decodes its own requests; with ``gather=True`` an all-gather of the
  (padded) per-rank results gives every rank the whole batch.

The per-shard call is a parameter (by default the library's
``flash_mla_with_kvcache``), so the partitioning and reassembly are tested on
the CPU with a stand-in call.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Shard:
    """Requests [start, end) of the batch, decoded on `device`."""
    start: int
    end: int
    device: torch.device

    @property
    def size(self) -> int:
        return self.end - self.start


def split_requests(batch: int, parts: int, cost: Optional[Sequence[float]] = None) -> List[Tuple[int, int]]:
    """Cut requests 0..batch-1 into `parts` contiguous ranges of near-equal cost.

    `cost[r]` is request r's work (for instance its number of valid index
    slots, or its length for a dense decode); every request costs the same by
    default.  Ranges may be empty when there are fewer requests than parts.
    The cut after part p is the first request whose cost prefix reaches
    (p + 1) / parts of the total, so the result depends only on the costs.
    """
    if batch < 0 or parts < 1:
        raise ValueError("batch must be >= 0 and parts >= 1")
    c = np.ones(batch, dtype=np.float64) if cost is None else np.asarray(cost, dtype=np.float64)
    if c.shape != (batch,) or (c < 0).any():
        raise ValueError("cost must hold one non-negative value per request")
    prefix = np.concatenate([[0.0], np.cumsum(c)])
    total = prefix[-1]
    cuts = [0]
    for p in range(1, parts):
        target = total * p / parts
        # first boundary whose prefix reaches the target, never before the previous cut
        k = int(np.searchsorted(prefix, target, side="left"))
        cuts.append(min(max(k, cuts[-1]), batch))
    cuts.append(batch)
    return [(cuts[i], cuts[i + 1]) for i in range(parts)]


def shard_requests(batch: int, devices: Sequence[torch.device],
                   cost: Optional[Sequence[float]] = None) -> List[Shard]:
    return [Shard(a, b, torch.device(d)) for (a, b), d in zip(split_requests(batch, len(devices), cost), devices)]


def _default_call(inputs: Dict[str, torch.Tensor], sched: Tuple[torch.Tensor, torch.Tensor], softmax_scale):
    import sparse_mla_decoding_b200 as smla
    return smla.flash_mla_with_kvcache(inputs["q"], inputs["kvcache"], inputs["block_table"], inputs["cache_seqlens"],
                                       inputs["indices"], sched[0], sched[1], softmax_scale=softmax_scale)


def _default_schedule(inputs: Dict[str, torch.Tensor]):
    import sparse_mla_decoding_b200 as smla
    q = inputs["q"]
    return smla.get_mla_metadata(inputs["cache_seqlens"], inputs["indices"].shape[-1], q.shape[2], s_q=q.shape[1])


def run_sharded(shards: Sequence[Shard], shard_inputs: Sequence[Dict[str, torch.Tensor]], out_device: torch.device,
                softmax_scale: Optional[float] = None,
                call: Optional[Callable] = None, schedule: Optional[Callable] = None
                ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode every shard on its own device and assemble (o, lse) on `out_device`.

    `shard_inputs[i]` holds shard i's tensors on its device: q [n_i, s_q, h_q,
    576], kvcache (that device's cache), block_table [n_i, ...], cache_seqlens
    [n_i], indices [n_i, s_q, topk].  Each shard is launched on its device's
    current stream before any result is copied back, so the devices work
    concurrently; the copies then wait for their own device only.
    """
    call = call or _default_call
    schedule = schedule or _default_schedule
    if len(shards) != len(shard_inputs):
        raise ValueError("one input dict per shard")
    live = [(s, x) for s, x in zip(shards, shard_inputs) if s.size > 0]
    if not live:
        raise ValueError("no requests to decode")
    batch = max(s.end for s in shards)
    q0 = live[0][1]["q"]
    s_q, h_q = q0.shape[1], q0.shape[2]
    results = []
    for s, x in live:
        if x["q"].shape[0] != s.size:
            raise ValueError(f"shard [{s.start}, {s.end}) got {x['q'].shape[0]} requests")
        with torch.cuda.device(s.device) if s.device.type == "cuda" else _nullctx():
            results.append((s, call(x, schedule(x), softmax_scale)))
    o = torch.empty((batch, s_q, h_q, 512), dtype=torch.bfloat16, device=out_device)
    lse = torch.empty((batch, s_q, h_q), dtype=torch.float32, device=out_device)
    for s, (o_s, lse_s) in results:
        o[s.start:s.end].copy_(o_s, non_blocking=True)
        lse[s.start:s.end].copy_(lse_s, non_blocking=True)
    return o, lse


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def decode_on_ranks(local_inputs: Dict[str, torch.Tensor], shard: Shard, batch: int,
                    softmax_scale: Optional[float] = None, gather: bool = True, group=None,
                    call: Optional[Callable] = None, schedule: Optional[Callable] = None):
    """One process per device: decode this rank's shard; optionally all-gather the batch.

    Every rank calls this with its own shard of the same split (from
    shard_requests over the ranks' devices).  Without `gather` the rank's own
    (o, lse) are returned.  With it, each rank's results are padded to the
    largest shard and all-gathered (the only collective; every rank takes it,
    empty shards included), and every rank gets (o, lse) for the whole batch.
    """
    import torch.distributed as dist
    call = call or _default_call
    schedule = schedule or _default_schedule
    world = dist.get_world_size(group)
    device = local_inputs["q"].device
    s_q, h_q = local_inputs["q"].shape[1], local_inputs["q"].shape[2]
    if shard.size > 0:
        o_l, lse_l = call(local_inputs, schedule(local_inputs), softmax_scale)
    else:
        o_l = torch.empty((0, s_q, h_q, 512), dtype=torch.bfloat16, device=device)
        lse_l = torch.empty((0, s_q, h_q), dtype=torch.float32, device=device)
    if not gather:
        return o_l, lse_l
    bounds = torch.tensor([shard.start, shard.end], dtype=torch.int64, device=device)
    all_bounds = [torch.empty_like(bounds) for _ in range(world)]
    dist.all_gather(all_bounds, bounds, group=group)
    spans = [(int(b[0]), int(b[1])) for b in all_bounds]
    width = max(e - s for s, e in spans)
    # bf16 o travels as pairs packed in int32 words (every backend gathers int32); lse as float32
    pad_o = torch.zeros((width, s_q, h_q, 256), dtype=torch.int32, device=device)
    pad_l = torch.full((width, s_q, h_q), float("-inf"), dtype=torch.float32, device=device)
    pad_o[:shard.size] = o_l.contiguous().view(torch.int32)
    pad_l[:shard.size] = lse_l
    got_o = [torch.empty_like(pad_o) for _ in range(world)]
    got_l = [torch.empty_like(pad_l) for _ in range(world)]
    dist.all_gather(got_o, pad_o, group=group)
    dist.all_gather(got_l, pad_l, group=group)
    o = torch.empty((batch, s_q, h_q, 512), dtype=torch.bfloat16, device=device)
    lse = torch.empty((batch, s_q, h_q), dtype=torch.float32, device=device)
    for (s, e), go, gl in zip(spans, got_o, got_l):
        o[s:e] = go[:e - s].view(torch.bfloat16)
        lse[s:e] = gl[:e - s]
    return o, lse

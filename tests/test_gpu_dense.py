"""Dense MLA decode on the GPU against the float64 oracle: every query token
attends to all its visible cache tokens (causal mask optional), over paged
FP8 rows (656 bytes) or BF16 rows (1152 bytes), with the scheduler that splits
the work by the requests' lengths.  The scheduler tables are compared bit for
bit; o and lse under the parity tolerances, on every query token."""
import os

import numpy as np
import pytest

import oracle
from sparse_mla_decoding_b200 import workloads as W

import parity_util as PU

pytestmark = pytest.mark.gpu


def _bf16_cache(w, lay):
    """BF16 rows: the generator's latent and RoPE bf16 values, concatenated (no quantisation)."""
    rows = lay.num_blocks * W.BLOCK
    cache = np.empty((rows, 576), dtype=np.uint16)
    for start, lat, rope in W.cache_values(w, rows, chunk_rows=max(rows, 1) if rows <= W.GEN_CHUNK_ROWS
                                           else W.GEN_CHUNK_ROWS * 4):
        cache[start:start + lat.shape[0], :512] = lat
        cache[start:start + lat.shape[0], 512:] = rope
    b = np.frombuffer(cache.astype("<u2").tobytes(), np.uint8).reshape(rows, 1152).copy()
    b[W.unused_rows(lay)] = 0xFF   # NaN bf16 patterns in rows no visible position reaches
    return b.reshape(lay.num_blocks, W.BLOCK, 1152)


def build(w, kv_format):
    lay = W.layout(w)
    if kv_format == oracle.KV_FP8:
        cache = PU.build_host_inputs(w).cache
    else:
        cache = _bf16_cache(w, lay)
    return dict(q_bits=W.queries(w), cache=cache, block_table=lay.block_table, seqlens=lay.seqlens.astype(np.int32))


def run(hi, w, kv_format, causal, num_sm_parts=None):
    import torch
    import sparse_mla_decoding_b200 as smla
    q = torch.from_numpy(hi["q_bits"].view(np.int16)).cuda().view(torch.bfloat16)
    kv = torch.from_numpy(hi["cache"]).cuda()
    bt = torch.from_numpy(hi["block_table"]).cuda()
    sl = torch.from_numpy(hi["seqlens"]).cuda()
    sm, ns, tp = smla.get_mla_metadata_dense(sl, w.h_q, s_q=w.s_q, causal=causal, num_sm_parts=num_sm_parts)
    ws = smla.new_workspace(w.batch, w.s_q, w.h_q, 1, sm.shape[0])
    o, lse = smla.flash_mla_dense_with_kvcache(q, kv, bt, sl, sm, ns, tp, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    st, raw = smla.get_device_status(ws)
    return o.float().cpu().numpy(), lse.cpu().numpy(), sm.cpu().numpy(), ns.cpu().numpy(), tp.cpu().numpy(), (st, raw)


SHAPES = [
    W.Workload("dense_h16_b3", batch=3, s_q=1, h_q=16, topk=1, seed=61, seqlens=(1, 64, 200)),
    W.Workload("dense_h64_sq2_ragged", batch=4, s_q=2, h_q=64, topk=1, seed=62, seqlens=(130, 63, 2, 1000)),
    W.Workload("dense_h128_varlen", batch=3, s_q=1, h_q=128, topk=1, seed=63, seqlens=(2048, 65, 700),
               outlier_channels=5),
    W.Workload("dense_h32_sq4_causal", batch=2, s_q=4, h_q=32, topk=1, seed=64, seqlens=(300, 3)),
]


@pytest.mark.parametrize("kv_format", [oracle.KV_FP8, oracle.KV_BF16], ids=["fp8", "bf16"])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("w", SHAPES, ids=[w.name for w in SHAPES])
def test_dense_decode_parity(w, causal, kv_format):
    hi = build(w, kv_format)
    o, lse, sm, ns, tp, (st, raw) = run(hi, w, kv_format, causal)
    assert st == 0, f"device status {raw:#x}"
    # the scheduler tables, bit for bit
    n = oracle.dense_tile_counts(hi["seqlens"], w.s_q, causal)
    sm_ref, ns_ref, tp_ref = oracle.sched_meta_varlen(n, sm.shape[0])
    assert np.array_equal(tp, tp_ref) and np.array_equal(ns, ns_ref) and np.array_equal(sm, sm_ref)
    ref = oracle.dense_decode(hi["q_bits"], hi["cache"], kv_format, hi["block_table"], hi["seqlens"], causal,
                              threads=os.cpu_count() or 1)
    PU.compare(o, lse, ref, f"{w.name} {'causal' if causal else 'full'} {'bf16' if kv_format else 'fp8'}")


@pytest.mark.parametrize("kv_format", [oracle.KV_FP8, oracle.KV_BF16], ids=["fp8", "bf16"])
def test_dense_h128_cluster_form_matches_default(kv_format):
    """The two-CTA cluster form of 128-head decodes (smla.set_head_pair_form) in
    the dense modes: bitwise equal to the default independent CTAs."""
    import sparse_mla_decoding_b200 as smla
    w = SHAPES[2]                    # dense_h128_varlen
    hi = build(w, kv_format)
    o1, l1, *_ , (st1, _) = run(hi, w, kv_format, True)
    prev = smla.set_head_pair_form(True)
    try:
        o2, l2, *_, (st2, _) = run(hi, w, kv_format, True)
    finally:
        smla.set_head_pair_form(prev)
    assert st1 == 0 and st2 == 0
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("parts", [1, 3, 148])
def test_dense_split_schedules(parts):
    """Every split count gives the same answer within the tolerances (one part: no combine)."""
    w = W.Workload("dense_splits", batch=2, s_q=1, h_q=64, topk=1, seed=65, seqlens=(1500, 400))
    hi = build(w, oracle.KV_FP8)
    o, lse, sm, ns, tp, (st, _) = run(hi, w, oracle.KV_FP8, True, num_sm_parts=parts)
    assert st == 0
    sm_ref, ns_ref, _ = oracle.sched_meta_varlen(oracle.dense_tile_counts(hi["seqlens"], 1, True), parts)
    assert np.array_equal(sm, sm_ref) and np.array_equal(ns, ns_ref)
    ref = oracle.dense_decode(hi["q_bits"], hi["cache"], oracle.KV_FP8, hi["block_table"], hi["seqlens"], True)
    PU.compare(o, lse, ref, f"dense parts={parts}")


def test_dense_scheduler_many_requests():
    """A scan over more requests than one CTA has threads."""
    import torch
    import sparse_mla_decoding_b200 as smla
    rng = np.random.default_rng(66)
    sl = rng.integers(0, 5000, 3000).astype(np.int32)
    sm, ns, tp = smla.get_mla_metadata_dense(torch.from_numpy(sl).cuda(), 64, s_q=1, causal=False,
                                             num_sm_parts=148)
    sm_ref, ns_ref, tp_ref = oracle.sched_meta_varlen(oracle.dense_tile_counts(sl, 1, False), 148)
    assert np.array_equal(tp.cpu().numpy(), tp_ref) and np.array_equal(ns.cpu().numpy(), ns_ref)
    assert np.array_equal(sm.cpu().numpy(), sm_ref)
    for s_q in (2, 3):
        sm, ns, tp = smla.get_mla_metadata_dense(torch.from_numpy(sl[:500]).cuda(), 64, s_q=s_q, causal=True,
                                                 num_sm_parts=74)
        sm_ref, ns_ref, tp_ref = oracle.sched_meta_varlen(oracle.dense_tile_counts(sl[:500], s_q, True), 74)
        assert np.array_equal(tp.cpu().numpy(), tp_ref) and np.array_equal(sm.cpu().numpy(), sm_ref)


def test_dense_bad_block_table_entry_is_skipped_and_flagged():
    w = W.Workload("dense_badbt", batch=1, s_q=1, h_q=16, topk=1, seed=67, seqlens=(256,))
    hi = build(w, oracle.KV_BF16)
    hi["block_table"] = hi["block_table"].copy()
    hi["block_table"][0, 1] = -7
    o, lse, *_, (st, raw) = run(hi, w, oracle.KV_BF16, False)
    assert st == 1 and raw & 2
    # positions 64..127 are skipped: the sparse oracle over the other positions
    keep = np.array([i for i in range(256) if not 64 <= i < 128], dtype=np.int32)
    q = hi["q_bits"][0, 0]
    k_rows = hi["cache"].reshape(-1, 1152)
    K = np.stack([oracle.bf16_row(k_rows[hi["block_table"][0, i // 64] * 64 + i % 64]) for i in keep])
    o_ref, lse_ref = oracle.attend(oracle.bf16_bits_to_f64(q), K, np.ones(len(keep), np.uint8))
    PU.compare(o, lse, {(0, 0): (o_ref, lse_ref)}, "dense badbt")

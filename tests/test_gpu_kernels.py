"""GPU parity of every kernel against the float64 oracle, through the C-ABI binding.

  * scheduler metadata: bit-exact against the oracle's restatement
  * KV writer (quantiser): bit-exact against the oracle's scalar quantiser
  * bounded device wait: gives up, flags the status word, GPU stays usable
  * split-KV decode + combine: o / lse within the stated tolerances on small
    workloads spanning several tiles and a ragged tail, every head count,
    split and unsplit schedules, invalid slots, all-invalid tokens, poisoned
    unused rows, exact single-slot outputs and run-to-run bitwise determinism
"""
import numpy as np
import pytest

import oracle
from sparse_mla_decoding_b200 import workloads as W

import parity_util as PU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available()
    return torch


@pytest.fixture(scope="module")
def smla(torch_cuda):
    import sparse_mla_decoding_b200 as m
    m.lib()
    return m


# ---------------------------------------------------------------------------
# scheduler
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("batch,s_q,topk,P", [(2, 1, 64, 148), (64, 1, 2048, 74), (128, 2, 2048, 148),
                                              (32, 1, 2048, 74), (1, 4096, 2048, 74), (7, 3, 100, 5),
                                              (1, 1, 1, 1), (5, 1, 7 * 64, 35), (13, 1, 128, 3),
                                              (3, 1, 6400, 7), (200, 1, 64, 16), (9, 1, 1000, 300)])
def test_sched_meta_bit_exact(smla, torch_cuda, batch, s_q, topk, P):
    torch = torch_cuda
    seqlens = torch.full((batch,), 100, dtype=torch.int32, device="cuda")
    sm, ns = smla.get_mla_metadata(seqlens, topk, 64, P, s_q=s_q)
    sm_ref, ns_ref = oracle.sched_meta(batch * s_q, -(-topk // 64), P)
    assert np.array_equal(sm.cpu().numpy(), sm_ref)
    assert np.array_equal(ns.cpu().numpy(), ns_ref)


# ---------------------------------------------------------------------------
# KV writer
# ---------------------------------------------------------------------------

def test_quantize_kv_bit_exact(smla, torch_cuda):
    torch = torch_cuda
    rng = np.random.default_rng(7)
    n = 777
    lat = rng.standard_normal((n, 512)).astype(np.float32) * np.float32(2.0)
    lat[::5, 3] *= 8.0
    lat[1, :128] = 0.0
    lat[2, :] = 0.0
    lat[3, 128:256] = 2.0 ** -120
    lat[4, 256:384] = -0.0
    lat[5, 384:] = np.float32(3e38)
    lat[6, 7] = -448.0
    lat_bits = W._to_bf16_bits(lat)
    rope_bits = W._to_bf16_bits(rng.standard_normal((n, 64)).astype(np.float32))
    ref = oracle.quantize_tokens(lat_bits, rope_bits)
    dev_lat = torch.from_numpy(lat_bits.view(np.int16)).cuda().view(torch.bfloat16)
    dev_rope = torch.from_numpy(rope_bits.view(np.int16)).cuda().view(torch.bfloat16)
    cache = torch.zeros((n, 656), dtype=torch.uint8, device="cuda")
    smla.quantize_kv(dev_lat, dev_rope, cache)
    got = cache.cpu().numpy()
    assert np.array_equal(got, ref)
    # scattered writes through a slot mapping; negative slots are skipped
    perm = rng.permutation(n + 40)[:n].astype(np.int64)
    perm[::9] = -1
    cache2 = torch.full((n + 40, 656), 0xAB, dtype=torch.uint8, device="cuda")
    smla.quantize_kv(dev_lat, dev_rope, cache2, torch.from_numpy(perm).cuda())
    got2 = cache2.cpu().numpy()
    for i in range(n):
        if perm[i] >= 0:
            assert np.array_equal(got2[perm[i]], ref[i])
    untouched = np.setdiff1d(np.arange(n + 40), perm[perm >= 0])
    assert (got2[untouched] == 0xAB).all()


# ---------------------------------------------------------------------------
# bounded wait
# ---------------------------------------------------------------------------

def test_bounded_wait_gives_up_and_flags(smla, torch_cuda):
    torch = torch_cuda
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert smla.get_device_status(ws) == (0, 0)
    smla.selftest_bounded_wait(ws, 2_000_000)       # 2 ms
    torch.cuda.synchronize()
    st, raw = smla.get_device_status(ws)
    assert st == 4 and raw & 1
    smla.reset_device_status(ws)
    assert smla.get_device_status(ws) == (0, 0)
    # the context is still usable
    assert float(torch.ones(4, device="cuda").sum()) == 4.0


# ---------------------------------------------------------------------------
# decode parity
# ---------------------------------------------------------------------------

def _check(w, num_sm_parts=None, tokens=None, indices=None, softmax_scale=None):
    hi = PU.build_host_inputs(w, indices=indices)
    o, lse, sm, ns = PU.run_gpu(hi, num_sm_parts=num_sm_parts, softmax_scale=softmax_scale)
    toks = tokens or [(b, t) for b in range(w.batch) for t in range(w.s_q)]
    ref = PU.oracle_tokens(hi, toks, softmax_scale=softmax_scale)
    return hi, o, lse, PU.compare(o, lse, ref, w.name), ns


def test_tiny_workload_all_tokens(smla):
    _check(W.TINY)


@pytest.mark.parametrize("h_q", [16, 32, 64, 128])
@pytest.mark.parametrize("topk", [1, 64, 100, 300])
def test_heads_and_ragged_topk(smla, h_q, topk):
    w = W.Workload(f"ragged_h{h_q}_k{topk}", batch=3, s_q=2, h_q=h_q, topk=topk, seed=100 + topk,
                   seqlens=(700, 130, 1000), index_mode="uniform", invalid_per_token=topk // 10)
    _check(w)


@pytest.mark.parametrize("P", [1, 2, 5, 37, 148])
def test_split_schedules(smla, P):
    w = W.Workload("splits", batch=4, s_q=1, h_q=64, topk=640, seed=77, seqlens=(2000, 1500, 700, 3000),
                   index_mode="uniform", invalid_per_token=40)
    _, _, _, _, ns = _check(w, num_sm_parts=P)
    if P >= 37:
        assert (np.diff(ns) > 1).any(), "expected at least one split request"


def test_h128_long_topk_many_splits(smla):
    w = W.Workload("h128_2048", batch=3, s_q=1, h_q=128, topk=2048, seed=91, seqlens=(8192, 4100, 2500),
                   index_mode="uniform", outlier_channels=5)
    _check(w)


@pytest.mark.parametrize("P", [None, 7], ids=["default_parts", "7_parts"])
def test_h128_head_pair_form_matches_independent_ctas(smla, torch_cuda, P):
    """The two-CTA cluster form (each CTA dequantises half of every tile and
    copies it to its peer) and the default independent CTAs give bitwise
    identical o and lse, and both pass the oracle comparison."""
    import sparse_mla_decoding_b200 as m
    w = W.Workload("h128_pairs", batch=3, s_q=2, h_q=128, topk=700, seed=93, seqlens=(3000, 900, 5000),
                   index_mode="uniform", invalid_per_token=50)
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    o1, l1, _, _ = PU.run_gpu(hi, dev_inputs=d, num_sm_parts=P)
    prev = m.set_head_pair_form(True)
    try:
        o2, l2, _, _ = PU.run_gpu(hi, dev_inputs=d, num_sm_parts=P)
    finally:
        m.set_head_pair_form(prev)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    toks = [(b, t) for b in range(w.batch) for t in range(w.s_q)]
    PU.compare(o2, l2, PU.oracle_tokens(hi, toks), w.name + " pair form")


def test_invalid_slots_and_all_invalid_tokens(smla):
    w = W.Workload("invalid", batch=3, s_q=2, h_q=64, topk=192, seed=5, seqlens=(300, 64, 1000),
                   index_mode="uniform")
    lay = W.layout(w)
    idx = W.indices(w, lay.seqlens)
    idx[0, 0, :] = -1                                  # every slot skipped -> o = 0, lse = -inf
    idx[1, 1, :] = np.arange(64, 64 + 192)             # all at or past seqlen 64 -> invalid
    idx[2, 0, ::3] = -5                                # other negative values are skips too
    idx[2, 1, 10:20] = 10 ** 6                         # far past the length
    _check(w, indices=idx)


def test_single_valid_slot_is_exact(smla):
    w = W.Workload("single", batch=2, s_q=1, h_q=32, topk=96, seed=8, seqlens=(500, 90), index_mode="uniform")
    lay = W.layout(w)
    idx = np.full((2, 1, 96), -1, np.int32)
    idx[0, 0, 70] = 321
    idx[1, 0, 0] = 89
    hi = PU.build_host_inputs(w, indices=idx)
    o, lse, _, _ = PU.run_gpu(hi)
    for b, pos in ((0, 321), (1, 89)):
        phys = hi.block_table[b, pos // 64] * 64 + pos % 64
        v = oracle.dequantize_row(hi.cache.reshape(-1, 656)[phys])[:512]
        assert np.array_equal(o[b, 0], np.broadcast_to(v, o[b, 0].shape))   # P = 1 exactly, V exact in bf16


def test_softmax_scale_argument(smla):
    w = W.TINY.with_(name="tiny_scale")
    _check(w, softmax_scale=0.11)


@pytest.mark.parametrize("bad_entry", [10 ** 6, -5], ids=["past_cache", "negative"])
def test_bad_block_table_entry_is_skipped_and_flagged(smla, torch_cuda, bad_entry):
    torch = torch_cuda
    w = W.Workload("badbt", batch=1, s_q=1, h_q=16, topk=64, seed=9, seqlens=(256,), index_mode="uniform")
    hi = PU.build_host_inputs(w)
    bt = hi.block_table.copy()
    bt[0, 2] = bad_entry                                # outside the cache
    d = PU.to_device(hi)
    d["block_table"] = torch.from_numpy(bt).cuda()
    import sparse_mla_decoding_b200 as m
    sm, ns = m.get_mla_metadata(d["cache_seqlens"], 64, 16, s_q=1)
    ws = m.new_workspace(1, 1, 16, 64, sm.shape[0])
    o, lse = m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"],
                                      sm, ns, workspace=ws)
    st, raw = m.get_device_status(ws)
    assert st == 1 and raw & 2
    # the skipped slots are those whose block is the bad one: oracle with them marked invalid
    idx = hi.indices.copy()
    idx[(idx >= 128) & (idx < 192)] = -1
    ref = PU.oracle_tokens(PU.HostInputs(hi.w, hi.q_bits, hi.cache, hi.block_table, hi.seqlens, idx), [(0, 0)])
    PU.compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref, "badbt")


def test_bitwise_deterministic(smla, torch_cuda):
    w = W.Workload("det", batch=4, s_q=1, h_q=128, topk=1024, seed=12, seqlens=(4096,) * 4, index_mode="uniform")
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    o1, l1, _, _ = PU.run_gpu(hi, dev_inputs=d)
    o2, l2, _, _ = PU.run_gpu(hi, dev_inputs=d)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_repeated_calls_with_many_request_ends_are_bitwise_identical(smla, torch_cuda):
    """Requests of one or two tiles put an epilogue (a wait for the last PV, then
    O read out of TMEM) on almost every tile, with split requests on both sides of
    every part boundary: the pattern where a softmax warp running ahead of the PV
    issuer could read O early.  Repeated calls must agree bit for bit, and the
    first must pass the oracle comparison."""
    w = W.Workload("many_ends", batch=96, s_q=1, h_q=128, topk=96, seed=14, seqlens=tuple([300, 70, 1500] * 32),
                   index_mode="uniform", invalid_per_token=9)
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    o1, l1, _, ns = PU.run_gpu(hi, dev_inputs=d, num_sm_parts=39)   # 5 tiles a part: every other boundary splits
    assert (np.diff(ns) > 1).any(), "expected split requests"
    for _ in range(4):
        o2, l2, _, _ = PU.run_gpu(hi, dev_inputs=d, num_sm_parts=39)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    toks = [(b, 0) for b in range(0, w.batch, 7)]
    PU.compare(o1, l1, PU.oracle_tokens(hi, toks), w.name)


def test_dequant_every_code_and_scale_range_is_exact(smla, torch_cuda):
    """A single valid slot makes o equal its value row exactly, so o exposes the
    dequantised latent values: every e4m3 code (NaN codes included) times
    scales from subnormal to > 2^8 must equal bf16(float(e4m3) * scale)."""
    torch = torch_cuda
    scales = [1.0, 2.0 ** -20, 3.7e-3, 300.0, 2.0 ** -130, 0.0, 1.5e-38, 123.456]
    rows = []
    for r, sc0 in enumerate(scales):
        row = np.zeros(656, np.uint8)
        codes = (np.arange(512) * 7 + 37 * r) % 256
        codes[(codes & 0x7F) == 0x7F] -= 1              # the NaN codes poison S as well: kept out here
        row[:512] = codes
        row[512:528] = np.array([sc0, scales[(r + 1) % len(scales)], scales[(r + 3) % len(scales)], 1.0],
                                np.float32).view(np.uint8)
        row[528:] = 0                                      # zero RoPE: the scores stay finite
        rows.append(row)
    n = len(rows)
    cache = np.zeros((1, 64, 656), np.uint8)
    cache[0, :n] = np.stack(rows)
    q_bits = W._to_bf16_bits(np.random.default_rng(3).standard_normal((n, 1, 16, 576)).astype(np.float32) * 0.01)
    idx = np.full((n, 1, 64), -1, np.int32)
    for r in range(n):
        idx[r, 0, 5] = r
    w = W.Workload("codes", batch=n, s_q=1, h_q=16, topk=64, seed=0, seqlens=(64,) * n)
    hi = PU.HostInputs(w, q_bits, cache, np.zeros((n, 1), np.int32), np.full(n, 64, np.int32), idx)
    d = PU.to_device(hi)
    import sparse_mla_decoding_b200 as m
    sm, ns = m.get_mla_metadata(d["cache_seqlens"], 64, 16, s_q=1)
    o, lse = m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns)
    o = o.float().cpu().numpy()
    for r in range(n):
        v = oracle.dequantize_row(cache[0, r])[:512]
        got = o[r, 0]
        assert np.array_equal(np.isnan(got), np.broadcast_to(np.isnan(v), got.shape)), f"row {r}: NaN pattern"
        ok = ~np.isnan(v)
        assert np.array_equal(got[:, ok], np.broadcast_to(v[ok], (16, ok.sum()))), f"row {r} (scale {scales[r]})"
    # a NaN code in a valid row reaches every score of the token: its output is NaN
    cache2 = cache.copy()
    cache2[0, 0, 100] = 0x7F
    d["kvcache"] = torch.from_numpy(cache2).cuda()
    o2, _ = m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns)
    assert np.isnan(o2[0, 0].float().cpu().numpy()).all()


def test_flags_reach_callers_without_a_workspace(smla, torch_cuda):
    """Calls that pass no workspace share one per device and stream; its status
    word must report a skipped bad block-table entry, survive the buffer being
    replaced by a larger one, and make check_device_status raise."""
    torch = torch_cuda
    import sparse_mla_decoding_b200 as m
    w = W.Workload("badbt_cached", batch=1, s_q=1, h_q=16, topk=64, seed=19, seqlens=(256,), index_mode="uniform")
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    d["block_table"][0, 1] = -1
    sm, ns = m.get_mla_metadata(d["cache_seqlens"], 64, 16, s_q=1)
    m.reset_cached_workspace_status()
    m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns)
    st, raw = m.cached_workspace_status()
    assert st == 1 and raw & 2
    # a larger call replaces the shared buffer; the flag is carried over
    w2 = W.Workload("grow_cached", batch=8, s_q=1, h_q=128, topk=512, seed=20, seqlens=(1024,) * 8,
                    index_mode="uniform")
    hi2 = PU.build_host_inputs(w2)
    d2 = PU.to_device(hi2)
    sm2, ns2 = m.get_mla_metadata(d2["cache_seqlens"], 512, 128, s_q=1)
    m.flash_mla_with_kvcache(d2["q"], d2["kvcache"], d2["block_table"], d2["cache_seqlens"], d2["indices"], sm2, ns2)
    st, raw = m.cached_workspace_status()
    assert st == 1 and raw & 2
    with pytest.raises(m.SmlaError):
        m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns,
                                 check_device_status=True)
    m.reset_cached_workspace_status()
    assert m.cached_workspace_status() == (0, 0)
    d["block_table"][0, 1] = hi.block_table[0, 1]
    m.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"], sm, ns,
                             check_device_status=True)

"""The allocation-free entry point, smla_flash_mla_with_kvcache_static_scratch.

It serves callers that cannot allocate device memory (allocator-less
runtimes, embedders that only hand over inputs and outputs, code where an
allocation would synchronise or is not allowed): its split-KV scratch lives in
a fixed 64 MiB array inside the library instead of a caller workspace.  Here it
is called through the C ABI and its output is checked against the regular
entry point's on two calls in a row (the array keeps the previous call's
contents, which must not leak into the next): within the parity tolerances,
and bit for bit, since the same kernels run with only the scratch pointer
changed.  A flagged condition (a bad block-table entry) must reach the
caller's status word through this entry point.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from sparse_mla_decoding_b200 import workloads as W

import parity_util as PU

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 64 * 1024 * 1024


def _entry():
    import sparse_mla_decoding_b200 as smla
    f = smla.lib().smla_flash_mla_with_kvcache_static_scratch
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    f.argtypes = [vp, vp, i64, vp, i32, vp, vp, vp, vp, i32, f32, i32, i32, i32, i32, vp, vp, vp, vp]
    f.restype = i32
    return f


def _call_static(d, sm, ns, w, o, lse, status=None):
    import torch
    f = _entry()
    return f(d["q"].data_ptr(), d["kvcache"].data_ptr(), d["kvcache"].shape[0], d["block_table"].data_ptr(),
             d["block_table"].shape[1], d["cache_seqlens"].data_ptr(), d["indices"].data_ptr(), sm.data_ptr(),
             ns.data_ptr(), sm.shape[0], -1.0, w.batch, w.s_q, w.h_q, d["indices"].shape[2], o.data_ptr(),
             lse.data_ptr(), None if status is None else status.data_ptr(),
             torch.cuda.current_stream().cuda_stream)


def _as_ref(o, lse):
    """Outputs of the regular entry point in the form parity_util.compare takes."""
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    return {(b, t): (o[b, t], lse[b, t]) for b in range(o.shape[0]) for t in range(o.shape[1])}


@pytest.mark.parametrize("w", [
    W.Workload("static_h128", batch=6, s_q=1, h_q=128, topk=2048, seed=41, seqlens=(8192, 5000, 3000, 8192, 2100,
                                                                                    7000),
               index_mode="uniform", outlier_channels=5),
    W.Workload("static_h64_sq2", batch=5, s_q=2, h_q=64, topk=700, seed=42, seqlens=(4096, 900, 3000, 64, 2000),
               index_mode="uniform", invalid_per_token=70),
], ids=lambda w: w.name)
def test_static_scratch_matches_regular_entry(w):
    import torch
    import sparse_mla_decoding_b200 as smla
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    sm, ns = smla.get_mla_metadata(d["cache_seqlens"], hi.indices.shape[2], w.h_q, s_q=w.s_q)
    assert smla.workspace_bytes(w.batch, w.s_q, w.h_q, hi.indices.shape[2], sm.shape[0]) <= SCRATCH_LIMIT
    o_ref, lse_ref = smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                                 d["indices"], sm, ns)
    torch.cuda.synchronize()
    ref = _as_ref(o_ref, lse_ref)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = _call_static(d, sm, ns, w, o, lse, status=status if call == 1 else None)
        assert rc == 0, f"call {call}: status {rc}"
        torch.cuda.synchronize()
        PU.compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref, f"{w.name} static-scratch call {call}")
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"call {call} differs from the regular entry"
    assert int(status.item()) == 0


def test_static_scratch_reports_flags_to_the_caller():
    """A valid index whose block-table entry lies outside the cache is skipped
    and flagged; the flag must arrive in the caller's status word, and the
    other rows must match the regular entry point bit for bit."""
    import torch
    import sparse_mla_decoding_b200 as smla
    w = W.Workload("static_badbt", batch=2, s_q=1, h_q=64, topk=256, seed=43, seqlens=(512, 300),
                   index_mode="uniform")
    hi = PU.build_host_inputs(w)
    d = PU.to_device(hi)
    bt = d["block_table"].clone()
    bt[0, 1] = -3
    d["block_table"] = bt
    sm, ns = smla.get_mla_metadata(d["cache_seqlens"], hi.indices.shape[2], w.h_q, s_q=w.s_q)
    ws = smla.new_workspace(w.batch, w.s_q, w.h_q, hi.indices.shape[2], sm.shape[0])
    o_ref, lse_ref = smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                                 d["indices"], sm, ns, workspace=ws)
    st, raw = smla.get_device_status(ws)
    assert st == 1 and raw & 2
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(lse_ref, float("nan"))
    assert _call_static(d, sm, ns, w, o, lse, status=status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) & 2
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_static_scratch_rejects_oversized_calls():
    import torch
    import sparse_mla_decoding_b200 as smla
    # 4096 requests x 128 heads of float32 partials need about 1 GiB, far past the 64 MiB array
    w = W.Workload("too_big", batch=4096, s_q=1, h_q=128, topk=2048, seed=1, seqlens=(64,) * 4096)
    need = smla.workspace_bytes(w.batch, w.s_q, w.h_q, w.topk, 74)
    assert need > SCRATCH_LIMIT
    small = dict(q=torch.zeros((1, 1, 128, 576), dtype=torch.bfloat16, device="cuda"),
                 kvcache=torch.zeros((1, 64, 656), dtype=torch.uint8, device="cuda"),
                 block_table=torch.zeros((1, 1), dtype=torch.int32, device="cuda"),
                 cache_seqlens=torch.zeros(1, dtype=torch.int32, device="cuda"),
                 indices=torch.zeros((1, 1, 2048), dtype=torch.int32, device="cuda"))
    sm = torch.zeros((74, 8), dtype=torch.int32, device="cuda")
    ns = torch.zeros(2, dtype=torch.int32, device="cuda")
    o = torch.zeros((1, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    rc = _call_static(small, sm, ns, w, o, lse)          # sizes say 4096 requests: rejected before any launch
    assert rc == 5
    assert smla.lib().smla_status_string(5) == b"SMLA_ERR_SCRATCH_LIMIT"

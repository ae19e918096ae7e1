"""flash_mla_sparse_fwd (sparse attention of many query tokens over one flat FP8
cache) against the float64 oracle, through the C ABI.

Shapes span several index tiles with a ragged tail, the single-CTA (16/32/64
heads) and the two-CTA (128 heads) forms, topk = 1, indices that are negative
or past the cache, and a query token with no valid slot.  The entry runs the
decode path on a flat cache, so it must also agree bit for bit with the decode
entry called on the same rows through an identity block table.
"""
import numpy as np
import pytest
import torch

import oracle
import parity_util as PU
import sparse_mla_decoding_b200 as smla

pytestmark = pytest.mark.gpu


def _inputs(seed, s_q, h_q, s_kv, topk, dead_token=None):
    rng = np.random.default_rng(seed)
    lat = torch.from_numpy(rng.standard_normal((s_kv, 512)).astype(np.float32)).to(torch.bfloat16)
    rope = torch.from_numpy(rng.standard_normal((s_kv, 64)).astype(np.float32)).to(torch.bfloat16)
    kv = oracle.quantize_tokens_bulk(lat.view(torch.int16).numpy().view(np.uint16),
                                     rope.view(torch.int16).numpy().view(np.uint16))
    q = torch.from_numpy(rng.standard_normal((s_q, h_q, 576)).astype(np.float32)).to(torch.bfloat16)
    q_bits = q.view(torch.int16).numpy().view(np.uint16)
    idx = rng.integers(-3, s_kv + 8, size=(s_q, 1, topk)).astype(np.int32)
    if dead_token is not None:
        idx[dead_token] = -1
    return q, q_bits, kv, idx


def _run(q, kv, idx, h_q, s_q, s_kv, topk):
    dev = torch.device("cuda", 0)
    parts = smla.default_num_sm_parts(h_q, dev)
    ws = smla.new_sparse_fwd_workspace(s_q, h_q, s_kv, topk, parts, dev)
    o, lse = smla.flash_mla_sparse_fwd(q.to(dev), torch.from_numpy(kv).to(dev), torch.from_numpy(idx).to(dev),
                                       workspace=ws)
    torch.cuda.synchronize()
    assert smla.get_device_status(ws) == (0, 0)
    return o, lse


@pytest.mark.parametrize("s_q,h_q,s_kv,topk", [(130, 64, 1000, 200), (70, 128, 333, 64), (9, 16, 64, 1),
                                               (33, 32, 5000, 300)])
def test_sparse_fwd_matches_oracle(s_q, h_q, s_kv, topk):
    q, q_bits, kv, idx = _inputs(7 + s_q, s_q, h_q, s_kv, topk, dead_token=min(3, s_q - 1))
    o, lse = _run(q, kv, idx, h_q, s_q, s_kv, topk)
    ref = oracle.sparse_prefill(q_bits, kv, idx)
    refs = {(0, t): v for t, v in ref.items()}
    PU.compare(o.float().cpu().numpy()[None], lse.cpu().numpy()[None], refs, what=f"sparse_fwd {s_q}x{h_q}")


def test_sparse_fwd_equals_decode_with_identity_block_table():
    s_q, h_q, s_kv, topk = 40, 128, 700, 128
    q, _, kv, idx = _inputs(99, s_q, h_q, s_kv, topk)
    o, lse = _run(q, kv, idx, h_q, s_q, s_kv, topk)
    dev = torch.device("cuda", 0)
    nb = (s_kv + 63) // 64
    cache = torch.zeros((nb * 64, 656), dtype=torch.uint8)
    cache[:s_kv] = torch.from_numpy(kv)
    cache = cache.view(nb, 64, 656).to(dev)
    seqlens = torch.tensor([s_kv], dtype=torch.int32, device=dev)
    sm, ns = smla.get_mla_metadata(seqlens, topk, h_q, s_q=s_q)
    o2, lse2 = smla.flash_mla_with_kvcache(q.to(dev)[None], cache, torch.arange(nb, dtype=torch.int32, device=dev)[None],
                                           seqlens, torch.from_numpy(idx).to(dev).view(1, s_q, topk), sm, ns)
    torch.cuda.synchronize()
    assert torch.equal(o, o2[0]) and torch.equal(lse, lse2[0])

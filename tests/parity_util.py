"""Shared helpers for the parity tests: build a workload's inputs on the host
(values from the seeded generator, cache rows from the oracle's quantiser,
unused rows poisoned), run the CUDA path through the C-ABI binding, and
compare with the float64 oracle under the stated tolerances."""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

import oracle
from sparse_mla_decoding_b200 import workloads as W

# Parity bar for floating point (o in bf16, lse in float32 natural log):
#   |o - o_ref| <= 1e-2 + half a bf16 ulp of o_ref, elementwise
#   ||o - o_ref||_2 / ||o_ref||_2 <= 5e-3
#   |lse - lse_ref| <= 1e-3, -inf exactly where no slot is valid (and o = 0 there)
# The half-ulp term is the rounding of the bf16 output format itself: no bf16
# value is closer than that to the exact result, and with outlier channels
# |o| exceeds 8, where half an ulp is 2^-5 > 1e-2.
TOL_O_MAX = 1e-2
TOL_O_REL_L2 = 5e-3
TOL_LSE = 1e-3


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


@dataclass
class HostInputs:
    w: W.Workload
    q_bits: np.ndarray          # [b, s_q, h, 576] uint16
    cache: np.ndarray           # [num_blocks, 64, 656] uint8
    block_table: np.ndarray     # [b, max_blocks] int32
    seqlens: np.ndarray         # [b] int32
    indices: np.ndarray         # [b, s_q, topk] int32


def build_host_inputs(w: W.Workload, indices: Optional[np.ndarray] = None) -> HostInputs:
    lay = W.layout(w)
    rows = lay.num_blocks * W.BLOCK
    cache = np.empty((rows, W.ROW_BYTES), dtype=np.uint8)
    for start, lat, rope in W.cache_values(w, rows, chunk_rows=max(rows, 1) if rows <= W.GEN_CHUNK_ROWS
                                           else W.GEN_CHUNK_ROWS * 4):
        cache[start:start + lat.shape[0]] = oracle.quantize_tokens_bulk(lat, rope)
    W.poison(cache, W.unused_rows(lay))
    idx = W.indices(w, lay.seqlens) if indices is None else indices.astype(np.int32)
    return HostInputs(w=w, q_bits=W.queries(w), cache=cache.reshape(lay.num_blocks, W.BLOCK, W.ROW_BYTES),
                      block_table=lay.block_table, seqlens=lay.seqlens.astype(np.int32), indices=idx)


def to_device(hi: HostInputs, device="cuda"):
    import torch
    q = torch.from_numpy(hi.q_bits.view(np.int16)).to(device).view(torch.bfloat16)
    return dict(q=q,
                kvcache=torch.from_numpy(hi.cache).to(device),
                block_table=torch.from_numpy(hi.block_table).to(device),
                cache_seqlens=torch.from_numpy(hi.seqlens).to(device),
                indices=torch.from_numpy(hi.indices).to(device))


def run_gpu(hi: HostInputs, num_sm_parts: Optional[int] = None, softmax_scale=None, dev_inputs=None):
    import torch
    import sparse_mla_decoding_b200 as smla
    d = dev_inputs or to_device(hi)
    sm, ns = smla.get_mla_metadata(d["cache_seqlens"], hi.indices.shape[2], hi.w.h_q, num_sm_parts, s_q=hi.w.s_q)
    ws = smla.new_workspace(hi.w.batch, hi.w.s_q, hi.w.h_q, hi.indices.shape[2], sm.shape[0])
    o, lse = smla.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], d["indices"],
                                         sm, ns, softmax_scale=softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    status, raw = smla.get_device_status(ws)
    assert status == 0, f"device status word set: {raw:#x}"
    return o.float().cpu().numpy(), lse.cpu().numpy(), sm.cpu().numpy(), ns.cpu().numpy()


def oracle_tokens(hi: HostInputs, tokens: Sequence[Tuple[int, int]], softmax_scale=None, threads: int = 8):
    scale = oracle.DEFAULT_SOFTMAX_SCALE if softmax_scale is None else softmax_scale
    return oracle.sparse_decode(hi.q_bits, hi.cache, hi.block_table, hi.seqlens, hi.indices, scale,
                                tokens=list(tokens), threads=threads)


def compare(o_gpu: np.ndarray, lse_gpu: np.ndarray, ref: Dict, what: str = "") -> dict:
    """Check every sampled token; return the worst errors seen."""
    worst = dict(o_max=0.0, o_max_beyond_rounding=0.0, o_rel_l2=0.0, lse=0.0)
    num = den = 0.0
    for (b, t), (o_ref, lse_ref) in ref.items():
        og = o_gpu[b, t].astype(np.float64)
        lg = lse_gpu[b, t].astype(np.float64)
        dead = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lg), dead), f"{what} token {(b, t)}: -inf lse mismatch"
        assert (og[dead] == 0).all(), f"{what} token {(b, t)}: o must be exactly 0 where no slot is valid"
        assert np.isfinite(og).all(), f"{what} token {(b, t)}: non-finite o"
        diff = np.abs(og - o_ref)
        worst["o_max"] = max(worst["o_max"], float(diff.max()) if og.size else 0.0)
        beyond = diff - half_ulp_bf16(o_ref)
        worst["o_max_beyond_rounding"] = max(worst["o_max_beyond_rounding"],
                                             float(beyond.max()) if og.size else 0.0)
        num += float(((og - o_ref) ** 2).sum())
        den += float((o_ref ** 2).sum())
        if (~dead).any():
            worst["lse"] = max(worst["lse"], float(np.abs(lg[~dead] - lse_ref[~dead]).max()))
    worst["o_rel_l2"] = (num / den) ** 0.5 if den > 0 else 0.0
    assert worst["o_max_beyond_rounding"] <= TOL_O_MAX, \
        f"{what}: max(|o-o_ref| - ulp/2) = {worst['o_max_beyond_rounding']:.3e} > {TOL_O_MAX}"
    assert worst["o_rel_l2"] <= TOL_O_REL_L2, f"{what}: rel L2 = {worst['o_rel_l2']:.3e} > {TOL_O_REL_L2}"
    assert worst["lse"] <= TOL_LSE, f"{what}: max|lse-lse_ref| = {worst['lse']:.3e} > {TOL_LSE}"
    return worst


def sample_tokens(w: W.Workload, k: int, seed: int = 123) -> List[Tuple[int, int]]:
    rng = np.random.default_rng(seed)
    all_tok = [(b, t) for b in range(w.batch) for t in range(w.s_q)]
    if k >= len(all_tok):
        return all_tok
    pick = rng.choice(len(all_tok), size=k, replace=False)
    # always include the first and last token (ragged edges of the schedule)
    chosen = {all_tok[0], all_tok[-1], *[all_tok[i] for i in pick]}
    return sorted(chosen)

"""Seeded synthetic workloads for sparse MLA decoding.

This module only draws random numbers and arranges them into the shapes the
operator consumes: query tokens, cache values (before quantisation), paged
block tables, per-request lengths and top-k index lists.  It holds none of the
operator's arithmetic (no quantisation, no attention), so both the CUDA path
and the float64 oracle can be fed from it without sharing any of the method.

Recipe (every stream has its own child seed of ``numpy.random.SeedSequence``):
  q        : N(0,1) float32 -> bf16 (round-to-nearest-even), [b, s_q, h_q, 576]
  latent   : N(0,1) float32, optional outlier channels x8, -> bf16, [rows, 512]
  rope     : N(0,1) float32 -> bf16, [rows, 64]
  blocks   : one random permutation of all used cache blocks (block size 64)
  indices  : per query token, distinct positions drawn as the workload says,
             then optionally a fixed number of slots set to -1
Unused rows (past a request's length inside its last block) and one spare
block that padded block-table slots point to are filled with NaN patterns
("poison") after quantisation, so any read of them shows up in the output.

The five named workloads are the decode shapes the operator is measured on:
a tiny 16-head check, a 128-head batch-64 decode, a 64-head two-token decode,
a long-context variable-length decode and a prefill-shaped 4096-token call.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Iterator, Optional, Sequence, Tuple

import numpy as np

DQK, DV, DROPE, ROW_BYTES, BLOCK = 576, 512, 64, 656, 64
GEN_CHUNK_ROWS = 1 << 16          # fixed chunk size for the cache-value streams


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    topk: int
    seed: int
    # per-request cache lengths: either a fixed tuple, or drawn uniformly from [lo, hi]
    seqlens: Optional[Tuple[int, ...]] = None
    seqlen_range: Optional[Tuple[int, int]] = None
    # index structure: "uniform" | "recent_mix" | "causal"
    index_mode: str = "uniform"
    invalid_per_token: int = 0        # slots set to -1 at random positions
    recent_window: int = 4096         # recent_mix: half the slots from the last `recent_window` positions
    causal_base: int = 0              # causal: token p may see positions < causal_base + p
    outlier_channels: int = 0         # latent channels multiplied by 8 before quantisation
    outlier_factor: float = 8.0

    def lengths(self) -> np.ndarray:
        if self.seqlens is not None:
            assert len(self.seqlens) == self.batch
            return np.asarray(self.seqlens, dtype=np.int64)
        lo, hi = self.seqlen_range
        rng = np.random.default_rng(_child(self.seed, "seqlens"))
        return rng.integers(lo, hi, size=self.batch, endpoint=True).astype(np.int64)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def summary(self) -> dict:
        d = dataclasses.asdict(self)
        return {k: v for k, v in d.items() if v not in (None, 0, "")}


# The measured shapes.  Lengths, index mixes and value distributions follow the
# decode configurations the operator is specified on; the readings of the
# open points (how many slots are -1, which channels are outliers) are stated
# in the repository's design notes.
TINY = Workload("tiny_h16_b2_topk64", batch=2, s_q=1, h_q=16, topk=64, seed=0, seqlens=(256, 200),
                index_mode="uniform", invalid_per_token=6)
DECODE_H128 = Workload("decode_h128_b64_topk2048", batch=64, s_q=1, h_q=128, topk=2048, seed=1,
                       seqlens=(8192,) * 64, index_mode="uniform", outlier_channels=5)
DECODE_H64_SQ2 = Workload("decode_h64_b128_sq2_topk2048", batch=128, s_q=2, h_q=64, topk=2048, seed=2,
                          seqlens=(32768,) * 128, index_mode="recent_mix", invalid_per_token=102)
LONG_VARLEN = Workload("longctx_varlen_h128_b32_topk2048", batch=32, s_q=1, h_q=128, topk=2048, seed=3,
                       seqlen_range=(4096, 131072), index_mode="uniform")
PREFILL_SHAPED = Workload("prefill_shaped_h128_sq4096_topk2048", batch=1, s_q=4096, h_q=128, topk=2048,
                          seed=4, seqlens=(65536,), index_mode="causal", causal_base=61440)

ALL = (TINY, DECODE_H128, DECODE_H64_SQ2, LONG_VARLEN, PREFILL_SHAPED)
BY_NAME = {w.name: w for w in ALL}

_STREAMS = ("q", "latent", "rope", "outliers", "blocks", "indices", "invalid", "seqlens")


def _child(seed: int, stream: str) -> np.random.SeedSequence:
    return np.random.SeedSequence(seed).spawn(len(_STREAMS))[_STREAMS.index(stream)]


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16) with round-to-nearest-even (torch's cast)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class Layout:
    """Paged-cache geometry of a workload (no values)."""
    seqlens: np.ndarray        # [b] int64
    blocks_per_req: np.ndarray  # [b]
    max_blocks: int
    num_used_blocks: int
    num_blocks: int            # used blocks + 1 spare (poisoned) block
    block_table: np.ndarray    # [b, max_blocks] int32 (padding -> spare block)
    spare_block: int


def layout(w: Workload) -> Layout:
    L = w.lengths()
    nb = (L + BLOCK - 1) // BLOCK
    used = int(nb.sum())
    maxb = int(max(1, nb.max() if len(nb) else 1))
    rng = np.random.default_rng(_child(w.seed, "blocks"))
    perm = rng.permutation(used).astype(np.int32)
    spare = used
    bt = np.full((w.batch, maxb), spare, dtype=np.int32)
    off = 0
    for i in range(w.batch):
        bt[i, :nb[i]] = perm[off:off + nb[i]]
        off += int(nb[i])
    return Layout(seqlens=L, blocks_per_req=nb, max_blocks=maxb, num_used_blocks=used,
                  num_blocks=used + 1, block_table=bt, spare_block=spare)


def queries(w: Workload) -> np.ndarray:
    """[b, s_q, h_q, 576] bf16 bit patterns."""
    rng = np.random.default_rng(_child(w.seed, "q"))
    x = rng.standard_normal((w.batch, w.s_q, w.h_q, DQK), dtype=np.float32)
    return _to_bf16_bits(x)


def outlier_channels(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(_child(w.seed, "outliers"))
    if w.outlier_channels <= 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(rng.choice(DV, size=w.outlier_channels, replace=False))


def cache_values(w: Workload, num_rows: int, chunk_rows: int = GEN_CHUNK_ROWS
                 ) -> Iterator[Tuple[int, np.ndarray, np.ndarray]]:
    """Yield (row_start, latent_bits [n,512], rope_bits [n,64]) for physical rows 0..num_rows-1.

    The streams are drawn in fixed GEN_CHUNK_ROWS pieces, so the values do not
    depend on the caller's chunk size (which must be a multiple of it, or the
    whole range)."""
    assert chunk_rows % GEN_CHUNK_ROWS == 0 or chunk_rows >= num_rows
    rl = np.random.default_rng(_child(w.seed, "latent"))
    rr = np.random.default_rng(_child(w.seed, "rope"))
    ch = outlier_channels(w)
    start = 0
    while start < num_rows:
        n = min(chunk_rows, num_rows - start)
        parts_l, parts_r = [], []
        done = 0
        while done < n:
            m = min(GEN_CHUNK_ROWS, n - done)
            lat = rl.standard_normal((m, DV), dtype=np.float32)
            if len(ch):
                lat[:, ch] *= np.float32(w.outlier_factor)
            parts_l.append(_to_bf16_bits(lat))
            parts_r.append(_to_bf16_bits(rr.standard_normal((m, DROPE), dtype=np.float32)))
            done += m
        yield start, np.concatenate(parts_l), np.concatenate(parts_r)
        start += n


def indices(w: Workload, seqlens: Sequence[int]) -> np.ndarray:
    """[b, s_q, topk] int32 top-k lists (logical positions within each request, -1 = skip)."""
    rng = np.random.default_rng(_child(w.seed, "indices"))
    rinv = np.random.default_rng(_child(w.seed, "invalid"))
    out = np.full((w.batch, w.s_q, w.topk), -1, dtype=np.int32)
    for b in range(w.batch):
        sl = int(seqlens[b])
        for t in range(w.s_q):
            if w.index_mode == "uniform":
                k = min(w.topk, sl)
                sel = rng.choice(sl, size=k, replace=False) if k > 0 else np.zeros(0, np.int64)
            elif w.index_mode == "recent_mix":
                win = min(w.recent_window, sl)
                k_recent = min(w.topk // 2, win)
                k_old = min(w.topk - k_recent, sl - win)
                recent = (sl - win) + rng.choice(win, size=k_recent, replace=False)
                old = rng.choice(sl - win, size=k_old, replace=False) if k_old > 0 else np.zeros(0, np.int64)
                sel = np.concatenate([recent, old])
                rng.shuffle(sel)
            elif w.index_mode == "causal":
                vis = min(sl, w.causal_base + t)
                k = min(w.topk, vis)
                sel = rng.choice(vis, size=k, replace=False) if k > 0 else np.zeros(0, np.int64)
            else:
                raise ValueError(w.index_mode)
            out[b, t, :len(sel)] = sel
            if w.invalid_per_token:
                pos = rinv.choice(w.topk, size=min(w.invalid_per_token, w.topk), replace=False)
                out[b, t, pos] = -1
    return out


def unused_rows(lay: Layout) -> np.ndarray:
    """Physical row ids that no valid index can reach (tails of last blocks + the spare block)."""
    rows = []
    for b in range(len(lay.seqlens)):
        nb = int(lay.blocks_per_req[b])
        if nb == 0:
            continue
        last = int(lay.block_table[b, nb - 1])
        used_in_last = int(lay.seqlens[b]) - (nb - 1) * BLOCK
        rows.extend(last * BLOCK + r for r in range(used_in_last, BLOCK))
    rows.extend(lay.spare_block * BLOCK + r for r in range(BLOCK))
    return np.asarray(rows, dtype=np.int64)


POISON_ROW = np.concatenate([
    np.full(512, 0x7F, dtype=np.uint8),                                        # e4m3 NaN codes
    np.frombuffer(np.array([0x7FC00000] * 4, dtype="<u4").tobytes(), np.uint8),  # NaN float32 scales
    np.frombuffer(np.array([0x7FC0] * 64, dtype="<u2").tobytes(), np.uint8),     # NaN bf16 RoPE
])
assert POISON_ROW.shape == (ROW_BYTES,)


def poison(cache_rows: np.ndarray, rows: np.ndarray) -> None:
    """Overwrite rows of a [num_rows, 656] uint8 cache view with the NaN pattern."""
    cache_rows[rows] = POISON_ROW

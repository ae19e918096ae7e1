"""Python face of the float64 CPU oracle (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or calls it.

Everything here is marshalling around ``oracle.c`` (numpy arrays <-> C
pointers) plus one bulk quantiser, ``quantize_tokens_bulk``, which restates
the per-tile quantisation with vectorised torch CPU float32 ops so that large
synthetic caches can be written in seconds; a CPU test pins it bit for bit to
the scalar C quantiser.  Sources are cited in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

DQK, DV, DROPE, ROW_BYTES, BLOCK = 576, 512, 64, 656, 64
DEFAULT_SOFTMAX_SCALE = 1.0 / math.sqrt(DQK)   # 1/24

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


class using_library:
    """Context manager that points the wrapper at another build of oracle.c
    (the mutation tests plant mistakes in a copy of the source)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def load(path: str) -> ctypes.CDLL:
    """Load a build of oracle.c and declare its C signatures."""
    L = ctypes.CDLL(path)
    c_u8p = ctypes.POINTER(ctypes.c_uint8)
    c_u16p = ctypes.POINTER(ctypes.c_uint16)
    c_i32p = ctypes.POINTER(ctypes.c_int32)
    c_dp = ctypes.POINTER(ctypes.c_double)
    L.smo_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.smo_e4m3_decode.restype = ctypes.c_double
    L.smo_e4m3_encode_satfinite.argtypes = [ctypes.c_float]
    L.smo_e4m3_encode_satfinite.restype = ctypes.c_uint8
    L.smo_bf16_from_float.argtypes = [ctypes.c_float]
    L.smo_bf16_from_float.restype = ctypes.c_uint16
    L.smo_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.smo_bf16_to_double.restype = ctypes.c_double
    L.smo_quantize_token.argtypes = [c_u16p, c_u16p, c_u8p]
    L.smo_quantize_token.restype = None
    L.smo_dequantize_row.argtypes = [c_u8p, c_dp]
    L.smo_dequantize_row.restype = None
    L.smo_attend.argtypes = [ctypes.c_int, c_dp, ctypes.c_int, c_dp, c_u8p, ctypes.c_double,
                             c_dp, c_dp, c_dp]
    L.smo_attend.restype = None
    L.smo_sparse_decode_token.argtypes = [ctypes.c_int, c_u16p, c_u8p, ctypes.c_int64, c_i32p,
                                          ctypes.c_int, ctypes.c_int32, c_i32p, ctypes.c_int,
                                          ctypes.c_double, c_dp, c_dp]
    L.smo_sparse_decode_token.restype = ctypes.c_int
    L.smo_combine.argtypes = [ctypes.c_int, ctypes.c_int, c_dp, c_dp, c_dp, c_dp]
    L.smo_combine.restype = None
    L.smo_sched_meta.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, c_i32p, c_i32p]
    L.smo_sched_meta.restype = ctypes.c_int
    L.smo_sched_meta_varlen.argtypes = [ctypes.c_int, c_i32p, ctypes.c_int, c_i32p, c_i32p, c_i32p]
    L.smo_sched_meta_varlen.restype = ctypes.c_int
    L.smo_bf16_row.argtypes = [c_u8p, c_dp]
    L.smo_bf16_row.restype = None
    L.smo_dense_visible_len.argtypes = [ctypes.c_int32, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    L.smo_dense_visible_len.restype = ctypes.c_int32
    L.smo_dense_decode_token.argtypes = [ctypes.c_int, c_u16p, c_u8p, ctypes.c_int, ctypes.c_int64, c_i32p,
                                         ctypes.c_int, ctypes.c_int32, ctypes.c_double, c_dp, c_dp]
    L.smo_dense_decode_token.restype = ctypes.c_int
    return L


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().smo_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    return int(lib().smo_e4m3_encode_satfinite(float(x)))


def bf16_from_float(x: float) -> int:
    return int(lib().smo_bf16_from_float(float(x)))


def bf16_to_float(h: int) -> float:
    return lib().smo_bf16_to_double(int(h) & 0xFFFF)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of bf16 bit patterns (uint16) as float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the 656-byte row
# --------------------------------------------------------------------------

def quantize_token(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """One token (512 + 64 bf16 bit patterns) -> 656 bytes, via the C quantiser."""
    lat = np.ascontiguousarray(latent_bits, dtype=np.uint16).reshape(DV)
    rop = np.ascontiguousarray(rope_bits, dtype=np.uint16).reshape(DROPE)
    row = np.zeros(ROW_BYTES, dtype=np.uint8)
    lib().smo_quantize_token(_ptr(lat, ctypes.c_uint16), _ptr(rop, ctypes.c_uint16), _ptr(row, ctypes.c_uint8))
    return row


def quantize_tokens(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """[N,512] + [N,64] bf16 bits -> [N,656] bytes with the scalar C quantiser (slow, exact)."""
    lat = np.ascontiguousarray(latent_bits, dtype=np.uint16).reshape(-1, DV)
    rop = np.ascontiguousarray(rope_bits, dtype=np.uint16).reshape(-1, DROPE)
    out = np.zeros((lat.shape[0], ROW_BYTES), dtype=np.uint8)
    L = lib()
    for i in range(lat.shape[0]):
        L.smo_quantize_token(_ptr(lat[i], ctypes.c_uint16), _ptr(rop[i], ctypes.c_uint16),
                             _ptr(out[i], ctypes.c_uint8))
    return out


def quantize_tokens_bulk(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """Vectorised restatement of the same per-tile quantiser with torch CPU ops.

    amax over each 1x128 tile (float32), scale = amax / 448 (float32 division),
    x / scale (float32 division), saturate to +-448, round to e4m3 with the
    library's round-to-nearest-even cast; all-zero tiles give scale 0 and zero
    bytes.  Pinned bit-exact to ``quantize_tokens`` by a CPU test.
    """
    import torch
    lat = torch.from_numpy(np.ascontiguousarray(latent_bits, dtype=np.uint16).reshape(-1, DV).view(np.int16))
    rop = np.ascontiguousarray(rope_bits, dtype=np.uint16).reshape(-1, DROPE)
    n = lat.shape[0]
    x = lat.view(torch.bfloat16).to(torch.float32).reshape(n, 4, 128)
    amax = x.abs().amax(dim=2, keepdim=True)
    scale = amax / torch.tensor(448.0, dtype=torch.float32)
    safe = torch.where(scale == 0, torch.ones_like(scale), scale)
    y = (x / safe).clamp(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    codes = torch.where(scale == 0, torch.zeros_like(codes), codes)
    out = np.empty((n, ROW_BYTES), dtype=np.uint8)
    out[:, :512] = codes.reshape(n, 512).numpy()
    out[:, 512:528] = scale.reshape(n, 4).contiguous().numpy().astype("<f4").view(np.uint8).reshape(n, 16)
    out[:, 528:] = rop.astype("<u2").view(np.uint8).reshape(n, 128)
    return out


def dequantize_row(row: np.ndarray) -> np.ndarray:
    """656 bytes -> the 576-wide key (float64; each value exactly a bf16)."""
    r = np.ascontiguousarray(row, dtype=np.uint8).reshape(ROW_BYTES)
    k = np.zeros(DQK, dtype=np.float64)
    lib().smo_dequantize_row(_ptr(r, ctypes.c_uint8), _ptr(k, ctypes.c_double))
    return k


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, valid: np.ndarray, softmax_scale: float = DEFAULT_SOFTMAX_SCALE,
           want_weights: bool = False):
    """Gathered softmax attention in float64: q [h,576], K [n,576], valid [n] -> (o [h,512], lse [h] (, w [h,n]))."""
    qd = np.ascontiguousarray(q, dtype=np.float64)
    Kd = np.ascontiguousarray(K, dtype=np.float64).reshape(-1, DQK)
    v = np.ascontiguousarray(valid, dtype=np.uint8).reshape(-1)
    h, n = qd.shape[0], Kd.shape[0]
    o = np.zeros((h, DV), dtype=np.float64)
    lse = np.zeros(h, dtype=np.float64)
    w = np.zeros((h, max(n, 1)), dtype=np.float64) if want_weights else None
    lib().smo_attend(h, _ptr(qd, ctypes.c_double), n, _ptr(Kd, ctypes.c_double) if n else None,
                     _ptr(v, ctypes.c_uint8) if n else None, float(softmax_scale),
                     _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                     _ptr(w, ctypes.c_double) if want_weights else None)
    if want_weights:
        return o, lse, w[:, :n]
    return o, lse


def combine(o_parts: np.ndarray, lse_parts: np.ndarray):
    """LSE-weighted combine: o_parts [S,h,512], lse_parts [S,h] -> (o [h,512], lse [h])."""
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    s, h = lp.shape
    o = np.zeros((h, DV), dtype=np.float64)
    lse = np.zeros(h, dtype=np.float64)
    lib().smo_combine(s, h, _ptr(op, ctypes.c_double), _ptr(lp, ctypes.c_double),
                      _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    return o, lse


def sparse_decode_token(q_bits: np.ndarray, kvcache: np.ndarray, block_table_row: np.ndarray, seqlen: int,
                        idx: np.ndarray, softmax_scale: float = DEFAULT_SOFTMAX_SCALE):
    """One query token: q_bits [h,576] bf16 bits, kvcache [num_blocks,64,656] uint8 -> (o [h,512], lse [h])."""
    qb = np.ascontiguousarray(q_bits, dtype=np.uint16)
    h = qb.shape[0]
    cache = kvcache if kvcache.flags["C_CONTIGUOUS"] else np.ascontiguousarray(kvcache)
    num_blocks = cache.size // (BLOCK * ROW_BYTES)
    bt = np.ascontiguousarray(block_table_row, dtype=np.int32)
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    o = np.zeros((h, DV), dtype=np.float64)
    lse = np.zeros(h, dtype=np.float64)
    rc = lib().smo_sparse_decode_token(h, _ptr(qb, ctypes.c_uint16), _ptr(cache.reshape(-1), ctypes.c_uint8),
                                       num_blocks, _ptr(bt, ctypes.c_int32), bt.shape[0], int(seqlen),
                                       _ptr(ix, ctypes.c_int32), ix.shape[0], float(softmax_scale),
                                       _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle: a valid index maps outside the block table or the cache")
    return o, lse


def sparse_decode(q_bits: np.ndarray, kvcache: np.ndarray, block_table: np.ndarray, cache_seqlens: np.ndarray,
                  indices: np.ndarray, softmax_scale: float = DEFAULT_SOFTMAX_SCALE, tokens=None,
                  threads: int = 1):
    """Reference outputs for query tokens of a batch.

    q_bits [b,s_q,h,576] (bf16 bits), indices [b,s_q,topk].  ``tokens`` is an
    optional list of (b, t) pairs (default: all).  Returns dict (b,t) -> (o, lse).
    Each token is computed single-threaded; ``threads`` > 1 fans tokens out
    over host threads (the C call releases the GIL).
    """
    b, s_q = indices.shape[0], indices.shape[1]
    if tokens is None:
        tokens = [(i, t) for i in range(b) for t in range(s_q)]
    cache = np.ascontiguousarray(kvcache)

    def one(bt):
        i, t = bt
        return bt, sparse_decode_token(q_bits[i, t], cache, block_table[i], int(cache_seqlens[i]),
                                       indices[i, t], softmax_scale)

    if threads <= 1:
        return dict(one(x) for x in tokens)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return dict(ex.map(one, tokens))


def sparse_prefill(q_bits: np.ndarray, kv_rows: np.ndarray, indices: np.ndarray,
                   softmax_scale: float = DEFAULT_SOFTMAX_SCALE, tokens=None):
    """Sparse attention of s_q query tokens over one flat FP8 cache.

    Follows "deepseek-ai/FlashMLA" (agentlenshq), section 使用方法 item 2
    (flash_mla_sparse_fwd(q, kv, indices, ...) with 3-D indices naming, per
    query token, the KV tokens it attends to) and 技術的な詳細 (-1 = ignored):
    token t attends to the rows kv_rows[i] of its indices with 0 <= i < s_kv,
    each row taken through the same dequantisation and attention as the
    sparse decode.  A flat cache is a paged one whose block table is the
    identity, so this calls ``sparse_decode_token`` with that table; the rows
    that pad the cache to whole 64-row blocks are never read.

    q_bits [s_q, h, 576] bf16 bits; kv_rows [s_kv, 656] uint8; indices
    [s_q, 1, topk] or [s_q, topk] int32.  Returns dict t -> (o [h, 512], lse [h]).
    """
    s_kv = kv_rows.shape[0]
    nb = (s_kv + BLOCK - 1) // BLOCK
    cache = np.zeros((nb * BLOCK, ROW_BYTES), dtype=np.uint8)
    cache[:s_kv] = kv_rows.reshape(s_kv, ROW_BYTES)
    cache = cache.reshape(nb, BLOCK, ROW_BYTES)
    table = np.arange(nb, dtype=np.int32)
    idx = indices.reshape(indices.shape[0], -1)
    if tokens is None:
        tokens = range(idx.shape[0])
    return {t: sparse_decode_token(q_bits[t], cache, table, s_kv, idx[t], softmax_scale) for t in tokens}


# --------------------------------------------------------------------------
# dense decode (every visible token; FP8 or BF16 cache rows)
# --------------------------------------------------------------------------

BF16_ROW_BYTES = 1152
KV_FP8, KV_BF16 = 0, 1


def bf16_row(row: np.ndarray) -> np.ndarray:
    """A 1152-byte BF16 cache row -> the 576-wide key in float64."""
    r = np.ascontiguousarray(row, dtype=np.uint8).reshape(-1)
    assert r.size == BF16_ROW_BYTES
    k = np.zeros(DQK, dtype=np.float64)
    lib().smo_bf16_row(_ptr(r, ctypes.c_uint8), _ptr(k, ctypes.c_double))
    return k


def dense_visible_len(seqlen: int, s_q: int, t: int, causal: bool) -> int:
    return int(lib().smo_dense_visible_len(int(seqlen), int(s_q), int(t), 1 if causal else 0))


def dense_decode_token(q_bits: np.ndarray, kvcache: np.ndarray, kv_format: int, block_table_row: np.ndarray,
                       length: int, softmax_scale: float = DEFAULT_SOFTMAX_SCALE):
    """One query token over cache positions 0..length-1: kvcache [num_blocks,64,row] uint8 with
    row = 656 (kv_format KV_FP8) or 1152 (KV_BF16) -> (o [h,512], lse [h])."""
    qb = np.ascontiguousarray(q_bits, dtype=np.uint16)
    h = qb.shape[0]
    row = BF16_ROW_BYTES if kv_format == KV_BF16 else ROW_BYTES
    cache = kvcache if kvcache.flags["C_CONTIGUOUS"] else np.ascontiguousarray(kvcache)
    num_blocks = cache.size // (BLOCK * row)
    bt = np.ascontiguousarray(block_table_row, dtype=np.int32)
    o = np.zeros((h, DV), dtype=np.float64)
    lse = np.zeros(h, dtype=np.float64)
    rc = lib().smo_dense_decode_token(h, _ptr(qb, ctypes.c_uint16), _ptr(cache.reshape(-1), ctypes.c_uint8),
                                      int(kv_format), num_blocks, _ptr(bt, ctypes.c_int32), bt.shape[0], int(length),
                                      float(softmax_scale), _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle: a position maps outside the block table or the cache")
    return o, lse


def dense_decode(q_bits: np.ndarray, kvcache: np.ndarray, kv_format: int, block_table: np.ndarray,
                 cache_seqlens: np.ndarray, causal: bool, softmax_scale: float = DEFAULT_SOFTMAX_SCALE,
                 tokens=None, threads: int = 1):
    """Dense decode of a batch: q_bits [b,s_q,h,576] -> dict (b,t) -> (o, lse); each token single-threaded,
    ``threads`` > 1 fans tokens out over host threads."""
    b, s_q = q_bits.shape[0], q_bits.shape[1]
    if tokens is None:
        tokens = [(i, t) for i in range(b) for t in range(s_q)]
    cache = np.ascontiguousarray(kvcache)

    def one(bt_):
        i, t = bt_
        n = dense_visible_len(int(cache_seqlens[i]), s_q, t, causal)
        return bt_, dense_decode_token(q_bits[i, t], cache, kv_format, block_table[i], n, softmax_scale)

    if threads <= 1:
        return dict(one(x) for x in tokens)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return dict(ex.map(one, tokens))


# --------------------------------------------------------------------------
# scheduler metadata
# --------------------------------------------------------------------------

def sched_meta(R: int, n: int, P: int):
    """Closed-form tile-scheduler metadata -> (sched_meta [P,8] int32, num_splits [R+1] int32)."""
    sm = np.zeros((P, 8), dtype=np.int32)
    ns = np.zeros(R + 1, dtype=np.int32)
    rc = lib().smo_sched_meta(R, n, P, _ptr(sm, ctypes.c_int32), _ptr(ns, ctypes.c_int32))
    if rc != 0:
        raise ValueError("oracle.sched_meta: invalid arguments")
    return sm, ns


def sched_meta_varlen(n_tiles: np.ndarray, P: int):
    """Scheduler metadata for per-request tile counts -> (sched_meta [P,8], num_splits [R+1], tile_prefix [R+1])."""
    n = np.ascontiguousarray(n_tiles, dtype=np.int32)
    R = n.shape[0]
    sm = np.zeros((P, 8), dtype=np.int32)
    ns = np.zeros(R + 1, dtype=np.int32)
    tp = np.zeros(R + 1, dtype=np.int32)
    rc = lib().smo_sched_meta_varlen(R, _ptr(n, ctypes.c_int32), P, _ptr(sm, ctypes.c_int32), _ptr(ns, ctypes.c_int32),
                                     _ptr(tp, ctypes.c_int32))
    if rc != 0:
        raise ValueError("oracle.sched_meta_varlen: invalid arguments")
    return sm, ns, tp


def dense_tile_counts(cache_seqlens: np.ndarray, s_q: int, causal: bool) -> np.ndarray:
    """Per request r = b * s_q + t of a dense decode: max(1, ceil(visible tokens / 64))."""
    out = []
    for sl in np.asarray(cache_seqlens):
        for t in range(s_q):
            n = dense_visible_len(int(sl), s_q, t, causal)
            out.append(max(1, (n + BLOCK - 1) // BLOCK))
    return np.asarray(out, dtype=np.int32)

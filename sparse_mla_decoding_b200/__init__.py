"""B200-native token-level sparse MLA decoding over a paged FP8 KV cache.

Thin Python binding of ``libsmla.so`` (C ABI in ``include/smla.h``): it only
checks shapes, allocates outputs with torch and passes raw device pointers and
the current CUDA stream through ctypes.  Every step of the computation runs in
the library's sm_100a kernels; there is no CPU or PyTorch fallback, and a
missing or unbuildable library raises.

    sched_meta, num_splits = get_mla_metadata(cache_seqlens, topk, h_q, s_q=s_q)
    for layer in layers:                    # the schedule is reused across layers
        o, lse = flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens,
                                        indices, sched_meta, num_splits)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Tuple

import torch

from . import build as _build

D_QK, D_V, D_ROPE, KV_ROW_BYTES, BLOCK_SIZE, INDEX_TILE = 576, 512, 64, 656, 64, 64
STATUS_NAMES = {0: "SMLA_OK", 1: "SMLA_ERR_INVALID_ARGUMENT", 2: "SMLA_ERR_UNSUPPORTED", 3: "SMLA_ERR_CUDA",
                4: "SMLA_ERR_DEVICE_TIMEOUT", 5: "SMLA_ERR_SCRATCH_LIMIT"}
# Raw flag bits of the device status word (kernel side, sticky until reset).
STATUS_FLAGS = {1: "a bounded device wait gave up", 2: "a valid index mapped outside the block table or the cache",
                4: "scheduler metadata inconsistent with the call's shapes"}

_lib = None
_lib_lock = threading.Lock()


class SmlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libsmla.so (building it with nvcc first if it is missing or stale)."""
    global _lib
    with _lib_lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
            L.smla_status_string.argtypes = [i32]
            L.smla_status_string.restype = ctypes.c_char_p
            L.smla_version.argtypes = []
            L.smla_version.restype = i32
            L.smla_last_cuda_error.argtypes = []
            L.smla_last_cuda_error.restype = i32
            L.smla_last_cuda_error_string.argtypes = []
            L.smla_last_cuda_error_string.restype = ctypes.c_char_p
            L.smla_set_head_pair_form.argtypes = [i32]
            L.smla_set_head_pair_form.restype = i32
            L.smla_default_num_sm_parts.argtypes = [i32, i32]
            L.smla_default_num_sm_parts.restype = i32
            L.smla_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
            L.smla_workspace_bytes.restype = sz
            L.smla_get_mla_metadata.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp]
            L.smla_get_mla_metadata.restype = i32
            L.smla_flash_mla_with_kvcache.argtypes = [vp, vp, i64, vp, i32, vp, vp, vp, vp, i32, f32, i32, i32, i32,
                                                      i32, vp, vp, vp, sz, vp]
            L.smla_flash_mla_with_kvcache.restype = i32
            L.smla_get_mla_metadata_dense.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
            L.smla_get_mla_metadata_dense.restype = i32
            L.smla_flash_mla_dense_with_kvcache.argtypes = [vp, vp, i32, i64, vp, i32, vp, vp, vp, vp, i32, f32, i32,
                                                            i32, i32, i32, vp, vp, vp, sz, vp]
            L.smla_flash_mla_dense_with_kvcache.restype = i32
            L.smla_flash_mla_sparse_fwd.argtypes = [vp, vp, i64, vp, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
            L.smla_flash_mla_sparse_fwd.restype = i32
            L.smla_sparse_fwd_workspace_bytes.argtypes = [i32, i32, i64, i32, i32]
            L.smla_sparse_fwd_workspace_bytes.restype = sz
            L.smla_quantize_kv.argtypes = [vp, vp, i64, vp, vp, i64, vp]
            L.smla_quantize_kv.restype = i32
            L.smla_get_device_status.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_uint32), vp]
            L.smla_get_device_status.restype = i32
            L.smla_reset_device_status.argtypes = [vp, vp]
            L.smla_reset_device_status.restype = i32
            L.smla_selftest_bounded_wait.argtypes = [vp, ctypes.c_uint64, vp]
            L.smla_selftest_bounded_wait.restype = i32
            _lib = L
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != 0:
        if rc == 3:   # SMLA_ERR_CUDA: name the CUDA runtime error behind it
            what = f"{what} ({lib().smla_last_cuda_error_string().decode()})"
        raise SmlaError(rc, what)


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def set_head_pair_form(enable: bool) -> bool:
    """Run 128-head decodes as two-CTA clusters that share dequantised tiles
    (True) or as independent CTAs (False, the default); returns the previous
    setting.  Process-wide; results are bitwise identical either way."""
    return bool(lib().smla_set_head_pair_form(1 if enable else 0))


def default_num_sm_parts(h_q: int, device: Optional[torch.device] = None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    n = lib().smla_default_num_sm_parts(h_q, dev.index if dev.index is not None else torch.cuda.current_device())
    if n < 1:
        raise SmlaError(3, "smla_default_num_sm_parts")
    return n


def workspace_bytes(batch: int, s_q: int, h_q: int, topk: int, num_sm_parts: int) -> int:
    n = lib().smla_workspace_bytes(batch, s_q, h_q, topk, num_sm_parts)
    if n == 0:
        raise SmlaError(1, "smla_workspace_bytes")
    return int(n)


def new_workspace(batch: int, s_q: int, h_q: int, topk: int, num_sm_parts: int,
                  device: Optional[torch.device] = None) -> torch.Tensor:
    """A zeroed workspace buffer (the zeroed header is the device status word)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.zeros(workspace_bytes(batch, s_q, h_q, topk, num_sm_parts), dtype=torch.uint8, device=dev)


_ws_cache: dict = {}
_ws_lock = threading.Lock()


def _ws_key(device: torch.device):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    return idx, torch.cuda.current_stream(idx).cuda_stream


def _cached_workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """The workspace used when a call passes none: one per (device, current stream).

    When a call needs more room, the buffer is replaced by a larger one and the
    old status header (the sticky device status word) is carried over on the
    stream, so flags raised by earlier calls are not lost.
    """
    key = _ws_key(device)
    with _ws_lock:
        ws = _ws_cache.get(key)
        if ws is None or ws.numel() < nbytes:
            new = torch.zeros(nbytes, dtype=torch.uint8, device=device)
            if ws is not None:
                new[:256].copy_(ws[:256])
            ws = new
            _ws_cache[key] = ws
    return ws


def cached_workspace_status(device: Optional[torch.device] = None) -> Tuple[int, int]:
    """(status, raw flags) of the device status word of the workspace that calls
    without a `workspace` argument share on `device` and the current stream.

    Kernels record skipped bad block-table entries, inconsistent scheduler
    metadata and bounded waits that gave up there; the flags stay set until
    reset_cached_workspace_status.  Synchronises the current stream.
    (0, 0) if no such call has run yet.
    """
    with _ws_lock:
        ws = _ws_cache.get(_ws_key(device))
    if ws is None:
        return 0, 0
    return get_device_status(ws)


def reset_cached_workspace_status(device: Optional[torch.device] = None) -> None:
    """Clear the status word of the shared workspace on `device` and the current stream."""
    with _ws_lock:
        ws = _ws_cache.get(_ws_key(device))
    if ws is not None:
        reset_device_status(ws)


def _raise_on_flags(workspace: torch.Tensor, what: str) -> None:
    st, raw = get_device_status(workspace)
    if st != 0:
        why = "; ".join(v for k, v in STATUS_FLAGS.items() if raw & k) or f"flags {raw:#x}"
        raise SmlaError(st, f"{what} (device status: {why})")


def get_mla_metadata(cache_seqlens: torch.Tensor, topk: int, h_q: int, num_sm_parts: Optional[int] = None,
                     s_q: int = 1) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tile-scheduler metadata for batch = len(cache_seqlens) requests of s_q query tokens.

    Returns (sched_meta int32 [num_sm_parts, 8], num_splits int32 [batch*s_q + 1]).
    """
    _require(cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32 and cache_seqlens.dim() == 1,
             "cache_seqlens must be a 1-D int32 CUDA tensor")
    dev = cache_seqlens.device
    if num_sm_parts is None:
        num_sm_parts = default_num_sm_parts(h_q, dev)
    batch = cache_seqlens.shape[0]
    sched_meta = torch.empty((num_sm_parts, 8), dtype=torch.int32, device=dev)
    num_splits = torch.empty((batch * s_q + 1,), dtype=torch.int32, device=dev)
    rc = lib().smla_get_mla_metadata(_ptr(cache_seqlens.contiguous()), batch, s_q, int(topk), int(h_q),
                                     int(num_sm_parts), _ptr(sched_meta), _ptr(num_splits), _stream(dev))
    _check(rc, "smla_get_mla_metadata")
    return sched_meta, num_splits


def flash_mla_with_kvcache(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, indices: torch.Tensor, sched_meta: torch.Tensor,
                           num_splits: torch.Tensor, softmax_scale: Optional[float] = None,
                           workspace: Optional[torch.Tensor] = None,
                           out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                           check_device_status: bool = False
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sparse MLA decode: returns (o bf16 [b, s_q, h_q, 512], lse float32 [b, s_q, h_q]).

    q: bf16 [b, s_q, h_q, 576]; kvcache: uint8 [num_blocks, 64, (1,) 656];
    block_table: int32 [b, max_blocks]; cache_seqlens: int32 [b];
    indices: int32 [b, s_q, topk] (negative or >= seqlen = skip);
    sched_meta / num_splits from get_mla_metadata with the same shapes.
    Device-side problems (a valid index whose block lies outside the block
    table or the cache, inconsistent metadata, a wait that gave up) set flags
    in the workspace's status word: read them with get_device_status(workspace),
    or with cached_workspace_status() when no workspace was passed.
    check_device_status=True synchronises after the call and raises SmlaError
    if any flag is set.
    """
    _require(q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.shape[-1] == D_QK,
             "q must be a bf16 CUDA tensor [b, s_q, h_q, 576]")
    b, s_q, h_q, _ = q.shape
    _require(kvcache.dtype == torch.uint8 and kvcache.shape[-1] == KV_ROW_BYTES and kvcache.shape[1] == BLOCK_SIZE,
             "kvcache must be uint8 [num_blocks, 64, (1,) 656]")
    _require(indices.dtype == torch.int32 and indices.dim() == 3 and tuple(indices.shape[:2]) == (b, s_q),
             "indices must be int32 [b, s_q, topk]")
    _require(block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == b,
             "block_table must be int32 [b, max_blocks]")
    _require(cache_seqlens.dtype == torch.int32 and tuple(cache_seqlens.shape) == (b,),
             "cache_seqlens must be int32 [b]")
    _require(sched_meta.dtype == torch.int32 and sched_meta.dim() == 2 and sched_meta.shape[1] == 8,
             "sched_meta must be int32 [num_sm_parts, 8]")
    _require(num_splits.dtype == torch.int32 and tuple(num_splits.shape) == (b * s_q + 1,),
             "num_splits must be int32 [b*s_q + 1]")
    for name, t in (("kvcache", kvcache), ("block_table", block_table), ("cache_seqlens", cache_seqlens),
                    ("indices", indices), ("sched_meta", sched_meta), ("num_splits", num_splits)):
        _require(t.is_cuda and t.device == q.device, f"{name} must be on {q.device}")
        _require(t.is_contiguous(), f"{name} must be contiguous")
    q = q.contiguous()
    topk = indices.shape[2]
    num_sm_parts = sched_meta.shape[0]
    dev = q.device
    nbytes = workspace_bytes(b, s_q, h_q, topk, num_sm_parts)
    if workspace is None:
        workspace = _cached_workspace(dev, nbytes)
    _require(workspace.is_cuda and workspace.numel() * workspace.element_size() >= nbytes,
             f"workspace needs {nbytes} bytes")
    if out is None:
        o = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((b, s_q, h_q), dtype=torch.float32, device=dev)
    else:
        o, lse = out
    scale = -1.0 if softmax_scale is None else float(softmax_scale)
    rc = lib().smla_flash_mla_with_kvcache(
        _ptr(q), _ptr(kvcache), kvcache.shape[0], _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
        _ptr(indices), _ptr(sched_meta), _ptr(num_splits), num_sm_parts, scale, b, s_q, h_q, topk, _ptr(o),
        _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check(rc, "smla_flash_mla_with_kvcache")
    if check_device_status:
        _raise_on_flags(workspace, "smla_flash_mla_with_kvcache")
    return o, lse


KV_FP8, KV_BF16 = 0, 1
BF16_ROW_BYTES = 1152


def get_mla_metadata_dense(cache_seqlens: torch.Tensor, h_q: int, s_q: int = 1, causal: bool = True,
                           num_sm_parts: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Scheduler metadata of a dense decode, split by the requests' visible lengths.

    Returns (sched_meta int32 [num_sm_parts, 8], num_splits int32 [b*s_q + 1],
    tile_prefix int32 [b*s_q + 1]); reusable across layers while the lengths stay.
    """
    _require(cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32 and cache_seqlens.dim() == 1,
             "cache_seqlens must be a 1-D int32 CUDA tensor")
    dev = cache_seqlens.device
    if num_sm_parts is None:
        num_sm_parts = default_num_sm_parts(h_q, dev)
    R = cache_seqlens.shape[0] * s_q
    sched_meta = torch.empty((num_sm_parts, 8), dtype=torch.int32, device=dev)
    num_splits = torch.empty((R + 1,), dtype=torch.int32, device=dev)
    tile_prefix = torch.empty((R + 1,), dtype=torch.int32, device=dev)
    rc = lib().smla_get_mla_metadata_dense(_ptr(cache_seqlens.contiguous()), cache_seqlens.shape[0], int(s_q), int(h_q),
                                           1 if causal else 0, int(num_sm_parts), _ptr(sched_meta), _ptr(num_splits),
                                           _ptr(tile_prefix), _stream(dev))
    _check(rc, "smla_get_mla_metadata_dense")
    return sched_meta, num_splits, tile_prefix


def _kv_format(kvcache: torch.Tensor) -> int:
    if kvcache.dtype == torch.uint8 and kvcache.shape[-1] == KV_ROW_BYTES:
        return KV_FP8
    if kvcache.dtype == torch.uint8 and kvcache.shape[-1] == BF16_ROW_BYTES:
        return KV_BF16
    if kvcache.dtype == torch.bfloat16 and kvcache.shape[-1] == D_QK:
        return KV_BF16
    raise ValueError("kvcache must be uint8 [..., 656] (FP8 rows), or bf16 [..., 576] / uint8 [..., 1152] (BF16 rows)")


def flash_mla_dense_with_kvcache(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                                 cache_seqlens: torch.Tensor, sched_meta: torch.Tensor, num_splits: torch.Tensor,
                                 tile_prefix: torch.Tensor, causal: bool = True,
                                 softmax_scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                                 out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                                 check_device_status: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Dense MLA decode: every query token attends to all its visible cache tokens.

    q: bf16 [b, s_q, h_q, 576]; kvcache: paged [num_blocks, 64, (1,) row] with FP8
    rows (uint8, 656 bytes) or BF16 rows (bf16 576 values, or uint8 1152 bytes);
    block_table: int32 [b, max_blocks]; cache_seqlens: int32 [b]; sched_meta /
    num_splits / tile_prefix from get_mla_metadata_dense with the same lengths,
    s_q and causal.  With causal=True token t of s_q sees the first
    seqlen - (s_q - 1 - t) cache positions.  Returns (o bf16 [b, s_q, h_q, 512],
    lse float32 [b, s_q, h_q]).
    """
    _require(q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.shape[-1] == D_QK,
             "q must be a bf16 CUDA tensor [b, s_q, h_q, 576]")
    b, s_q, h_q, _ = q.shape
    fmt = _kv_format(kvcache)
    _require(kvcache.shape[1] == BLOCK_SIZE and kvcache.is_contiguous(), "kvcache must be contiguous [num_blocks, 64, ...]")
    _require(block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == b,
             "block_table must be int32 [b, max_blocks]")
    _require(cache_seqlens.dtype == torch.int32 and tuple(cache_seqlens.shape) == (b,),
             "cache_seqlens must be int32 [b]")
    _require(sched_meta.dtype == torch.int32 and sched_meta.dim() == 2 and sched_meta.shape[1] == 8,
             "sched_meta must be int32 [num_sm_parts, 8]")
    for name, t in (("num_splits", num_splits), ("tile_prefix", tile_prefix)):
        _require(t.dtype == torch.int32 and tuple(t.shape) == (b * s_q + 1,), f"{name} must be int32 [b*s_q + 1]")
    for name, t in (("kvcache", kvcache), ("block_table", block_table), ("cache_seqlens", cache_seqlens),
                    ("sched_meta", sched_meta), ("num_splits", num_splits), ("tile_prefix", tile_prefix)):
        _require(t.is_cuda and t.device == q.device, f"{name} must be on {q.device}")
        _require(t.is_contiguous(), f"{name} must be contiguous")
    q = q.contiguous()
    num_sm_parts = sched_meta.shape[0]
    dev = q.device
    nbytes = workspace_bytes(b, s_q, h_q, 1, num_sm_parts)
    if workspace is None:
        workspace = _cached_workspace(dev, nbytes)
    _require(workspace.is_cuda and workspace.numel() * workspace.element_size() >= nbytes,
             f"workspace needs {nbytes} bytes")
    if out is None:
        o = torch.empty((b, s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((b, s_q, h_q), dtype=torch.float32, device=dev)
    else:
        o, lse = out
    scale = -1.0 if softmax_scale is None else float(softmax_scale)
    rc = lib().smla_flash_mla_dense_with_kvcache(
        _ptr(q), _ptr(kvcache), fmt, kvcache.shape[0], _ptr(block_table), block_table.shape[1], _ptr(cache_seqlens),
        _ptr(sched_meta), _ptr(num_splits), _ptr(tile_prefix), num_sm_parts, scale, 1 if causal else 0, b, s_q, h_q,
        _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check(rc, "smla_flash_mla_dense_with_kvcache")
    if check_device_status:
        _raise_on_flags(workspace, "smla_flash_mla_dense_with_kvcache")
    return o, lse


def sparse_fwd_workspace_bytes(s_q: int, h_q: int, s_kv: int, topk: int, num_sm_parts: int) -> int:
    n = lib().smla_sparse_fwd_workspace_bytes(s_q, h_q, s_kv, topk, num_sm_parts)
    if n == 0:
        raise SmlaError(1, "smla_sparse_fwd_workspace_bytes")
    return int(n)


def flash_mla_sparse_fwd(q: torch.Tensor, kv: torch.Tensor, indices: torch.Tensor,
                         softmax_scale: Optional[float] = None, num_sm_parts: Optional[int] = None,
                         workspace: Optional[torch.Tensor] = None,
                         out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                         check_device_status: bool = False
                         ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sparse attention of s_q query tokens over one flat FP8 cache: (o bf16 [s_q, h_q, 512], lse [s_q, h_q]).

    q: bf16 [s_q, h_q, 576]; kv: uint8 [s_kv, (1,) 656] (656-byte rows, one KV head);
    indices: int32 [s_q, 1, topk] (or [s_q, topk]), negative or >= s_kv = skip.
    A workspace from new_sparse_fwd_workspace may be passed; its first 256 bytes are
    the device status word (get_device_status).
    """
    _require(q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 3 and q.shape[-1] == D_QK,
             "q must be a bf16 CUDA tensor [s_q, h_q, 576]")
    s_q, h_q, _ = q.shape
    _require(kv.dtype == torch.uint8 and kv.shape[-1] == KV_ROW_BYTES and kv.dim() in (2, 3) and
             (kv.dim() == 2 or kv.shape[1] == 1), "kv must be uint8 [s_kv, (1,) 656]")
    _require(indices.dtype == torch.int32 and indices.shape[0] == s_q and
             (indices.dim() == 2 or (indices.dim() == 3 and indices.shape[1] == 1)),
             "indices must be int32 [s_q, 1, topk] or [s_q, topk]")
    for name, t in (("kv", kv), ("indices", indices)):
        _require(t.is_cuda and t.device == q.device, f"{name} must be on {q.device}")
        _require(t.is_contiguous(), f"{name} must be contiguous")
    q = q.contiguous()
    s_kv = kv.shape[0]
    topk = indices.shape[-1]
    dev = q.device
    if num_sm_parts is None:
        num_sm_parts = default_num_sm_parts(h_q, dev)
    nbytes = sparse_fwd_workspace_bytes(s_q, h_q, s_kv, topk, num_sm_parts)
    if workspace is None:
        workspace = _cached_workspace(dev, nbytes)
    _require(workspace.is_cuda and workspace.numel() * workspace.element_size() >= nbytes,
             f"workspace needs {nbytes} bytes")
    if out is None:
        o = torch.empty((s_q, h_q, D_V), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((s_q, h_q), dtype=torch.float32, device=dev)
    else:
        o, lse = out
    scale = -1.0 if softmax_scale is None else float(softmax_scale)
    rc = lib().smla_flash_mla_sparse_fwd(_ptr(q), _ptr(kv), s_kv, _ptr(indices), s_q, h_q, topk, int(num_sm_parts),
                                         scale, _ptr(o), _ptr(lse), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(dev))
    _check(rc, "smla_flash_mla_sparse_fwd")
    if check_device_status:
        _raise_on_flags(workspace, "smla_flash_mla_sparse_fwd")
    return o, lse


def new_sparse_fwd_workspace(s_q: int, h_q: int, s_kv: int, topk: int, num_sm_parts: int,
                             device: Optional[torch.device] = None) -> torch.Tensor:
    """A zeroed workspace for flash_mla_sparse_fwd (the zeroed header is the device status word)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.zeros(sparse_fwd_workspace_bytes(s_q, h_q, s_kv, topk, num_sm_parts), dtype=torch.uint8,
                       device=dev)


def quantize_kv(latent: torch.Tensor, rope: torch.Tensor, kvcache: torch.Tensor,
                slot_mapping: Optional[torch.Tensor] = None) -> None:
    """Write tokens (bf16 latent [n, 512] and rope [n, 64]) into 656-byte FP8 rows of kvcache."""
    _require(latent.is_cuda and latent.dtype == torch.bfloat16 and latent.dim() == 2 and latent.shape[1] == D_V,
             "latent must be bf16 [n, 512] on CUDA")
    _require(rope.dtype == torch.bfloat16 and tuple(rope.shape) == (latent.shape[0], D_ROPE),
             "rope must be bf16 [n, 64]")
    _require(kvcache.dtype == torch.uint8 and kvcache.shape[-1] == KV_ROW_BYTES and kvcache.is_contiguous(),
             "kvcache must be contiguous uint8 [..., 656]")
    if slot_mapping is not None:
        _require(slot_mapping.dtype == torch.int64 and tuple(slot_mapping.shape) == (latent.shape[0],),
                 "slot_mapping must be int64 [n]")
        slot_mapping = slot_mapping.contiguous()
    latent, rope = latent.contiguous(), rope.contiguous()
    num_rows = kvcache.numel() // KV_ROW_BYTES
    rc = lib().smla_quantize_kv(_ptr(latent), _ptr(rope), latent.shape[0], _ptr(slot_mapping), _ptr(kvcache),
                                num_rows, _stream(latent.device))
    _check(rc, "smla_quantize_kv")


def get_device_status(workspace: torch.Tensor) -> Tuple[int, int]:
    """(status, raw flags) of a workspace's sticky status word; synchronises the current stream."""
    st = ctypes.c_int(0)
    raw = ctypes.c_uint32(0)
    rc = lib().smla_get_device_status(_ptr(workspace), ctypes.byref(st), ctypes.byref(raw), _stream(workspace.device))
    _check(rc, "smla_get_device_status")
    return st.value, raw.value


def reset_device_status(workspace: torch.Tensor) -> None:
    _check(lib().smla_reset_device_status(_ptr(workspace), _stream(workspace.device)), "smla_reset_device_status")


def selftest_bounded_wait(workspace: torch.Tensor, limit_ns: int) -> None:
    _check(lib().smla_selftest_bounded_wait(_ptr(workspace), int(limit_ns), _stream(workspace.device)),
           "smla_selftest_bounded_wait")


def default_softmax_scale() -> float:
    return 1.0 / math.sqrt(D_QK)

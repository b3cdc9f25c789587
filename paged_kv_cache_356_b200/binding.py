"""Thin Python binding of include/pa.h: the same names, argument marshalling only.

Device entry points take CUDA torch tensors (PyTorch only provides the device
memory and the stream) and enqueue the library's kernels on the current
stream; every step of the computation runs in libpa_b200.so.  CPU tensors
are rejected; there is no fallback path.  Allocator entry points take and
return host numpy arrays.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import numpy as np

from . import _lib
from ._lib import (PA_BF16, PA_DECODE_AUTO, PA_DECODE_CUDA_CORES, PA_DECODE_TENSOR_CORES,  # noqa: F401
                   PA_DEV_TIMEOUT, PA_SHARED_PREFIX_AUTO, PA_SHARED_PREFIX_MMA_SYNC, PA_SHARED_PREFIX_TCGEN05,
                   PA_SHARED_PREFIX_TCGEN05_SERIAL, PA_SHARED_PREFIX_TCGEN05_2CTA,
                   PA_SHARED_PREFIX_TCGEN05_ITEMS, PA_FAULT_NONE,
                   PA_FAULT_WITHHOLD_FIRST_ITEM, PA_VERIFY_AUTO, PA_VERIFY_JOINT, PA_VERIFY_PER_SEQUENCE,
                   PA_DEV_BAD_CTX, PA_DEV_BAD_PAGE, PA_DEV_BAD_PAIR, PA_DEV_BAD_PLAN, PA_DEV_BAD_SLOT, PA_ERR_NOT_FOUND,
                   PA_DEV_BAD_UPDATE,
                   PA_ERR_OOM, PA_F16, PA_F32, PA_PARTITION_TOKENS)


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[pa status {status}] {message}")
        self.status = status


class PagedAttentionOOM(PagedAttentionError, MemoryError):
    """The free-page pool cannot satisfy the request (state unchanged)."""


class SequenceNotFound(PagedAttentionError, KeyError):
    pass


def _check(status: int) -> None:
    if status == 0:
        return
    msg = _lib.last_error()
    if status == _lib.PA_ERR_OOM:
        raise PagedAttentionOOM(status, msg)
    if status == _lib.PA_ERR_NOT_FOUND:
        raise SequenceNotFound(status, msg)
    raise PagedAttentionError(status, msg)


def _torch():
    import torch
    return torch


def dtype_code(dtype) -> int:
    torch = _torch()
    codes = {torch.float32: PA_F32, torch.bfloat16: PA_BF16, torch.float16: PA_F16}
    if dtype not in codes:
        raise TypeError(f"unsupported dtype {dtype}")
    return codes[dtype]


def _cuda(t, name, dtype=None, contiguous=True):
    if not hasattr(t, "is_cuda") or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _opt_status(dev_status):
    if dev_status is None:
        return None
    torch = _torch()
    return _cuda(dev_status, "dev_status", torch.int32)


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _cache_shape(key_cache, value_cache):
    if key_cache.dim() != 4 or key_cache.shape != value_cache.shape or key_cache.dtype != value_cache.dtype:
        raise ValueError("caches must both be [num_blocks, num_kv_heads, block_size, head_dim] of one dtype")
    return tuple(int(x) for x in key_cache.shape)


# ---- device entry points ----------------------------------------------------------

def pa_reshape_and_cache(key, value, slot_mapping, key_cache, value_cache, dev_status=None, stream=None) -> None:
    """Store token t's K/V rows at physical slot slot_mapping[t] (negative: skip)."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if key.dim() != 3 or tuple(key.shape[1:]) != (hkv, d) or key.shape != value.shape:
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim] matching the cache")
    for name, t in (("key", key), ("value", value)):
        if t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{name}: heads and dims must be contiguous")
    t_tokens = int(key.shape[0])
    if slot_mapping.dim() != 1 or slot_mapping.shape[0] != t_tokens:
        raise ValueError("slot_mapping must be [num_tokens]")
    _check(_lib.load().pa_reshape_and_cache(
        _cuda(key, "key", key_cache.dtype, contiguous=False), _cuda(value, "value", key_cache.dtype, contiguous=False),
        key.stride(0), value.stride(0), _cuda(slot_mapping, "slot_mapping", torch.int64), t_tokens,
        _cuda(key_cache, "key_cache"), _cuda(value_cache, "value_cache"), nb, bs, hkv, d,
        dtype_code(key_cache.dtype), _opt_status(dev_status), _stream_handle(stream, key_cache.device)))


def pa_copy_blocks(key_cache, value_cache, block_mapping, dev_status=None, stream=None) -> None:
    """Copy page src onto page dst (all heads, all slots, K and V) for each row (src, dst)."""
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise ValueError("block_mapping must be [num_pairs, 2]")
    _check(_lib.load().pa_copy_blocks(
        _cuda(key_cache, "key_cache"), _cuda(value_cache, "value_cache"),
        _cuda(block_mapping, "block_mapping", torch.int64), int(block_mapping.shape[0]), nb, bs, hkv, d,
        dtype_code(key_cache.dtype), _opt_status(dev_status), _stream_handle(stream, key_cache.device)))


def pa_block_tables_apply(block_tables, updates, num_updates=None, dev_status=None, stream=None) -> None:
    """Write (row, column, page) updates (device int32 [k, 3], the first num_updates rows) into the
    device int32 [num_rows, max_blocks_per_seq] tables in place."""
    torch = _torch()
    if block_tables.dim() != 2 or block_tables.dtype != torch.int32 or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [num_rows, max_blocks_per_seq] tensor")
    if updates.dim() != 2 or updates.shape[1] != 3:
        raise ValueError("updates must be [k, 3]")
    k = int(updates.shape[0]) if num_updates is None else int(num_updates)
    if k < 0 or k > updates.shape[0]:
        raise ValueError("num_updates outside [0, updates.shape[0]]")
    _check(_lib.load().pa_block_tables_apply(
        _cuda(block_tables, "block_tables", torch.int32), int(block_tables.shape[0]), int(block_tables.shape[1]),
        _cuda(updates, "updates", torch.int32), k, _opt_status(dev_status),
        _stream_handle(stream, block_tables.device)))


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int) -> int:
    return int(_lib.load().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_context_len))


def _decode_args(q, key_cache, value_cache, block_tables, context_lens, scale, out, workspace, dev_status, stream):
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != key_cache.dtype:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim] of the cache dtype")
    num_seqs, hq = int(q.shape[0]), int(q.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != num_seqs:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq]")
    if context_lens.dim() != 1 or context_lens.shape[0] != num_seqs:
        raise ValueError("context_lens must be [num_seqs]")
    mb = int(block_tables.shape[1])
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    need = pa_decode_workspace_size(num_seqs, hq, d, mb * bs)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _cuda(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = (_cuda(q, "q"), _cuda(key_cache, "key_cache"), _cuda(value_cache, "value_cache"),
            _cuda(block_tables, "block_tables", torch.int32), mb, _cuda(context_lens, "context_lens", torch.int32),
            num_seqs, hq, hkv, d, bs, nb, float(scale), _cuda(out, "out"), dtype_code(q.dtype), ws_ptr, ws_bytes,
            _opt_status(dev_status), _stream_handle(stream, q.device))
    return args, out


def pa_decode(q, key_cache, value_cache, block_tables, context_lens, scale: float, out=None, workspace=None,
              dev_status=None, stream=None):
    """One decode step of paged attention; returns ``out`` [num_seqs, num_q_heads, head_dim].

    ``workspace`` (uint8, >= pa_decode_workspace_size bytes, 256-byte aligned)
    is allocated with torch if not given.
    """
    args, out = _decode_args(q, key_cache, value_cache, block_tables, context_lens, scale, out, workspace,
                             dev_status, stream)
    _check(_lib.load().pa_decode(*args))
    return out


def pa_decode_partitions(q, key_cache, value_cache, block_tables, context_lens, scale: float, out, workspace,
                         dev_status=None, stream=None):
    """First step of pa_decode: per-partition partials (or final rows of one-partition sequences)."""
    args, out = _decode_args(q, key_cache, value_cache, block_tables, context_lens, scale, out, workspace,
                             dev_status, stream)
    _check(_lib.load().pa_decode_partitions(*args))
    return out


def pa_decode_reduce(context_lens, max_context_len: int, out, workspace, stream=None):
    """Second step of pa_decode: log-sum-exp merge of the workspace partials into ``out``."""
    torch = _torch()
    num_seqs, hq, d = (int(x) for x in out.shape)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.load().pa_decode_reduce(
        _cuda(context_lens, "context_lens", torch.int32), num_seqs, hq, d, int(max_context_len), _cuda(out, "out"),
        dtype_code(out.dtype), _cuda(workspace, "workspace"), ws_bytes, _stream_handle(stream, out.device)))
    return out


def pa_decode_verify_workspace_size(num_seqs: int, num_query_tokens: int, num_q_heads: int, head_dim: int,
                                    max_context_len: int) -> int:
    return int(_lib.load().pa_decode_verify_workspace_size(num_seqs, num_query_tokens, num_q_heads, head_dim,
                                                           max_context_len))


def pa_decode_verify(q, key_cache, value_cache, block_tables, context_lens, scale: float, out=None, workspace=None,
                     dev_status=None, stream=None):
    """Attention of T query tokens per sequence, each over the keys up to its own position.

    ``q`` is [num_seqs, T, num_q_heads, head_dim]: the last T positions of each
    context (their K/V already in the cache).  Returns ``out`` of q's shape.
    """
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if q.dim() != 4 or q.shape[3] != d or q.dtype != key_cache.dtype:
        raise ValueError("q must be [num_seqs, num_query_tokens, num_q_heads, head_dim] of the cache dtype")
    num_seqs, nq, hq = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    if block_tables.dim() != 2 or block_tables.shape[0] != num_seqs:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq]")
    if context_lens.dim() != 1 or context_lens.shape[0] != num_seqs:
        raise ValueError("context_lens must be [num_seqs]")
    mb = int(block_tables.shape[1])
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    need = pa_decode_verify_workspace_size(num_seqs, nq, hq, d, mb * bs)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _cuda(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.load().pa_decode_verify(
        _cuda(q, "q"), _cuda(key_cache, "key_cache"), _cuda(value_cache, "value_cache"),
        _cuda(block_tables, "block_tables", torch.int32), mb, _cuda(context_lens, "context_lens", torch.int32),
        num_seqs, nq, hq, hkv, d, bs, nb, float(scale), _cuda(out, "out"), dtype_code(q.dtype), ws_ptr, ws_bytes,
        _opt_status(dev_status), _stream_handle(stream, q.device)))
    return out


def pa_decode_fixed_scratch(q, key_cache, value_cache, block_tables, context_lens, scale: float, out,
                            dev_status=None, stream=None):
    """pa_decode without a workspace argument, for callers that may not allocate device memory.

    Nothing is allocated here or in the library: ``out`` is the caller's, and
    the split-context partials use the library's fixed 32 MiB device array
    (calls needing more are rejected).  Calls that overlap on the GPU race on
    that array.  The first call on a device does a one-time set-up: make it
    before any stream capture.
    """
    torch = _torch()
    nb, hkv, bs, d = _cache_shape(key_cache, value_cache)
    if q.dim() != 3 or q.shape[2] != d or q.dtype != key_cache.dtype:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim] of the cache dtype")
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    num_seqs, hq = int(q.shape[0]), int(q.shape[1])
    if block_tables.dim() != 2 or block_tables.shape[0] != num_seqs or context_lens.shape != (num_seqs,):
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq], context_lens [num_seqs]")
    _check(_lib.load().pa_decode_fixed_scratch(
        _cuda(q, "q"), _cuda(key_cache, "key_cache"), _cuda(value_cache, "value_cache"),
        _cuda(block_tables, "block_tables", torch.int32), int(block_tables.shape[1]),
        _cuda(context_lens, "context_lens", torch.int32), num_seqs, hq, hkv, d, bs, nb, float(scale),
        _cuda(out, "out"), dtype_code(q.dtype), _opt_status(dev_status), _stream_handle(stream, q.device)))
    return out


def pa_decode_shared_prefix(q, key_cache, value_cache, block_tables, context_lens, scale: float, plan, out=None,
                            workspace=None, dev_status=None, stream=None):
    """pa_decode for a batch whose groups share leading pages; ``plan`` from prefix_plan_to_device().

    The result equals pa_decode's; shared whole partitions are read once per group.
    """
    args, out = _decode_args(q, key_cache, value_cache, block_tables, context_lens, scale, out, workspace,
                             dev_status, stream)
    torch = _torch()
    fp, ch, mem = plan["first_partition"], plan["chunks"], plan["members"]
    if fp.shape != (q.shape[0],):
        raise ValueError("plan's first_partition must have one entry per sequence")
    _check(_lib.load().pa_decode_shared_prefix(
        *args[:17], _cuda(fp, "first_partition", torch.int32), _cuda(ch, "chunks", torch.int32),
        int(plan["num_chunks"]), _cuda(mem, "members", torch.int32), int(plan["num_members"]),
        int(plan["max_shared_partitions"]), int(plan["min_shared_partitions"]), *args[17:]))
    return out


def pa_set_decode_kernel(kernel: int) -> None:
    _check(_lib.load().pa_set_decode_kernel(int(kernel)))


def pa_set_shared_prefix_kernel(kernel: int) -> None:
    _check(_lib.load().pa_set_shared_prefix_kernel(int(kernel)))


def pa_set_verify_path(path: int) -> None:
    """PA_VERIFY_AUTO, PA_VERIFY_PER_SEQUENCE or PA_VERIFY_JOINT (process-wide)."""
    _check(_lib.load().pa_set_verify_path(int(path)))


def pa_set_verify_tiling(rows_per_cta: int) -> None:
    """Rows per CTA of the per-sequence verify kernel: 8, 16, 32, or 0 for the default."""
    _check(_lib.load().pa_set_verify_tiling(int(rows_per_cta)))


def pa_set_fault_injection(mode: int) -> None:
    """Test hook for the device-side timeout path (see include/pa.h)."""
    _check(_lib.load().pa_set_fault_injection(int(mode)))


def pa_eval_exp2(x, method: int = 0, stream=None):
    """2^x on the device as the decode kernels evaluate it (method 0: FMA-pipe cubic, 1: the
    special-function unit); ``x`` a contiguous float32 CUDA tensor.  Test hook."""
    torch = _torch()
    y = torch.empty_like(x)
    _check(_lib.load().pa_eval_exp2(_cuda(x, "x", torch.float32), _cuda(y, "y", torch.float32), x.numel(),
                                    int(method), _stream_handle(stream, x.device)))
    return y


def pa_set_decode_tiling(warps: int, stages: int) -> None:
    _check(_lib.load().pa_set_decode_tiling(int(warps), int(stages)))


def pa_version() -> str:
    return _lib.load().pa_version().decode()


# ---- host allocator ---------------------------------------------------------------

def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def pa_block_alloc_create(num_blocks: int, block_size: int, initial_free_order: Optional[Sequence[int]] = None):
    order = None
    if initial_free_order is not None:
        order = np.ascontiguousarray(initial_free_order, dtype=np.int32)
        if order.shape != (num_blocks,):
            raise ValueError("initial_free_order must have num_blocks entries")
    h = ctypes.c_void_p()
    _check(_lib.load().pa_block_alloc_create(num_blocks, block_size, _i32p(order) if order is not None else None,
                                             ctypes.byref(h)))
    return h.value


def pa_block_alloc_destroy(handle) -> None:
    if handle:
        _lib.load().pa_block_alloc_destroy(handle)


def pa_block_alloc_allocate_sequence(handle, seq: int, num_tokens: int) -> None:
    _check(_lib.load().pa_block_alloc_allocate_sequence(handle, seq, num_tokens))


def pa_block_alloc_append_token(handle, seq: int) -> Tuple[int, int, int]:
    """Returns (slot, cow_src, cow_dst); cow_* are -1 when no page was forked."""
    slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.load().pa_block_alloc_append_token(handle, seq, ctypes.byref(slot), ctypes.byref(src),
                                                   ctypes.byref(dst)))
    return slot.value, src.value, dst.value


def pa_block_alloc_append_tokens(handle, seqs: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """One position for each of ``seqs`` in order, in one call: (slots int64 [n], cow pairs int32 [n, 2],
    -1 where no page was forked).  On failure raises; the appends before the failing one stand."""
    ids = np.ascontiguousarray(seqs, dtype=np.int64)
    n = len(ids)
    slots = np.empty(n, dtype=np.int64)
    src = np.empty(n, dtype=np.int32)
    dst = np.empty(n, dtype=np.int32)
    done = ctypes.c_int32()
    _check(_lib.load().pa_block_alloc_append_tokens(handle, _i64p(ids), n, _i64p(slots), _i32p(src), _i32p(dst),
                                                    ctypes.byref(done)))
    return slots, np.stack([src, dst], axis=1)


def pa_block_alloc_fork(handle, parent: int, child: int) -> None:
    _check(_lib.load().pa_block_alloc_fork(handle, parent, child))


def pa_block_alloc_free_sequence(handle, seq: int) -> None:
    _check(_lib.load().pa_block_alloc_free_sequence(handle, seq))


def pa_block_alloc_slot_mapping(handle, seq: int, start: int, count: int) -> np.ndarray:
    out = np.empty(max(count, 0), dtype=np.int64)
    _check(_lib.load().pa_block_alloc_slot_mapping(handle, seq, start, count, _i64p(out)))
    return out


def pa_block_alloc_block_table(handle, seq: int) -> np.ndarray:
    lib = _lib.load()
    n = ctypes.c_int32(-1)
    st = lib.pa_block_alloc_block_table(handle, seq, None, 0, ctypes.byref(n))  # length query
    if n.value < 0:
        _check(st)
    out = np.empty(n.value, dtype=np.int32)
    if n.value > 0:
        _check(lib.pa_block_alloc_block_table(handle, seq, _i32p(out), n.value, ctypes.byref(n)))
    return out


def pa_block_alloc_block_tables(handle, seqs: Sequence[int], max_blocks_per_seq: int, pad: int = -1,
                                out: Optional[np.ndarray] = None, lens_out: Optional[np.ndarray] = None):
    """Padded [n, max_blocks_per_seq] int32 tables and [n] int32 token counts (into out / lens_out if given)."""
    ids = np.ascontiguousarray(seqs, dtype=np.int64)
    tables = np.empty((len(ids), max_blocks_per_seq), dtype=np.int32) if out is None else out
    lens = np.empty(len(ids), dtype=np.int32) if lens_out is None else lens_out
    if tables.shape != (len(ids), max_blocks_per_seq) or tables.dtype != np.int32 or not tables.flags.c_contiguous:
        raise ValueError("out must be a C-contiguous int32 [n, max_blocks_per_seq] array")
    if lens.shape != (len(ids),) or lens.dtype != np.int32:
        raise ValueError("lens_out must be an int32 [n] array")
    _check(_lib.load().pa_block_alloc_block_tables(handle, _i64p(ids), len(ids), _i32p(tables),
                                                   max_blocks_per_seq, pad, _i32p(lens)))
    return tables, lens


def pa_block_alloc_table_updates(handle, seqs: Sequence[int], max_blocks_per_seq: int, pad: int = -1,
                                 out: Optional[np.ndarray] = None, lens_out: Optional[np.ndarray] = None):
    """(row, column, page) updates since the last call for the batch `seqs` (int32 [k, 3], a view of
    `out` when given) and the [n] int32 token counts.  Without `out` the array is sized to fit; a
    given `out` too small raises (the allocator is left unchanged)."""
    ids = np.ascontiguousarray(seqs, dtype=np.int64)
    lens = np.empty(len(ids), dtype=np.int32) if lens_out is None else lens_out
    if lens.shape != (len(ids),) or lens.dtype != np.int32:
        raise ValueError("lens_out must be an int32 [n] array")
    lib = _lib.load()
    n_out = ctypes.c_int32(0)
    if out is None:
        st = lib.pa_block_alloc_table_updates(handle, _i64p(ids), len(ids), max_blocks_per_seq, pad, None, 0,
                                              ctypes.byref(n_out), None)
        if st not in (_lib.PA_OK, _lib.PA_ERR_INVALID):
            _check(st)
        out = np.empty((max(1, n_out.value), 3), dtype=np.int32)
    if out.ndim != 2 or out.shape[1] != 3 or out.dtype != np.int32 or not out.flags.c_contiguous:
        raise ValueError("out must be a C-contiguous int32 [cap, 3] array")
    _check(lib.pa_block_alloc_table_updates(handle, _i64p(ids), len(ids), max_blocks_per_seq, pad, _i32p(out),
                                            int(out.shape[0]), ctypes.byref(n_out), _i32p(lens)))
    return out[:n_out.value], lens


def pa_block_alloc_num_tokens(handle, seq: int) -> int:
    return int(_lib.load().pa_block_alloc_num_tokens(handle, seq))


def pa_block_alloc_num_free(handle) -> int:
    return int(_lib.load().pa_block_alloc_num_free(handle))


def pa_block_alloc_num_sequences(handle) -> int:
    return int(_lib.load().pa_block_alloc_num_sequences(handle))


def pa_block_alloc_ref_count(handle, page: int) -> int:
    return int(_lib.load().pa_block_alloc_ref_count(handle, page))


def pa_block_alloc_free_pool(handle) -> np.ndarray:
    n = pa_block_alloc_num_free(handle)
    out = np.empty(n, dtype=np.int32)
    got = ctypes.c_int32()
    _check(_lib.load().pa_block_alloc_free_pool(handle, _i32p(out), n, ctypes.byref(got)))
    return out


def pa_block_alloc_stats(handle, alarm_free_fraction: float = _lib.PA_LOW_FREE_FRACTION) -> dict:
    """Pool occupancy and internal fragmentation (pa_pool_stats) as a dict."""
    st = _lib.PoolStats()
    _check(_lib.load().pa_block_alloc_stats(handle, float(alarm_free_fraction), ctypes.byref(st)))
    out = {name: getattr(st, name) for name, _ in _lib.PoolStats._fields_ if name != "reserved0"}
    out["low_free_alarm"] = bool(out["low_free_alarm"])
    return out


def pa_block_alloc_prefix_plan(handle, seqs: Sequence[int], group_size: int) -> dict:
    """Host prefix plan of a batch (see include/pa.h): numpy arrays and counts."""
    ids = np.ascontiguousarray(seqs, dtype=np.int64)
    n = len(ids)
    first = np.zeros(max(n, 1), dtype=np.int32)
    chunks = np.zeros((max(n, 1), 4), dtype=np.int32)
    members = np.zeros(max(n, 1), dtype=np.int32)
    nc, nm, msp, mnp = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.load().pa_block_alloc_prefix_plan(handle, _i64p(ids), n, group_size, _i32p(first), _i32p(chunks),
                                                  _i32p(members), ctypes.byref(nc), ctypes.byref(nm),
                                                  ctypes.byref(msp), ctypes.byref(mnp)))
    return {"first_partition": first[:n], "chunks": chunks[:max(nc.value, 1)], "members": members[:max(nm.value, 1)],
            "num_chunks": nc.value, "num_members": nm.value, "max_shared_partitions": msp.value,
            "min_shared_partitions": mnp.value}


def prefix_plan_to_device(plan: dict, device="cuda") -> dict:
    """Copy a host prefix plan's arrays to the device (PyTorch is the allocator)."""
    torch = _torch()
    out = dict(plan)
    for k in ("first_partition", "chunks", "members"):
        out[k] = torch.from_numpy(np.ascontiguousarray(plan[k])).to(device)
    return out


class BlockAllocator:
    """Owns one pa_block_alloc handle; methods map one-to-one onto the C calls."""

    def __init__(self, num_blocks: int, block_size: int, initial_free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.handle = pa_block_alloc_create(num_blocks, block_size, initial_free_order)

    def close(self) -> None:
        if self.handle:
            pa_block_alloc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def allocate_sequence(self, seq, num_tokens):
        pa_block_alloc_allocate_sequence(self.handle, seq, num_tokens)

    def append_token(self, seq):
        return pa_block_alloc_append_token(self.handle, seq)

    def append_tokens(self, seqs):
        return pa_block_alloc_append_tokens(self.handle, seqs)

    def fork(self, parent, child):
        pa_block_alloc_fork(self.handle, parent, child)

    def free_sequence(self, seq):
        pa_block_alloc_free_sequence(self.handle, seq)

    def slot_mapping(self, seq, start, count):
        return pa_block_alloc_slot_mapping(self.handle, seq, start, count)

    def block_table(self, seq):
        return pa_block_alloc_block_table(self.handle, seq)

    def block_tables(self, seqs, max_blocks_per_seq, pad=-1, out=None, lens_out=None):
        return pa_block_alloc_block_tables(self.handle, seqs, max_blocks_per_seq, pad, out, lens_out)

    def table_updates(self, seqs, max_blocks_per_seq, pad=-1, out=None, lens_out=None):
        return pa_block_alloc_table_updates(self.handle, seqs, max_blocks_per_seq, pad, out, lens_out)

    def num_tokens(self, seq):
        return pa_block_alloc_num_tokens(self.handle, seq)

    def num_free(self):
        return pa_block_alloc_num_free(self.handle)

    def num_sequences(self):
        return pa_block_alloc_num_sequences(self.handle)

    def ref_count(self, page):
        return pa_block_alloc_ref_count(self.handle, page)

    def free_pool(self):
        return pa_block_alloc_free_pool(self.handle)

    def prefix_plan(self, seqs, group_size):
        return pa_block_alloc_prefix_plan(self.handle, seqs, group_size)

    def stats(self, alarm_free_fraction=_lib.PA_LOW_FREE_FRACTION):
        return pa_block_alloc_stats(self.handle, alarm_free_fraction)

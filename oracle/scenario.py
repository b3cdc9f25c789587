"""Run a workload trace through the oracle pieces -- TEST INFRASTRUCTURE ONLY (oracle).

The workload object is passed in (duck-typed: ``trace``, ``token_kv``,
``query``, shapes); this module imports nothing from the CUDA path.
Trace ops: allocate, fork, append, copy_pending, write, decode (see the
workload generator for their meaning).
"""
from __future__ import annotations

import numpy as np

from . import attention, cache_ops
from .allocator import PagePool


def run(workload, with_data: bool = True, decode_seqs=None) -> dict:
    """Execute ``workload.trace``; return allocator state (and the allocator), caches, slots, copy pairs
    and output.

    ``with_data=False`` runs the allocator and slot bookkeeping only (no cache
    arrays, no attention), which is cheap even for the largest workloads.
    ``decode_seqs`` restricts the fp64 attention to those sequences.
    """
    w = workload
    mgr = PagePool(w.num_blocks, w.block_size, w.initial_free_order())
    store = np.uint16 if w.dtype in ("bf16", "f16") else np.float32
    kc = vc = None
    if with_data:
        kc = np.zeros((w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim), dtype=store)
        vc = np.zeros_like(kc)
    pending, all_pairs, write_slots, append_slots = [], [], [], []
    result = {}
    for op in w.trace:
        kind = op[0]
        if kind == "allocate":
            mgr.admit(op[1], op[2])
        elif kind == "fork":
            mgr.share(op[1], op[2])
        elif kind == "append":
            for _ in range(op[2]):
                slot, pair = mgr.extend(op[1])
                append_slots.append(slot)
                if pair is not None:
                    pending.append(pair)
        elif kind == "copy_pending":
            if with_data and pending:
                cache_ops.copy_blocks(kc, vc, pending)
            all_pairs.extend(pending)
            pending = []
        elif kind == "write":
            _, seq, start, count = op
            slots = np.array([mgr.slot(seq, p) for p in range(start, start + count)], dtype=np.int64)
            write_slots.append(slots)
            if with_data:
                k, v = w.token_kv(seq, start, count)
                cache_ops.reshape_and_cache(k, v, slots, kc, vc)
        elif kind == "decode":
            tables = np.full((w.num_seqs, w.max_blocks_per_seq), -1, dtype=np.int32)
            for b in range(w.num_seqs):
                t = mgr.tables[b]
                tables[b, :len(t)] = t
            ctx = np.array([mgr.lengths[b] for b in range(w.num_seqs)], dtype=np.int32)
            result["block_tables"] = tables
            result["context_lens"] = ctx
            if with_data:
                result["out"] = attention.decode_attention(w.query(), kc, vc, tables, ctx, w.scale,
                                                           w.dtype, seqs=decode_seqs)
        else:
            raise ValueError(f"unknown trace op {kind!r}")
    result.update(state=mgr.state(), manager=mgr, key_cache=kc, value_cache=vc, cow_pairs=all_pairs,
                  write_slots=np.concatenate(write_slots) if write_slots else np.zeros(0, np.int64),
                  append_slots=np.array(append_slots, dtype=np.int64))
    return result

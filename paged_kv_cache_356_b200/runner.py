"""Drive a workload trace through the C ABI: the host allocator plus the CUDA kernels.

This is how a serving loop uses the library: admit / fork / grow sequences
with ``pa_block_alloc``, copy the pages that copy-on-write forked with
``pa_copy_blocks``, store new tokens with ``pa_reshape_and_cache``, and run
``pa_decode`` over the block tables the allocator exports.  Trace ops are
those of ``workloads`` (allocate, fork, append, copy_pending, write, decode).

Consecutive ``write`` ops are issued as one ``pa_reshape_and_cache`` call
(split into chunks of at most ``max_chunk_tokens`` tokens to bound the
staging memory).  The last write group before ``decode`` is kept on the
device as the decode step's own cache write, so a benchmark can replay
exactly one step: that write, then the decode.
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np

from . import binding as pa


class TraceRunner:
    def __init__(self, workload, device: str = "cuda", max_chunk_tokens: int = 1 << 17, threads: int = 8,
                 shared_prefix: bool = False):
        import torch

        self.torch = torch
        self.w = w = workload
        self.device = torch.device(device)
        self.dtype = {"bf16": torch.bfloat16, "f32": torch.float32, "f16": torch.float16}[w.dtype]
        self.alloc = pa.BlockAllocator(w.num_blocks, w.block_size, w.initial_free_order())
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
        self.key_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.value_cache = torch.zeros(shape, dtype=self.dtype, device=self.device)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.max_chunk_tokens = max_chunk_tokens
        self.threads = threads
        self.cow_pairs: List[tuple] = []
        self.write_slots: List[np.ndarray] = []
        self.step_write = None   # (key, value, slots) of the write group before decode, on the device
        self.q = self.block_tables = self.context_lens = self.out = self.workspace = None
        self.shared_prefix = shared_prefix
        self.plan = None

    # -- helpers ----------------------------------------------------------------------
    def _to_device(self, host: np.ndarray):
        torch = self.torch
        if host.dtype == np.uint16:
            t = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16 if self.w.dtype == "bf16" else torch.float16)
        else:
            t = torch.from_numpy(host)
        return t.to(self.device, non_blocking=False)

    def _flush_writes(self, ops, keep: bool) -> None:
        if not ops:
            return
        torch = self.torch
        chunks, cur, n = [], [], 0
        for op in ops:
            if cur and n + op[3] > self.max_chunk_tokens:
                chunks.append(cur)
                cur, n = [], 0
            cur.append(op)
            n += op[3]
        chunks.append(cur)
        for chunk in chunks:
            slots = np.concatenate([self.alloc.slot_mapping(op[1], op[2], op[3]) for op in chunk])
            self.write_slots.append(slots)
            k, v = self.w.batched_token_kv(chunk, threads=self.threads)
            kd, vd = self._to_device(k), self._to_device(v)
            sd = torch.from_numpy(slots).to(self.device)
            pa.pa_reshape_and_cache(kd, vd, sd, self.key_cache, self.value_cache, dev_status=self.dev_status)
            if keep and len(chunks) == 1:
                self.step_write = (kd, vd, sd)

    # -- execution ----------------------------------------------------------------------
    def run(self, decode: bool = True) -> Optional[object]:
        """Execute the trace; returns the decode output (device tensor) if reached."""
        torch = self.torch
        pending, group = [], []
        trace = self.w.trace
        for i, op in enumerate(trace):
            kind = op[0]
            if kind == "write":
                group.append(op)
                continue
            if group:
                self._flush_writes(group, keep=(kind == "decode"))
                group = []
            if kind == "allocate":
                self.alloc.allocate_sequence(op[1], op[2])
            elif kind == "fork":
                self.alloc.fork(op[1], op[2])
            elif kind == "append":
                for _ in range(op[2]):
                    _, src, dst = self.alloc.append_token(op[1])
                    if src >= 0:
                        pending.append((src, dst))
            elif kind == "copy_pending":
                if pending:
                    mapping = torch.tensor(pending, dtype=torch.int64, device=self.device)
                    pa.pa_copy_blocks(self.key_cache, self.value_cache, mapping, dev_status=self.dev_status)
                self.cow_pairs.extend(pending)
                pending = []
            elif kind == "decode":
                self.prepare_decode()
                if decode:
                    self.decode()
            else:
                raise ValueError(f"unknown trace op {kind!r}")
        if group:
            self._flush_writes(group, keep=False)
        return self.out

    def prepare_decode(self) -> None:
        torch = self.torch
        w = self.w
        tables, lens = self.alloc.block_tables(list(range(w.num_seqs)), w.max_blocks_per_seq, pad=-1)
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(lens).to(self.device)
        self.q = self._to_device(np.ascontiguousarray(w.query()))
        self.out = torch.empty_like(self.q)
        need = pa.pa_decode_workspace_size(w.num_seqs, w.num_q_heads, w.head_dim,
                                           w.max_blocks_per_seq * w.block_size)
        # NaN bytes to start with: a partial that no kernel wrote reaches the output as NaN.
        self.workspace = torch.full((max(need, 256),), 0xFF, dtype=torch.uint8, device=self.device)
        if self.shared_prefix:
            host = self.alloc.prefix_plan(list(range(w.num_seqs)), w.group_size)
            self.plan = pa.prefix_plan_to_device(host, self.device)

    def decode(self, stream=None):
        if self.plan is not None:
            return pa.pa_decode_shared_prefix(self.q, self.key_cache, self.value_cache, self.block_tables,
                                              self.context_lens, self.w.scale, self.plan, out=self.out,
                                              workspace=self.workspace, dev_status=self.dev_status, stream=stream)
        return pa.pa_decode(self.q, self.key_cache, self.value_cache, self.block_tables, self.context_lens,
                            self.w.scale, out=self.out, workspace=self.workspace, dev_status=self.dev_status,
                            stream=stream)

    def step(self, stream=None):
        """One decode step on resident inputs: the step's cache write, then decode."""
        if self.step_write is not None:
            k, v, s = self.step_write
            pa.pa_reshape_and_cache(k, v, s, self.key_cache, self.value_cache, dev_status=self.dev_status,
                                    stream=stream)
        return self.decode(stream)

    # -- inspection ---------------------------------------------------------------------
    def allocator_state(self) -> dict:
        w = self.w
        a = self.alloc
        seqs = {}
        for b in range(w.num_seqs):
            seqs[b] = [int(p) for p in a.block_table(b)]
        return {
            "free_pool": [int(p) for p in a.free_pool()],
            "ref_count": [a.ref_count(p) for p in range(w.num_blocks)],
            "block_tables": seqs,
            "num_tokens": {b: a.num_tokens(b) for b in range(w.num_seqs)},
        }

    def status(self) -> int:
        return int(self.dev_status.item())

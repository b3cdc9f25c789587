"""Seeded synthetic workloads for the paged decode path.

This module only prepares inputs: shapes, context-length draws, the initial
order of the free-page pool, per-token K/V values, query values, and the
trace of allocator / cache operations a workload performs.  It holds none of
the method's arithmetic (no block-table translation, no allocator policy, no
attention), so that the CUDA path and the CPU oracle can both consume it
without sharing any code that computes a result.

Random streams: every array is drawn from numpy's PCG64 seeded with a
``SeedSequence`` whose entropy is ``(workload seed, stream tag, ...)``, so any
sub-array (one sequence's prefill, one write) can be regenerated on its own.

bf16 values are returned as ``uint16`` bit patterns.  A bf16 N(0,1) value is
drawn by inverse-CDF sampling: a uniform 16-bit index selects the
``(i + 1/2) / 65536`` quantile of the standard normal, rounded to bf16.  At
bf16's 8-bit mantissa this is indistinguishable from rounding an fp32 normal
draw, and it is an order of magnitude faster on the host, which matters for
the 2.9 GB Llama-3-70B-shaped cache.  fp32 values are plain fp32 normal draws.

Workloads (the five configurations of the decode path):

``tiny``      2 sequences of 36 and 42 tokens, block 16, a pool of 16 pages
              in seeded random order, 4 q heads / 1 kv head, head_dim 64, fp32.
``llama8b``   64 sequences, 32 q / 8 kv heads, head_dim 128, bf16, block 16,
              context ~ U{128..4096}, pool 1.25x the pages used, shuffled.
``llama70b``  256 sequences, 64 q / 8 kv heads, head_dim 128, bf16, block 16,
              context = floor(exp(U(ln 512, ln 8192))), pool 1.25x, shuffled.
``prefix``    100 sequences forked from one 10,000-token prefix, tails
              ~ U{1..512}, 32 q / 8 kv heads, head_dim 128, bf16, block 32.
``beam32k``   8 beams forked from one 32,768-token prompt, 64 own tokens each,
              64 q / 8 kv heads, head_dim 128, bf16, block 16.
"""
from __future__ import annotations

import math
import statistics
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np

# Stream tags of the SeedSequence entropy tuple.
_TAG_LENGTHS = 1
_TAG_POOL = 2
_TAG_QUERY = 3
_TAG_KV = 4
_TAG_DRAFT = 5

_BF16_NORMAL_TABLE = None


def float32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); return uint16 bits.

    Input preparation only: both paths receive the same bits.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def _bf16_normal_table() -> np.ndarray:
    global _BF16_NORMAL_TABLE
    if _BF16_NORMAL_TABLE is None:
        nd = statistics.NormalDist()
        q = np.array([nd.inv_cdf((i + 0.5) / 65536.0) for i in range(65536)], dtype=np.float64)
        _BF16_NORMAL_TABLE = float32_to_bf16_bits(q.astype(np.float32))
    return _BF16_NORMAL_TABLE


def _rng(*entropy: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(entropy))))


def normal_values(rng: np.random.Generator, n: int, dtype: str) -> np.ndarray:
    """n i.i.d. N(0,1) values: uint16 bf16 bits for 'bf16', float32 for 'f32'."""
    if dtype == "bf16":
        idx = rng.integers(0, 65536, size=n, dtype=np.uint16)
        return _bf16_normal_table()[idx]
    if dtype == "f32":
        return rng.standard_normal(n, dtype=np.float32)
    raise ValueError(f"unsupported dtype {dtype!r}")


# ---------------------------------------------------------------------------
# Trace of operations.  Each op is a tuple whose first item names it:
#   ("allocate", seq, num_tokens)   admit a sequence with num_tokens slots
#   ("fork", parent, child)         child shares all of parent's pages
#   ("append", seq, count)          grow seq by count tokens, one at a time
#   ("copy_pending",)               copy every page pair that appends forked
#   ("write", seq, start, count)    store K/V of positions [start, start+count)
#   ("decode",)                     one decode step over all sequences 0..B-1
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    kind: str  # "independent" | "prefix" | "beam"
    context_lens: Tuple[int, ...]
    num_blocks: int
    prefix_len: int = 0
    trace: Tuple[tuple, ...] = field(default=(), repr=False)

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def max_context_len(self) -> int:
        return max(self.context_lens) if self.context_lens else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return max(1, -(-self.max_context_len // self.block_size))

    # -- data ---------------------------------------------------------------
    def initial_free_order(self) -> np.ndarray:
        """Seeded permutation of 0..num_blocks-1: the pool's starting order."""
        return _rng(self.seed, _TAG_POOL).permutation(self.num_blocks).astype(np.int32)

    def query(self) -> np.ndarray:
        """q of the decode step, [num_seqs, num_q_heads, head_dim]."""
        n = self.num_seqs * self.num_q_heads * self.head_dim
        vals = normal_values(_rng(self.seed, _TAG_QUERY), n, self.dtype)
        return vals.reshape(self.num_seqs, self.num_q_heads, self.head_dim)

    def token_kv(self, seq: int, start: int, count: int) -> Tuple[np.ndarray, np.ndarray]:
        """K and V written by ``("write", seq, start, count)``: [count, Hkv, D] each."""
        n = count * self.num_kv_heads * self.head_dim
        rng = _rng(self.seed, _TAG_KV, seq, start)
        k = normal_values(rng, n, self.dtype).reshape(count, self.num_kv_heads, self.head_dim)
        v = normal_values(rng, n, self.dtype).reshape(count, self.num_kv_heads, self.head_dim)
        return k, v

    def draft_query(self, num_tokens: int) -> np.ndarray:
        """q of a draft-verification step, [num_seqs, num_tokens, num_q_heads, head_dim]."""
        n = self.num_seqs * num_tokens * self.num_q_heads * self.head_dim
        vals = normal_values(_rng(self.seed, _TAG_DRAFT, num_tokens, 0), n, self.dtype)
        return vals.reshape(self.num_seqs, num_tokens, self.num_q_heads, self.head_dim)

    def draft_kv(self, num_tokens: int) -> Tuple[np.ndarray, np.ndarray]:
        """K and V of the draft tokens, stored at the last ``num_tokens`` positions of each
        sequence before the verification step: [num_seqs * num_tokens, Hkv, D] each, sequence-major."""
        n = self.num_seqs * num_tokens * self.num_kv_heads * self.head_dim
        rng = _rng(self.seed, _TAG_DRAFT, num_tokens, 1)
        shape = (self.num_seqs * num_tokens, self.num_kv_heads, self.head_dim)
        return normal_values(rng, n, self.dtype).reshape(shape), normal_values(rng, n, self.dtype).reshape(shape)

    def writes(self) -> List[tuple]:
        return [op for op in self.trace if op[0] == "write"]

    def batched_token_kv(self, ops: List[tuple], threads: int = 8):
        """Concatenate token_kv of several write ops (drawn in parallel threads)."""
        with ThreadPoolExecutor(max(1, threads)) as ex:
            parts = list(ex.map(lambda op: self.token_kv(op[1], op[2], op[3]), ops))
        if not parts:
            shape = (0, self.num_kv_heads, self.head_dim)
            dt = np.uint16 if self.dtype == "bf16" else np.float32
            return np.zeros(shape, dt), np.zeros(shape, dt)
        return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]))

    # -- lineage --------------------------------------------------------------
    def segments(self, seq: int) -> List[Tuple[int, int, int, int]]:
        """Where each position of ``seq`` got its data, from the trace alone.

        Returns ``(position, count, writer_seq, write_start)`` runs covering the
        positions written for ``seq``: a forked child inherits its parent's
        runs at the time of the fork, then adds its own writes.
        """
        runs = {}
        for op in self.trace:
            if op[0] == "allocate":
                runs[op[1]] = []
            elif op[0] == "fork":
                runs[op[2]] = list(runs[op[1]])
            elif op[0] == "write":
                _, s, start, count = op
                runs[s].append((start, count, s, start))
        return sorted(runs.get(seq, []))

    def sequence_kv(self, seq: int) -> Tuple[np.ndarray, np.ndarray]:
        """Contiguous K, V of ``seq`` in position order, [ctx, Hkv, D], from the trace."""
        ks, vs = [], []
        pos = 0
        for start, count, writer, wstart in self.segments(seq):
            if start != pos:
                raise ValueError(f"sequence {seq}: positions {pos}..{start} were never written")
            k, v = self.token_kv(writer, wstart, count)
            ks.append(k)
            vs.append(v)
            pos += count
        if pos != self.context_lens[seq]:
            raise ValueError(f"sequence {seq}: {pos} positions written, context {self.context_lens[seq]}")
        return np.concatenate(ks), np.concatenate(vs)


def _independent_trace(context_lens) -> Tuple[tuple, ...]:
    """Admit every sequence with ctx-1 tokens, prefill them, then append and write the new token.

    A sequence of context 0 is admitted empty and never written.
    """
    ops = []
    for b, ctx in enumerate(context_lens):
        ops.append(("allocate", b, max(ctx - 1, 0)))
    for b, ctx in enumerate(context_lens):
        if ctx - 1 > 0:
            ops.append(("write", b, 0, ctx - 1))
    for b, ctx in enumerate(context_lens):
        if ctx > 0:
            ops.append(("append", b, 1))
    for b, ctx in enumerate(context_lens):
        if ctx > 0:
            ops.append(("write", b, ctx - 1, 1))
    ops.append(("decode",))
    return tuple(ops)


def _shared_trace(prefix_len, tails) -> Tuple[tuple, ...]:
    """Sequence 0 holds the prefix; 1..B-1 fork from it; each appends its tail.

    The tails but their last token are appended (in sequence order), the
    pending page copies made and the tokens written; then every sequence
    appends its new token, the pages that append forked are copied, the new
    tokens are written (the decode step's own cache write) and the step
    decodes.  A tail of one token is just the new token.
    """
    ops = [("allocate", 0, prefix_len), ("write", 0, 0, prefix_len)]
    for b in range(1, len(tails)):
        ops.append(("fork", 0, b))
    for b, t in enumerate(tails):
        if t > 1:
            ops.append(("append", b, t - 1))
    ops.append(("copy_pending",))
    for b, t in enumerate(tails):
        if t > 1:
            ops.append(("write", b, prefix_len, t - 1))
    for b in range(len(tails)):
        ops.append(("append", b, 1))
    ops.append(("copy_pending",))
    for b, t in enumerate(tails):
        ops.append(("write", b, prefix_len + t - 1, 1))
    ops.append(("decode",))
    return tuple(ops)


def _pool_size(pages_needed: int) -> int:
    return int(math.ceil(1.25 * pages_needed))


def tiny(seed: int = 0) -> Workload:
    ctx = (36, 42)
    return Workload("tiny", seed, 2, 4, 1, 64, 16, "f32", "independent", ctx, 16,
                    trace=_independent_trace(ctx))


def _independent(name, seed, num_seqs, hq, hkv, d, bs, ctx) -> Workload:
    ctx = tuple(int(c) for c in ctx)
    pages = sum(-(-c // bs) for c in ctx)
    return Workload(name, seed, num_seqs, hq, hkv, d, bs, "bf16", "independent", ctx,
                    _pool_size(pages), trace=_independent_trace(ctx))


def llama8b(seed: int = 1, num_seqs: int = 64, lo: int = 128, hi: int = 4096, block_size: int = 16) -> Workload:
    ctx = _rng(seed, _TAG_LENGTHS).integers(lo, hi + 1, size=num_seqs)
    return _independent("llama8b", seed, num_seqs, 32, 8, 128, block_size, ctx)


def llama70b(seed: int = 2, num_seqs: int = 256, lo: int = 512, hi: int = 8192, block_size: int = 16) -> Workload:
    u = _rng(seed, _TAG_LENGTHS).uniform(math.log(lo), math.log(hi), size=num_seqs)
    ctx = np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int64)
    return _independent("llama70b", seed, num_seqs, 64, 8, 128, block_size, ctx)


def prefix(seed: int = 3, num_seqs: int = 100, prefix_len: int = 10_000, max_tail: int = 512,
           block_size: int = 32) -> Workload:
    tails = _rng(seed, _TAG_LENGTHS).integers(1, max_tail + 1, size=num_seqs)
    ctx = tuple(int(prefix_len + t) for t in tails)
    bound = -(-prefix_len // block_size) + num_seqs * (1 + -(-max_tail // block_size))
    return Workload("prefix", seed, num_seqs, 32, 8, 128, block_size, "bf16", "prefix", ctx,
                    _pool_size(bound), prefix_len=prefix_len,
                    trace=_shared_trace(prefix_len, [int(t) for t in tails]))


def beam32k(seed: int = 4, num_beams: int = 8, prompt_len: int = 32_768, own: int = 64,
            block_size: int = 16) -> Workload:
    ctx = tuple([prompt_len + own] * num_beams)
    bound = -(-prompt_len // block_size) + num_beams * (1 + -(-own // block_size))
    return Workload("beam32k", seed, num_beams, 64, 8, 128, block_size, "bf16", "beam", ctx,
                    _pool_size(bound), prefix_len=prompt_len,
                    trace=_shared_trace(prompt_len, [own] * num_beams))


def custom(name: str, seed: int, context_lens, num_q_heads: int, num_kv_heads: int,
           head_dim: int, block_size: int, dtype: str, num_blocks: int = 0) -> Workload:
    """An independent-sequences workload with explicit lengths (edge cases)."""
    ctx = tuple(int(c) for c in context_lens)
    pages = sum(-(-max(c, 1) // block_size) for c in ctx)
    nb = num_blocks or max(1, _pool_size(pages))
    return Workload(name, seed, len(ctx), num_q_heads, num_kv_heads, head_dim, block_size, dtype,
                    "independent", ctx, nb, trace=_independent_trace(ctx))


WORKLOADS = {"tiny": tiny, "llama8b": llama8b, "llama70b": llama70b,
             "prefix": prefix, "beam32k": beam32k}


def by_name(name: str, **kw) -> Workload:
    return WORKLOADS[name](**kw)

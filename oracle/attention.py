"""Decode attention over a paged KV cache, in fp64 -- TEST INFRASTRUCTURE ONLY (oracle).

What the path computes, stated plainly:

* Block-table translation (Internals, "2. The Dynamic Block Table"; Glossary,
  "Technical Architecture" and "On-the-Fly CUDA Block Fetching"): logical
  position j of sequence b lives in physical page ``block_table[b][j // bs]``
  at slot ``j % bs``.  ``gather_sequence`` follows the table and returns the
  sequence's keys or values as one contiguous array.
* Scaled dot-product attention for one new query per head (Internals,
  "3. Fused PagedAttention CUDA Kernel": the kernel runs scaled dot-product
  attention on the keys and values it fetched through the table).  The
  textbook definition: ``s_j = scale * q . k_j``, ``p = softmax(s)``,
  ``out = sum_j p_j v_j``, over every stored position ``j < context_len``.

Readings (the pages are silent): query head h reads kv head ``h // G`` with
``G = H_q / H_kv`` (consecutive grouping); no mask beyond ``j < context_len``;
an empty sequence yields zeros.

``partition_attention`` / ``lse_merge`` state the split-context form the
decode path uses for long sequences: per 512-token partition the normalised
partial output ``o_p``, the partition's score maximum ``m_p`` and
``l_p = sum exp(s_j - m_p)``; merging them with weights ``l_p * exp(m_p - M)``
reproduces the unsplit softmax exactly (up to rounding).

``verify_attention`` is the same attention for several query tokens per
sequence (draft-token verification), each seeing the keys up to its own
position.
"""
from __future__ import annotations

import numpy as np


def to_float64(values: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored values to fp64: bf16 bits (uint16), float16 or float32."""
    a = np.asarray(values)
    if dtype == "bf16":
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "f16":
        return a.view(np.float16).astype(np.float64)
    if dtype == "f32":
        return a.astype(np.float32).astype(np.float64)
    raise ValueError(f"unsupported dtype {dtype!r}")


def gather_sequence(cache: np.ndarray, block_table, context_len: int) -> np.ndarray:
    """Contiguous ``[context_len, H_kv, D]`` rows of one sequence, read through its table."""
    bs = cache.shape[2]
    pos = np.arange(context_len)
    pages = np.asarray(block_table, dtype=np.int64)[pos // bs]
    return cache[pages, :, pos % bs, :]


def softmax_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """Textbook attention of one query row over contiguous keys/values (fp64)."""
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1:], dtype=np.float64)
    s = scale * (keys @ q)
    e = np.exp(s - s.max())
    return (e / e.sum()) @ values


def decode_attention(q, key_cache, value_cache, block_tables, context_lens, scale: float,
                     dtype: str, seqs=None) -> np.ndarray:
    """fp64 output ``[B, H_q, D]`` of one decode step (rows of ``seqs`` only, if given).

    ``q`` is ``[B, H_q, D]``; caches are ``[pages, H_kv, bs, D]`` in their stored
    type; ``block_tables`` ``[B, max_blocks]``; ``context_lens`` ``[B]``.
    """
    q64 = to_float64(q, dtype)
    num_seqs, num_q_heads, head_dim = q64.shape
    num_kv_heads = key_cache.shape[1]
    group = num_q_heads // num_kv_heads
    out = np.zeros((num_seqs, num_q_heads, head_dim), dtype=np.float64)
    for b in (range(num_seqs) if seqs is None else seqs):
        ctx = int(context_lens[b])
        keys = to_float64(gather_sequence(key_cache, block_tables[b], ctx), dtype)
        values = to_float64(gather_sequence(value_cache, block_tables[b], ctx), dtype)
        for h in range(num_q_heads):
            out[b, h] = softmax_attention(q64[b, h], keys[:, h // group, :], values[:, h // group, :], scale)
    return out


def partition_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float,
                        partition_tokens: int = 512):
    """Per-partition ``(o_p, m_p, l_p)`` of one query row over contiguous keys/values."""
    parts = []
    for start in range(0, keys.shape[0], partition_tokens):
        kp = keys[start:start + partition_tokens]
        vp = values[start:start + partition_tokens]
        s = scale * (kp @ q)
        m = s.max()
        e = np.exp(s - m)
        parts.append(((e @ vp) / e.sum(), m, e.sum()))
    return parts


def lse_merge(parts) -> np.ndarray:
    """Combine partition partials: ``sum_p w_p o_p / sum_p w_p`` with ``w_p = l_p e^(m_p - M)``."""
    m_all = max(m for _, m, _ in parts)
    weights = [l * np.exp(m - m_all) for _, m, l in parts]
    return sum(w * o for w, (o, _, _) in zip(weights, parts)) / sum(weights)


def visible_keys(context_len: int, num_tokens: int, t: int) -> int:
    """Keys that query token t of ``num_tokens`` sees: positions ``0 .. context_len - num_tokens + t``."""
    return max(0, context_len - num_tokens + t + 1)


def verify_attention(q, key_cache, value_cache, block_tables, context_lens, scale: float,
                     dtype: str, seqs=None) -> np.ndarray:
    """fp64 output ``[B, T, H_q, D]`` for T query tokens per sequence (draft verification).

    Internals, "The Mathematical Cause of KV Cache Fragmentation", points to
    speculative-decoding kernels that check several draft tokens of a sequence
    at once against its paged memory.  Reading (the page gives no formula):
    the T query tokens of sequence b are the last T positions of its context,
    ``pos_t = context_lens[b] - T + t``, their own K/V already written; token
    t attends causally, i.e. to the keys ``j <= pos_t``, and to nothing else.
    A token with ``pos_t < 0`` sees no key and yields zeros.  With T = 1 this
    is ``decode_attention``.

    ``q`` is ``[B, T, H_q, D]``; the other arguments are as in ``decode_attention``.
    """
    q64 = to_float64(q, dtype)
    num_seqs, num_tokens, num_q_heads, head_dim = q64.shape
    num_kv_heads = key_cache.shape[1]
    group = num_q_heads // num_kv_heads
    out = np.zeros(q64.shape, dtype=np.float64)
    for b in (range(num_seqs) if seqs is None else seqs):
        ctx = int(context_lens[b])
        keys = to_float64(gather_sequence(key_cache, block_tables[b], ctx), dtype)
        values = to_float64(gather_sequence(value_cache, block_tables[b], ctx), dtype)
        for t in range(num_tokens):
            visible = visible_keys(ctx, num_tokens, t)
            for h in range(num_q_heads):
                out[b, t, h] = softmax_attention(q64[b, t, h], keys[:visible, h // group, :],
                                                 values[:visible, h // group, :], scale)
    return out

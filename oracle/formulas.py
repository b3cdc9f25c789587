"""Closed-form quantities the pages state -- TEST INFRASTRUCTURE ONLY (oracle).

Each function is the definition written out, with the passage it follows.
"""
from __future__ import annotations

from typing import List, Tuple


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """Fixed-size pages needed for ``num_tokens`` tokens: the ceiling of n / bs.

    Glossary, "Step-by-Step Implementation Framework" (42 tokens take 3 pages
    of 16); Internals, "Implementation: Custom Block Manager Simulation in
    Python" (a sequence is given its token count rounded up to whole blocks).
    """
    if num_tokens < 0 or block_size <= 0:
        raise ValueError("num_tokens must be >= 0 and block_size > 0")
    return (num_tokens + block_size - 1) // block_size


def logical_blocks(num_tokens: int, block_size: int) -> List[Tuple[int, int]]:
    """Inclusive token ranges of each logical block of a sequence.

    Glossary, "Logical Block Partitioning" and the "Technical Architecture"
    diagram (36 tokens -> blocks 0-15, 16-31, 32-35); Internals,
    "1. Fixed-Size Block Fragmentation".
    """
    out = []
    for i in range(blocks_needed(num_tokens, block_size)):
        first = i * block_size
        last = min(first + block_size, num_tokens) - 1
        out.append((first, last))
    return out


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
    """KV-cache bytes one token occupies: 2 (K and V) x L x H_kv x D x P.

    Internals, "The Mathematical Cause of KV Cache Fragmentation" (the
    per-token memory equation; 327,680 bytes for Llama 3 70B in FP16).
    """
    return 2 * num_layers * num_kv_heads * head_dim * bytes_per_elem


def internal_waste_fraction(reserved_tokens: int, used_tokens: int) -> float:
    """Share of a reservation that holds no token: (reserved - used) / reserved.

    Internals, "The Mathematical Cause of KV Cache Fragmentation", item
    "1. Internal Fragmentation" (512 of 4,096 reserved tokens used: 87.5%).
    """
    if reserved_tokens <= 0 or used_tokens < 0 or used_tokens > reserved_tokens:
        raise ValueError("need 0 <= used <= reserved, reserved > 0")
    return (reserved_tokens - used_tokens) / reserved_tokens


def paged_waste_slots(num_tokens: int, block_size: int) -> int:
    """Unused slots of a paged sequence: whole pages held minus tokens stored.

    With pages allocated on demand only the last page can be partly empty
    (Glossary, "Technical Architecture": 36 tokens hold 3 pages, 12 slots
    free in the last).
    """
    return blocks_needed(num_tokens, block_size) * block_size - num_tokens

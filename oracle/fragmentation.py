"""Occupancy and internal fragmentation of the page pool -- TEST INFRASTRUCTURE ONLY (oracle).

Internals, "The Mathematical Cause of KV Cache Fragmentation": internal
fragmentation is memory reserved for a request that holds none of its tokens
(item 1 of that section).  Under paging a sequence reserves only the pages its
tokens need, so only a page's unwritten slots are wasted; a page that several
sequences share after a fork is one physical page, and its filled slots are the
most that any holder has stored in it.  "Architectural Recommendations for
Infrastructure Engineers", item 3: raise an alert when the free pages fall
below 10 percent of the pool.

``pool_stats`` reads an allocator state as ``PagePool.state()``
returns it and states every quantity by its definition.
"""
from __future__ import annotations

LOW_FREE_FRACTION = 0.10


def pool_stats(state: dict, num_blocks: int, block_size: int,
               alarm_free_fraction: float = LOW_FREE_FRACTION) -> dict:
    refs = state["ref_count"]
    tables = state["block_tables"]
    tokens = state["num_tokens"]
    filled = {}                       # page -> slots holding a token
    for seq, table in tables.items():
        n = tokens[seq]
        for i, page in enumerate(table):
            filled[page] = max(filled.get(page, 0), min(block_size, n - i * block_size))
    used = sum(1 for r in refs if r > 0)
    free = len(state["free_pool"])
    physical = sum(filled.values())
    waste = used * block_size - physical
    free_fraction = free / num_blocks if num_blocks > 0 else 0.0
    return {
        "num_blocks": num_blocks,
        "block_size": block_size,
        "free_pages": free,
        "used_pages": used,
        "shared_pages": sum(1 for r in refs if r > 1),
        "num_sequences": len(tables),
        "logical_tokens": sum(tokens.values()),
        "physical_tokens": physical,
        "waste_slots": waste,
        "waste_fraction": waste / (used * block_size) if used > 0 else 0.0,
        "free_fraction": free_fraction,
        "low_free_alarm": num_blocks > 0 and free_fraction < alarm_free_fraction,
    }

"""Writing tokens into page slots and copying whole pages -- TEST INFRASTRUCTURE ONLY (oracle).

Cache layout (a reading: the pages fix none): ``cache[page, kv_head, slot_in_page, d]``,
one array for K and one for V, element type as stored (uint16 bf16 bits or
float32), so that both operations here are pure data movement and can be
compared bit for bit.
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(key, value, slot_mapping, key_cache, value_cache) -> None:
    """Store token t's K/V rows ``[kv_head, d]`` at physical slot ``slot_mapping[t]``.

    Slot s is page ``s // bs``, offset ``s % bs``; a negative slot means the
    token is padding and is skipped.  New tokens land in the pages allocated
    for them (Internals, "2. The Dynamic Block Table": pages come on demand
    from the free pool as tokens are generated).
    """
    bs = key_cache.shape[2]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        page, off = divmod(slot, bs)
        key_cache[page, :, off, :] = key[t]
        value_cache[page, :, off, :] = value[t]


def copy_blocks(key_cache, value_cache, pairs) -> None:
    """Copy every slot of page ``src`` onto page ``dst``, K and V, for each pair.

    The device half of a copy-on-write fork (Glossary, "Copy-on-Write Memory
    Forking"; Internals, "Copy-on-Write and Prefix Sharing").
    """
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        key_cache[dst] = key_cache[src]
        value_cache[dst] = value_cache[src]

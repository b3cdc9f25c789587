"""pa_block_alloc_table_updates: applying its (row, column, page) triples to the tables it produced
last gives the full export, and a decode step ships only the entries that changed."""
import random

import numpy as np
import pytest

from paged_kv_cache_356_b200 import binding as pa


def _apply(mirror, updates):
    """The triples written into a host copy of the tables (what pa_block_tables_apply does on the
    device); each entry at most once per call."""
    seen = set()
    for row, col, page in updates.tolist():
        assert (row, col) not in seen, "an entry named twice in one call"
        seen.add((row, col))
        mirror[row, col] = page


def _check(alloc, mirror, batch, mb, pad=-1):
    updates, lens = alloc.table_updates(batch, mb, pad)
    _apply(mirror, updates)
    full, full_lens = alloc.block_tables(batch, mb, pad)
    np.testing.assert_array_equal(mirror[:len(batch)], full)
    np.testing.assert_array_equal(lens, full_lens)
    return updates


@pytest.mark.parametrize("seed", range(12))
def test_random_streams_rebuild_the_full_export(seed):
    """Allocate, fork, append (with copy-on-write), free and reorder the batch at random; after every
    export the updated copy equals pa_block_alloc_block_tables.  Rows start as garbage."""
    rng = random.Random(seed)
    bs, nb, mb = rng.choice([1, 2, 4, 16]), 400, 40
    alloc = pa.BlockAllocator(nb, bs, np.random.default_rng(seed).permutation(nb))
    mirror = np.random.default_rng(seed + 100).integers(-1000, 1000, size=(64, mb)).astype(np.int32)
    live, next_id = [], 0
    batch = []
    for step in range(300):
        op = rng.random()
        try:
            if op < 0.15 or not live:
                alloc.allocate_sequence(next_id, rng.randrange(0, 6 * bs))
                live.append(next_id)
                next_id += 1
            elif op < 0.25:
                alloc.fork(rng.choice(live), next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.32 and len(live) > 1:
                s = rng.choice(live)
                alloc.free_sequence(s)
                live.remove(s)
            else:
                for s in rng.sample(live, rng.randint(1, len(live))):
                    if alloc.num_tokens(s) < mb * bs:
                        alloc.append_token(s)
        except RuntimeError:
            pass  # pool exhausted: the failed op changed nothing
        if step % 3 == 0 and live:
            kind = rng.random()
            if kind < 0.5 and batch and all(s in live for s in batch):
                pass  # the same batch again: only logged entries move
            elif kind < 0.7:
                batch = sorted(live)[:48]
            else:
                batch = rng.sample(live, min(len(live), rng.randint(1, 48)))
            _check(alloc, mirror, batch, mb)


def test_decode_steps_ship_only_new_blocks():
    """A batch that only grows: after the first export, a step's updates are exactly the sequences
    whose new token starts a block, one entry each."""
    bs, mb = 16, 64
    alloc = pa.BlockAllocator(4096, bs)
    lens = [100, 16, 31, 512, 17, 1]
    for s, n in enumerate(lens):
        alloc.allocate_sequence(s, n)
    batch = list(range(len(lens)))
    mirror = np.full((len(batch), mb), 7, np.int32)
    first = _check(alloc, mirror, batch, mb)
    assert len(first) == len(batch) * mb  # rows new to the export: whole, pad included
    for _ in range(40):
        starts = [s for s in batch if alloc.num_tokens(s) % bs == 0]
        for s in batch:
            alloc.append_token(s)
        upd = _check(alloc, mirror, batch, mb)
        assert sorted(upd[:, 0].tolist()) == sorted(starts)
    assert len(_check(alloc, mirror, batch, mb)) == 0  # nothing changed: nothing shipped


def test_copy_on_write_replacement_is_shipped():
    bs, mb = 4, 8
    alloc = pa.BlockAllocator(64, bs)
    alloc.allocate_sequence(0, 6)
    alloc.fork(0, 1)
    mirror = np.zeros((2, mb), np.int32)
    _check(alloc, mirror, [0, 1], mb)
    _, src, dst = alloc.append_token(1)  # position 6 sits in shared page 1: forked
    assert src >= 0 and dst >= 0
    upd = _check(alloc, mirror, [0, 1], mb)
    assert upd.tolist() == [[1, 1, dst]]


def test_row_reuse_pads_the_previous_occupant_and_moves_are_whole():
    bs, mb = 4, 10
    alloc = pa.BlockAllocator(64, bs)
    alloc.allocate_sequence(0, 30)   # 8 pages
    alloc.allocate_sequence(1, 5)    # 2 pages
    mirror = np.zeros((2, mb), np.int32)
    _check(alloc, mirror, [0, 1], mb)
    upd = _check(alloc, mirror, [1, 0], mb)   # swapped rows: both whole, row 0 padded past 2 entries
    assert sorted(set(upd[:, 0].tolist())) == [0, 1]
    assert len(upd) == 8 + 8                  # row 0: 2 pages + 6 pads of the old 8; row 1: 8 pages
    alloc.free_sequence(0)
    alloc.allocate_sequence(0, 3)             # same id, new pages: whole again
    upd = _check(alloc, mirror, [1, 0], mb)
    assert set(upd[:, 0].tolist()) == {1}


def test_duplicate_rows_and_width_change():
    bs = 4
    alloc = pa.BlockAllocator(64, bs)
    alloc.allocate_sequence(5, 9)
    mirror = np.zeros((3, 12), np.int32)
    _check(alloc, mirror, [5, 5, 5], 12)
    alloc.append_token(5)
    alloc.append_token(5)
    alloc.append_token(5)   # token 12 starts block 3
    _check(alloc, mirror, [5, 5, 5], 12)
    mirror2 = np.full((3, 6), 99, np.int32)
    upd = _check(alloc, mirror2, [5, 5, 5], 6)   # a new width starts over: every entry of every row
    assert len(upd) == 3 * 6


def test_too_small_buffer_raises_and_changes_nothing():
    bs, mb = 4, 8
    alloc = pa.BlockAllocator(64, bs)
    alloc.allocate_sequence(0, 10)
    alloc.allocate_sequence(1, 3)
    with pytest.raises(RuntimeError):
        alloc.table_updates([0, 1], mb, out=np.zeros((3, 3), np.int32))
    mirror = np.zeros((2, mb), np.int32)
    upd = _check(alloc, mirror, [0, 1], mb)
    assert len(upd) == 2 * mb


def test_bad_arguments():
    alloc = pa.BlockAllocator(16, 4)
    alloc.allocate_sequence(0, 40)          # 10 pages
    with pytest.raises(RuntimeError):
        alloc.table_updates([0], 8)         # more pages than the table width
    with pytest.raises(RuntimeError):
        alloc.table_updates([3], 16)        # unknown sequence
    with pytest.raises(ValueError):
        alloc.table_updates([0], 16, out=np.zeros((4, 2), np.int32))

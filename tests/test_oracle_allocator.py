"""Pins of oracle/allocator.py: the pages' worked examples, the listing's stated
behaviour, and invariants that any ref-counted page pool must keep."""
import random

import pytest

from oracle.allocator import OutOfPages, PagePool


def test_block_manager_test_allocate_and_free(golden):
    g = golden("internals_block_manager_test.txt")
    m = PagePool(g["total_pages"], g["block_size"])
    pages = m.admit(1, g["num_tokens"])
    assert len(pages) == g["pages_allocated"]
    assert m.free_count() == g["free_after_allocate"]
    m.drop(1)
    assert m.free_count() == g["free_after_free"]


def test_allocator_simulation_42_tokens(golden):
    g = golden("glossary_allocator_simulation.txt")
    m = PagePool(g["total_pages"], g["block_size"])
    assert len(m.admit(0, g["num_tokens"])) == g["pages_allocated"]
    assert m.free_count() == g["total_pages"] - g["pages_allocated"]


@pytest.mark.parametrize("fixture", ["glossary_36_token_diagram.txt", "internals_block_table_flowchart.txt"])
def test_translation_matches_printed_tables(golden, fixture):
    g = golden(fixture)
    table = [page for _, _, _, page in g["blocks"]]
    total = max(table) + 5
    # Put the printed pages at the front of the pool so allocation reproduces the table.
    order = table + [p for p in range(total) if p not in table]
    m = PagePool(total, g["block_size"], order)
    assert m.admit(0, g["num_tokens"]) == table
    for _, first, last, page in g["blocks"]:
        for tok in range(first, last + 1):
            slot = m.slot(0, tok)
            assert slot // g["block_size"] == page
            assert slot % g["block_size"] == tok - first


def test_pages_leave_front_and_return_to_back():
    # The listing takes pages with pop(0) and returns freed pages with append, in table order.
    m = PagePool(10, 16)
    assert m.admit("a", 32) == [0, 1]
    assert m.admit("b", 33) == [2, 3, 4]
    m.drop("a")
    assert list(m.pool) == [5, 6, 7, 8, 9, 0, 1]
    assert m.admit("c", 80) == [5, 6, 7, 8, 9]
    assert m.admit("d", 17) == [0, 1]


def test_out_of_pages_is_all_or_nothing():
    m = PagePool(5, 16)
    m.admit(0, 40)
    before = m.state()
    with pytest.raises(MemoryError):
        m.admit(1, 16 * 3)
    assert m.state() == before
    m.admit(1, 16 * 2)
    assert m.free_count() == 0
    with pytest.raises(OutOfPages):
        for _ in range(100):
            m.extend(1)
    # the failing append changed nothing: sequence 1 is full at 32 tokens
    assert m.lengths[1] == 32 and m.free_count() == 0


def test_free_unknown_sequence_is_noop():
    m = PagePool(4, 16)
    m.admit(0, 20)
    before = m.state()
    m.drop(12345)
    assert m.state() == before


@pytest.mark.parametrize("bs", [2, 3, 16, 32])
def test_append_takes_page_exactly_when_listing_says(bs):
    """Growing by one token takes a page iff the count after the append is 1 mod bs (bs > 1)."""
    m = PagePool(1000, bs)
    m.admit(0, 0)
    for count_after in range(1, 10 * bs):
        before = len(m.tables[0])
        m.extend(0)
        took = len(m.tables[0]) - before
        assert took == (1 if count_after % bs == 1 else 0), count_after


def test_append_block_size_one_takes_page_every_token():
    m = PagePool(10, 1)
    m.admit(0, 0)
    for i in range(10):
        slot, pair = m.extend(0)
        assert pair is None and len(m.tables[0]) == i + 1 and slot == i


def test_append_slots_follow_table():
    m = PagePool(8, 4, [5, 2, 7, 0, 1, 3, 4, 6])
    m.admit(0, 3)          # page 5
    slots = [m.extend(0)[0] for _ in range(6)]
    # positions 3..8: page 5 offset 3, then page 2 offsets 0..3, then page 7 offset 0
    assert slots == [5 * 4 + 3, 2 * 4 + 0, 2 * 4 + 1, 2 * 4 + 2, 2 * 4 + 3, 7 * 4 + 0]


def test_fork_shares_pages_and_counts_references():
    m = PagePool(20, 16)
    parent = m.admit(0, 40)
    for c in range(1, 4):
        m.share(0, c)
    assert all(m.tables[c] == parent for c in range(4))
    assert all(m.holders[p] == 4 for p in parent)
    assert m.free_count() == 20 - 3
    # free the parent: pages stay allocated while children hold them
    m.drop(0)
    assert all(m.holders[p] == 3 for p in parent) and m.free_count() == 17
    for c in range(1, 4):
        m.drop(c)
    assert m.free_count() == 20 and all(r == 0 for r in m.holders)


def test_copy_on_write_last_holder_writes_in_place():
    # 100 sequences share a prefix whose last page is half full: 99 copies.
    bs = 32
    m = PagePool(313 + 99, bs)
    prefix = m.admit(0, 10_000)
    assert len(prefix) == 313
    last = prefix[-1]
    for c in range(1, 100):
        m.share(0, c)
    pairs = []
    for s in range(100):
        slot, pair = m.extend(s)
        if pair is not None:
            pairs.append(pair)
            assert pair[0] == last and m.tables[s][-1] == pair[1]
        assert slot == m.tables[s][-1] * bs + 10_000 % bs
    assert len(pairs) == 99
    assert m.tables[99][-1] == last           # the last writer kept the shared page
    assert m.holders[last] == 1
    assert len({p for _, p in pairs}) == 99          # all copies distinct
    assert m.free_count() == 0                         # exactly 313 + 99 pages used
    assert all(m.holders[p] == 100 for p in prefix[:-1])
    # the shared full pages were never copied
    assert all(m.tables[s][:-1] == prefix[:-1] for s in range(100))


def test_copy_on_write_not_needed_when_new_token_starts_block():
    m = PagePool(10, 16)
    m.admit(0, 32)
    m.share(0, 1)
    slot, pair = m.extend(1)
    assert pair is None and len(m.tables[1]) == 3
    assert m.tables[1][:2] == m.tables[0]


def _check_invariants(m):
    held = [p for t in m.tables.values() for p in t]
    for page in range(m.num_pages):
        assert m.holders[page] == held.count(page)
    assert set(m.pool).isdisjoint(held)
    assert len(m.pool) + len(set(held)) == m.num_pages
    assert len(set(m.pool)) == len(m.pool)
    for s, t in m.tables.items():
        assert len(t) == -(-m.lengths[s] // m.block_size)


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_keep_invariants(seed):
    rnd = random.Random(seed)
    bs = rnd.choice([1, 2, 4, 16])
    m = PagePool(64, bs, rnd.sample(range(64), 64))
    next_id = 0
    for _ in range(400):
        op = rnd.random()
        live = list(m.tables)
        try:
            if op < 0.25 or not live:
                m.admit(next_id, rnd.randint(0, 3 * bs))
                next_id += 1
            elif op < 0.45:
                m.share(rnd.choice(live), next_id)
                next_id += 1
            elif op < 0.85:
                m.extend(rnd.choice(live))
            else:
                m.drop(rnd.choice(live))
        except MemoryError:
            pass
        _check_invariants(m)

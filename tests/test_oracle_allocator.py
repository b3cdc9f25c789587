"""Pins of oracle/allocator.py: the pages' worked examples, the listing's stated
behaviour, and invariants that any ref-counted page pool must keep."""
import random

import pytest

from oracle.allocator import OutOfPages, PagedBlockManager


def test_block_manager_test_allocate_and_free(golden):
    g = golden("internals_block_manager_test.txt")
    m = PagedBlockManager(g["total_pages"], g["block_size"])
    pages = m.allocate_sequence(1, g["num_tokens"])
    assert len(pages) == g["pages_allocated"]
    assert m.num_free() == g["free_after_allocate"]
    m.free_sequence(1)
    assert m.num_free() == g["free_after_free"]


def test_allocator_simulation_42_tokens(golden):
    g = golden("glossary_allocator_simulation.txt")
    m = PagedBlockManager(g["total_pages"], g["block_size"])
    assert len(m.allocate_sequence(0, g["num_tokens"])) == g["pages_allocated"]
    assert m.num_free() == g["total_pages"] - g["pages_allocated"]


@pytest.mark.parametrize("fixture", ["glossary_36_token_diagram.txt", "internals_block_table_flowchart.txt"])
def test_translation_matches_printed_tables(golden, fixture):
    g = golden(fixture)
    table = [page for _, _, _, page in g["blocks"]]
    total = max(table) + 5
    # Put the printed pages at the front of the pool so allocation reproduces the table.
    order = table + [p for p in range(total) if p not in table]
    m = PagedBlockManager(total, g["block_size"], order)
    assert m.allocate_sequence(0, g["num_tokens"]) == table
    for _, first, last, page in g["blocks"]:
        for tok in range(first, last + 1):
            slot = m.slot(0, tok)
            assert slot // g["block_size"] == page
            assert slot % g["block_size"] == tok - first


def test_pages_leave_front_and_return_to_back():
    # The listing takes pages with pop(0) and returns freed pages with append, in table order.
    m = PagedBlockManager(10, 16)
    assert m.allocate_sequence("a", 32) == [0, 1]
    assert m.allocate_sequence("b", 33) == [2, 3, 4]
    m.free_sequence("a")
    assert list(m.free_pool) == [5, 6, 7, 8, 9, 0, 1]
    assert m.allocate_sequence("c", 80) == [5, 6, 7, 8, 9]
    assert m.allocate_sequence("d", 17) == [0, 1]


def test_out_of_pages_is_all_or_nothing():
    m = PagedBlockManager(5, 16)
    m.allocate_sequence(0, 40)
    before = m.state()
    with pytest.raises(MemoryError):
        m.allocate_sequence(1, 16 * 3)
    assert m.state() == before
    m.allocate_sequence(1, 16 * 2)
    assert m.num_free() == 0
    with pytest.raises(OutOfPages):
        for _ in range(100):
            m.append_token(1)
    # the failing append changed nothing: sequence 1 is full at 32 tokens
    assert m.num_tokens[1] == 32 and m.num_free() == 0


def test_free_unknown_sequence_is_noop():
    m = PagedBlockManager(4, 16)
    m.allocate_sequence(0, 20)
    before = m.state()
    m.free_sequence(12345)
    assert m.state() == before


@pytest.mark.parametrize("bs", [2, 3, 16, 32])
def test_append_takes_page_exactly_when_listing_says(bs):
    """append_token takes a page iff the count after the append is 1 mod bs (bs > 1)."""
    m = PagedBlockManager(1000, bs)
    m.allocate_sequence(0, 0)
    for count_after in range(1, 10 * bs):
        before = len(m.block_tables[0])
        m.append_token(0)
        took = len(m.block_tables[0]) - before
        assert took == (1 if count_after % bs == 1 else 0), count_after


def test_append_block_size_one_takes_page_every_token():
    m = PagedBlockManager(10, 1)
    m.allocate_sequence(0, 0)
    for i in range(10):
        slot, pair = m.append_token(0)
        assert pair is None and len(m.block_tables[0]) == i + 1 and slot == i


def test_append_slots_follow_table():
    m = PagedBlockManager(8, 4, [5, 2, 7, 0, 1, 3, 4, 6])
    m.allocate_sequence(0, 3)          # page 5
    slots = [m.append_token(0)[0] for _ in range(6)]
    # positions 3..8: page 5 offset 3, then page 2 offsets 0..3, then page 7 offset 0
    assert slots == [5 * 4 + 3, 2 * 4 + 0, 2 * 4 + 1, 2 * 4 + 2, 2 * 4 + 3, 7 * 4 + 0]


def test_fork_shares_pages_and_counts_references():
    m = PagedBlockManager(20, 16)
    parent = m.allocate_sequence(0, 40)
    for c in range(1, 4):
        m.fork(0, c)
    assert all(m.block_tables[c] == parent for c in range(4))
    assert all(m.ref_count[p] == 4 for p in parent)
    assert m.num_free() == 20 - 3
    # free the parent: pages stay allocated while children hold them
    m.free_sequence(0)
    assert all(m.ref_count[p] == 3 for p in parent) and m.num_free() == 17
    for c in range(1, 4):
        m.free_sequence(c)
    assert m.num_free() == 20 and all(r == 0 for r in m.ref_count)


def test_copy_on_write_last_holder_writes_in_place():
    # 100 sequences share a prefix whose last page is half full: 99 copies.
    bs = 32
    m = PagedBlockManager(313 + 99, bs)
    prefix = m.allocate_sequence(0, 10_000)
    assert len(prefix) == 313
    last = prefix[-1]
    for c in range(1, 100):
        m.fork(0, c)
    pairs = []
    for s in range(100):
        slot, pair = m.append_token(s)
        if pair is not None:
            pairs.append(pair)
            assert pair[0] == last and m.block_tables[s][-1] == pair[1]
        assert slot == m.block_tables[s][-1] * bs + 10_000 % bs
    assert len(pairs) == 99
    assert m.block_tables[99][-1] == last           # the last writer kept the shared page
    assert m.ref_count[last] == 1
    assert len({p for _, p in pairs}) == 99          # all copies distinct
    assert m.num_free() == 0                         # exactly 313 + 99 pages used
    assert all(m.ref_count[p] == 100 for p in prefix[:-1])
    # the shared full pages were never copied
    assert all(m.block_tables[s][:-1] == prefix[:-1] for s in range(100))


def test_copy_on_write_not_needed_when_new_token_starts_block():
    m = PagedBlockManager(10, 16)
    m.allocate_sequence(0, 32)
    m.fork(0, 1)
    slot, pair = m.append_token(1)
    assert pair is None and len(m.block_tables[1]) == 3
    assert m.block_tables[1][:2] == m.block_tables[0]


def _check_invariants(m):
    held = [p for t in m.block_tables.values() for p in t]
    for page in range(m.total_pages):
        assert m.ref_count[page] == held.count(page)
    assert set(m.free_pool).isdisjoint(held)
    assert len(m.free_pool) + len(set(held)) == m.total_pages
    assert len(set(m.free_pool)) == len(m.free_pool)
    for s, t in m.block_tables.items():
        assert len(t) == -(-m.num_tokens[s] // m.block_size)


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_keep_invariants(seed):
    rnd = random.Random(seed)
    bs = rnd.choice([1, 2, 4, 16])
    m = PagedBlockManager(64, bs, rnd.sample(range(64), 64))
    next_id = 0
    for _ in range(400):
        op = rnd.random()
        live = list(m.block_tables)
        try:
            if op < 0.25 or not live:
                m.allocate_sequence(next_id, rnd.randint(0, 3 * bs))
                next_id += 1
            elif op < 0.45:
                m.fork(rnd.choice(live), next_id)
                next_id += 1
            elif op < 0.85:
                m.append_token(rnd.choice(live))
            else:
                m.free_sequence(rnd.choice(live))
        except MemoryError:
            pass
        _check_invariants(m)

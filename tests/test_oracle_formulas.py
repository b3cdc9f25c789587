"""Pins of oracle/formulas.py against numbers the pages print (tests/golden)."""
import pytest

from oracle import formulas


def test_36_token_diagram_blocks(golden):
    g = golden("glossary_36_token_diagram.txt")
    ranges = formulas.logical_blocks(g["num_tokens"], g["block_size"])
    assert ranges == [(first, last) for _, first, last, _ in g["blocks"]]


def test_flowchart_blocks(golden):
    g = golden("internals_block_table_flowchart.txt")
    ranges = formulas.logical_blocks(g["num_tokens"], g["block_size"])
    assert ranges == [(first, last) for _, first, last, _ in g["blocks"]]


def test_42_tokens_take_3_pages(golden):
    g = golden("glossary_allocator_simulation.txt")
    n = formulas.blocks_needed(g["num_tokens"], g["block_size"])
    assert n == g["pages_allocated"]
    assert n * g["block_size"] == g["token_capacity"]


def test_32_tokens_take_2_pages(golden):
    g = golden("internals_block_manager_test.txt")
    assert formulas.blocks_needed(g["num_tokens"], g["block_size"]) == g["pages_allocated"]


def test_kv_bytes_llama3_70b(golden):
    g = golden("internals_kv_bytes.txt")
    per_token = formulas.kv_bytes_per_token(g["num_layers"], g["num_kv_heads"], g["head_dim"],
                                            g["bytes_per_elem"])
    assert per_token == g["bytes_per_token"]
    assert per_token / 1024 == g["kib_per_token"]
    reserved = per_token * g["reserved_tokens"]
    assert reserved == 1_342_177_280
    # The page's "1.31 GB" and "1.15 GB" are these byte counts in units of 1.024e9 bytes.
    assert round(reserved / 1.024e9, 2) == g["reported_gb_reserved"]
    wasted = per_token * (g["reserved_tokens"] - g["used_tokens"])
    assert round(wasted / 1.024e9, 2) == g["reported_gb_wasted"]


def test_internal_waste_87_5_percent(golden):
    g = golden("internals_kv_bytes.txt")
    w = formulas.internal_waste_fraction(g["reserved_tokens"], g["used_tokens"])
    assert w * 100 == g["waste_percent"]


def test_kv_bytes_each_factor_matters():
    base = formulas.kv_bytes_per_token(80, 8, 128, 2)
    # doubling any one factor doubles the result: no factor dropped or squared
    assert formulas.kv_bytes_per_token(160, 8, 128, 2) == 2 * base
    assert formulas.kv_bytes_per_token(80, 16, 128, 2) == 2 * base
    assert formulas.kv_bytes_per_token(80, 8, 256, 2) == 2 * base
    assert formulas.kv_bytes_per_token(80, 8, 128, 4) == 2 * base
    # one layer, one head, one dim, one byte: K and V
    assert formulas.kv_bytes_per_token(1, 1, 1, 1) == 2


@pytest.mark.parametrize("bs", [1, 2, 3, 16, 32])
def test_blocks_needed_brute_force(bs):
    for n in range(0, 200):
        # brute force: count distinct block indices of positions 0..n-1
        assert formulas.blocks_needed(n, bs) == len({p // bs for p in range(n)})
        assert formulas.paged_waste_slots(n, bs) == formulas.blocks_needed(n, bs) * bs - n
        assert 0 <= formulas.paged_waste_slots(n, bs) <= bs - 1


def test_36_token_waste():
    # 36 tokens in 3 pages of 16 leave 12 slots of the last page free.
    assert formulas.paged_waste_slots(36, 16) == 12


def test_logical_blocks_cover_every_token_once():
    for bs in (1, 4, 16, 32):
        for n in (0, 1, bs - 1, bs, bs + 1, 5 * bs + 3):
            if n < 0:
                continue
            covered = [t for first, last in formulas.logical_blocks(n, bs) for t in range(first, last + 1)]
            assert covered == list(range(n))

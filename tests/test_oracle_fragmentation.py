"""Pins of oracle/fragmentation.py: the pages' worked numbers, closed forms and
a brute-force count of occupied slots; planted mistakes must fail them."""
import numpy as np
import pytest

from oracle import formulas, fragmentation
from oracle.allocator import PagePool


def _stats(mgr, alarm=fragmentation.LOW_FREE_FRACTION):
    return fragmentation.pool_stats(mgr.state(), mgr.num_pages, mgr.block_size, alarm)


def test_one_sequence_of_36_tokens_wastes_12_of_48_slots():
    """Glossary, "Technical Architecture": 36 tokens in 16-token pages hold 3 pages, 12 slots free."""
    mgr = PagePool(16, 16)
    mgr.admit(0, 36)
    st = _stats(mgr)
    assert (st["used_pages"], st["physical_tokens"], st["waste_slots"]) == (3, 36, 12)
    assert st["waste_fraction"] == 12 / 48
    assert st["free_pages"] == 13 and st["free_fraction"] == 13 / 16 and not st["low_free_alarm"]


@pytest.mark.parametrize("bs", [1, 2, 7, 16, 32])
def test_independent_sequences_waste_their_last_pages(bs):
    rng = np.random.default_rng(bs)
    lens = [int(x) for x in rng.integers(0, 300, size=12)]
    mgr = PagePool(sum(formulas.blocks_needed(n, bs) for n in lens) + 5, bs)
    for s, n in enumerate(lens):
        mgr.admit(s, n)
    st = _stats(mgr)
    assert st["waste_slots"] == sum(formulas.paged_waste_slots(n, bs) for n in lens)
    assert st["logical_tokens"] == st["physical_tokens"] == sum(lens)
    assert st["shared_pages"] == 0


def test_a_fork_shares_its_pages_and_copy_on_write_splits_one():
    mgr = PagePool(16, 16)
    mgr.admit(0, 36)
    mgr.share(0, 1)
    st = _stats(mgr)
    assert (st["used_pages"], st["shared_pages"], st["logical_tokens"], st["physical_tokens"]) == (3, 3, 72, 36)
    mgr.extend(1)                     # writes into the shared last page: copy-on-write
    st = _stats(mgr)
    # pages 0-1 shared (32 tokens once), parent's last page 4 tokens, the child's copy 5
    assert (st["used_pages"], st["shared_pages"], st["physical_tokens"], st["waste_slots"]) == (4, 2, 41, 64 - 41)


def test_the_alarm_fires_below_ten_percent_free():
    """Internals, "Architectural Recommendations", item 3: alert under 10 percent free pages."""
    mgr = PagePool(20, 4)
    mgr.admit(0, 4 * 18)        # 2 of 20 free: exactly 10 percent, no alarm
    assert not _stats(mgr)["low_free_alarm"]
    mgr.admit(1, 1)             # 1 of 20 free
    assert _stats(mgr)["low_free_alarm"]
    mgr.drop(0)
    assert not _stats(mgr)["low_free_alarm"]
    assert _stats(mgr, alarm=0.99)["low_free_alarm"]


def test_empty_pool_and_empty_state():
    st = _stats(PagePool(0, 16))
    assert st["free_fraction"] == 0.0 and st["waste_fraction"] == 0.0 and not st["low_free_alarm"]
    st = _stats(PagePool(8, 16))
    assert (st["used_pages"], st["waste_slots"], st["free_fraction"]) == (0, 0, 1.0)


def _random_manager(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([2, 4, 16]))
    mgr = PagePool(400, bs, rng.permutation(400))
    live = []
    for step in range(120):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                s = step
                mgr.admit(s, int(rng.integers(0, 40)))
                live.append(s)
            elif op == 1:
                mgr.share(int(rng.choice(live)), 1000 + step)
                live.append(1000 + step)
            elif op == 2:
                for _ in range(int(rng.integers(1, 6))):
                    mgr.extend(int(rng.choice(live)))
            else:
                s = int(rng.choice(live))
                mgr.drop(s)
                live.remove(s)
        except MemoryError:
            pass
    return mgr


def _brute_physical(mgr):
    """Occupied slots counted one by one: every position of every sequence marks its slot."""
    return len({mgr.slot(s, p) for s in mgr.tables for p in range(mgr.lengths[s])})


@pytest.mark.parametrize("seed", range(6))
def test_physical_tokens_match_a_slot_by_slot_count(seed):
    mgr = _random_manager(seed)
    st = _stats(mgr)
    assert st["physical_tokens"] == _brute_physical(mgr)
    assert st["used_pages"] == mgr.num_pages - mgr.free_count()
    assert st["waste_slots"] == st["used_pages"] * mgr.block_size - _brute_physical(mgr)
    assert st["logical_tokens"] == sum(mgr.lengths.values())


def _fills_summed(state, bs):
    """Mistake: a shared page's fill summed over its holders."""
    out = {}
    for seq, table in state["block_tables"].items():
        for i, page in enumerate(table):
            out[page] = out.get(page, 0) + min(bs, state["num_tokens"][seq] - i * bs)
    return sum(out.values())


@pytest.mark.parametrize("mutant", [_fills_summed])
def test_planted_mistakes_are_caught(monkeypatch, mutant):
    """A plausible mistake in the fill of shared pages fails the slot-by-slot pin, on states with forks.
    (Every holder of a shared page has the same fill in it, since a write into a shared page copies it
    first, so taking any one holder's fill is not a mistake; counting it per holder is.)"""
    caught = 0
    for seed in range(6):
        mgr = _random_manager(seed)
        if mutant(mgr.state(), mgr.block_size) != _brute_physical(mgr):
            caught += 1
    assert caught > 0

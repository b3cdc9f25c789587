"""The oracle trace runner and the workload generator, checked on the CPU.

The runner is pinned by the pages' sharing rules: a forked sequence sees its
parent's prefix; after copy-on-write every sequence reads exactly its own
tokens (nobody sees another's tail) and the pages it did not write are
untouched; reference counts add up.  The generator is checked for
determinism, sub-range regeneration and the stated length / value
distributions.
"""
import math

import numpy as np
import pytest

from oracle import attention, scenario
from paged_kv_cache_356_b200 import workloads


def _seq_rows_match_lineage(w, res):
    for b in range(w.num_seqs):
        ctx = int(res["context_lens"][b])
        table = res["block_tables"][b]
        k_ref, v_ref = w.sequence_kv(b)
        np.testing.assert_array_equal(attention.gather_sequence(res["key_cache"], table, ctx), k_ref)
        np.testing.assert_array_equal(attention.gather_sequence(res["value_cache"], table, ctx), v_ref)


def test_tiny_scenario():
    w = workloads.tiny()
    res = scenario.run(w)
    assert list(res["context_lens"]) == [36, 42]
    # 36 tokens -> 3 pages, 42 tokens -> 3 pages, out of a pool of 16
    assert [len(t) for t in res["state"]["block_tables"].values()] == [3, 3]
    assert len(res["state"]["free_pool"]) == 10
    _seq_rows_match_lineage(w, res)
    assert res["out"].shape == (2, 4, 64)
    # the pool order is the seeded permutation: tables are its first six entries
    order = w.initial_free_order().tolist()
    tables = res["state"]["block_tables"]
    assert sorted(tables[0] + tables[1]) == sorted(order[:6])


def test_prefix_scenario_copy_on_write():
    w = workloads.prefix(num_seqs=5, prefix_len=70, max_tail=40)
    res = scenario.run(w)
    # the prefix ends mid-page (70 % 32 = 6), so all but the last writer copy it
    assert len(res["cow_pairs"]) == 4
    assert len({src for src, _ in res["cow_pairs"]}) == 1
    _seq_rows_match_lineage(w, res)
    st = res["state"]
    held = [p for t in st["block_tables"].values() for p in t]
    assert all(st["ref_count"][p] == held.count(p) for p in range(w.num_blocks))
    # the two full prefix pages are still shared by all five sequences
    first_two = st["block_tables"][0][:2]
    assert all(st["block_tables"][b][:2] == first_two for b in range(5))
    assert all(st["ref_count"][p] == 5 for p in first_two)


def test_beam_scenario_no_copy_when_prompt_fills_pages():
    w = workloads.beam32k(num_beams=3, prompt_len=64, own=20)
    res = scenario.run(w)
    assert res["cow_pairs"] == []
    _seq_rows_match_lineage(w, res)


def test_forked_child_matches_parent_before_divergence():
    w = workloads.prefix(num_seqs=3, prefix_len=50, max_tail=3)
    res = scenario.run(w, with_data=True)
    kc, vc = res["key_cache"], res["value_cache"]
    # decode every sequence over the shared prefix only, with one common query
    q = np.repeat(w.query()[:1], 3, axis=0)
    ctx = np.full(3, 50)
    out = attention.decode_attention(q, kc, vc, res["block_tables"], ctx, w.scale, w.dtype)
    np.testing.assert_array_equal(out[1], out[0])
    np.testing.assert_array_equal(out[2], out[0])


def test_allocator_only_run_matches_full_run():
    w = workloads.llama8b(num_seqs=6, lo=10, hi=90)
    a = scenario.run(w, with_data=False)
    b = scenario.run(w, with_data=True)
    assert a["state"] == b["state"]
    np.testing.assert_array_equal(a["write_slots"], b["write_slots"])
    np.testing.assert_array_equal(a["block_tables"], b["block_tables"])


# -- generator ---------------------------------------------------------------------------

def test_generator_is_deterministic_and_regenerates_subranges():
    w = workloads.llama8b(num_seqs=4, lo=20, hi=40)
    k1, v1 = w.token_kv(2, 0, 30)
    k2, v2 = w.token_kv(2, 0, 30)
    np.testing.assert_array_equal(k1, k2)
    np.testing.assert_array_equal(v1, v2)
    assert not np.array_equal(k1, v1)
    k3, _ = w.token_kv(3, 0, 30)
    assert not np.array_equal(k1, k3)
    np.testing.assert_array_equal(workloads.llama8b(num_seqs=4, lo=20, hi=40).query(), w.query())


def test_bf16_normal_moments():
    rng = np.random.default_rng(0)
    bits = workloads.normal_values(np.random.Generator(np.random.PCG64(5)), 2_000_000, "bf16")
    x = attention.to_float64(bits, "bf16")
    assert abs(x.mean()) < 3e-3 and abs(x.std() - 1.0) < 3e-3
    # about 68.27% within one sigma
    assert abs(np.mean(np.abs(x) < 1.0) - 0.6827) < 3e-3
    del rng


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5, 1.0 + 2 ** -9], dtype=np.float32)
    bits = workloads.float32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins; 1 + 3*2^-8 -> 1 + 2^-6
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xBFC0, 0x3F80]


def test_length_distributions():
    w2 = workloads.llama8b()
    assert w2.num_seqs == 64 and min(w2.context_lens) >= 128 and max(w2.context_lens) <= 4096
    w3 = workloads.llama70b()
    c = np.array(w3.context_lens)
    assert w3.num_seqs == 256 and c.min() >= 512 and c.max() <= 8192
    # log-uniform: the median sits near the geometric mean 2048
    assert 1400 < np.median(c) < 3000
    assert abs(c.mean() - 7680 / math.log(16)) < 400
    pages = sum(-(-x // 16) for x in c)
    assert w3.num_blocks == math.ceil(1.25 * pages)
    w4 = workloads.prefix()
    tails = np.array(w4.context_lens) - 10_000
    assert tails.min() >= 1 and tails.max() <= 512 and w4.block_size == 32
    w5 = workloads.beam32k()
    assert set(w5.context_lens) == {32_832} and w5.num_seqs == 8


@pytest.mark.parametrize("name", ["tiny", "llama8b", "llama70b", "prefix", "beam32k"])
def test_trace_positions_cover_context(name):
    w = workloads.by_name(name)
    for b in range(w.num_seqs):
        pos = 0
        for start, count, _, _ in w.segments(b):
            assert start == pos
            pos += count
        assert pos == w.context_lens[b]


@pytest.mark.parametrize("name", ["llama70b", "prefix", "beam32k"])
def test_full_size_allocator_runs(name):
    w = workloads.by_name(name)
    res = scenario.run(w, with_data=False)
    assert list(res["context_lens"]) == list(w.context_lens)
    if name == "prefix":
        assert len(res["cow_pairs"]) == 99
    else:
        assert res["cow_pairs"] == []

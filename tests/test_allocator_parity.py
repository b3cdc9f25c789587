"""The C++ pa_block_alloc against the oracle allocator: bit-exact state after
every operation of random op streams and of every workload trace (host only)."""
import random

import numpy as np
import pytest

from oracle import scenario
from oracle.allocator import PagePool
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads


def _state(a: pa.BlockAllocator, seqs, total):
    return {
        "free_pool": [int(p) for p in a.free_pool()],
        "ref_count": [a.ref_count(p) for p in range(total)],
        "block_tables": {s: [int(p) for p in a.block_table(s)] for s in sorted(seqs)},
        "num_tokens": {s: a.num_tokens(s) for s in sorted(seqs)},
    }


def test_block_manager_test_example(golden):
    g = golden("internals_block_manager_test.txt")
    a = pa.BlockAllocator(g["total_pages"], g["block_size"])
    a.allocate_sequence(1, g["num_tokens"])
    assert len(a.block_table(1)) == g["pages_allocated"] and a.num_free() == g["free_after_allocate"]
    a.free_sequence(1)
    assert a.num_free() == g["free_after_free"]


def test_errors_leave_state_unchanged():
    a = pa.BlockAllocator(5, 16)
    a.allocate_sequence(0, 40)
    before = _state(a, [0], 5)
    with pytest.raises(MemoryError):
        a.allocate_sequence(1, 48)
    with pytest.raises(pa.PagedAttentionError):
        a.allocate_sequence(0, 1)          # duplicate id
    with pytest.raises(KeyError):
        a.append_token(7)                   # unknown sequence
    with pytest.raises(KeyError):
        a.fork(9, 10)
    with pytest.raises(pa.PagedAttentionError):
        a.fork(0, 0)                        # child exists
    with pytest.raises(pa.PagedAttentionError):
        a.slot_mapping(0, 30, 20)           # beyond the sequence
    a.free_sequence(1234)                   # unknown: no-op
    assert _state(a, [0], 5) == before
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockAllocator(4, 16, [0, 1, 1, 2])   # not a permutation


def test_cow_without_output_pointers_is_rejected():
    import ctypes
    a = pa.BlockAllocator(8, 4)
    a.allocate_sequence(0, 3)
    a.fork(0, 1)
    slot = ctypes.c_int64()
    st = pa._lib.load().pa_block_alloc_append_token(a.handle, 1, ctypes.byref(slot), None, None)
    assert st == -1
    assert a.num_tokens(1) == 3 and a.num_free() == 7


def test_block_tables_export():
    a = pa.BlockAllocator(10, 4, [3, 1, 4, 0, 5, 9, 2, 6, 8, 7])
    a.allocate_sequence(10, 5)      # pages 3, 1
    a.allocate_sequence(20, 0)
    a.allocate_sequence(30, 9)      # pages 4, 0, 5
    tables, lens = a.block_tables([30, 10, 20], 4, pad=-7)
    assert tables.tolist() == [[4, 0, 5, -7], [3, 1, -7, -7], [-7, -7, -7, -7]]
    assert lens.tolist() == [9, 5, 0]
    with pytest.raises(pa.PagedAttentionError):
        a.block_tables([30], 2)
    assert a.slot_mapping(30, 3, 4).tolist() == [4 * 4 + 3, 0 * 4 + 0, 0 * 4 + 1, 0 * 4 + 2]


@pytest.mark.parametrize("seed", range(8))
def test_random_streams_match_oracle(seed):
    rnd = random.Random(seed)
    bs = rnd.choice([1, 2, 3, 4, 16, 32])
    total = rnd.choice([8, 33, 64])
    order = rnd.sample(range(total), total)
    ref = PagePool(total, bs, order)
    dut = pa.BlockAllocator(total, bs, order)
    live, next_id = [], 0
    for _ in range(500):
        op = rnd.random()
        ref_exc = dut_exc = None
        if op < 0.2 or not live:
            n = rnd.randint(0, 3 * bs + 1)
            try:
                ref.admit(next_id, n)
            except MemoryError as e:
                ref_exc = e
            try:
                dut.allocate_sequence(next_id, n)
            except MemoryError as e:
                dut_exc = e
            if ref_exc is None:
                live.append(next_id)
            next_id += 1
        elif op < 0.35:
            parent = rnd.choice(live)
            ref.share(parent, next_id)
            dut.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.85:
            s = rnd.choice(live)
            try:
                r = ref.extend(s)
            except MemoryError as e:
                ref_exc = e
            try:
                d = dut.append_token(s)
            except MemoryError as e:
                dut_exc = e
            if ref_exc is None and dut_exc is None:
                slot, pair = r
                assert d[0] == slot
                assert (d[1], d[2]) == (pair if pair is not None else (-1, -1))
        else:
            s = rnd.choice(live)
            ref.drop(s)
            dut.free_sequence(s)
            live.remove(s)
        assert (ref_exc is None) == (dut_exc is None)
        assert _state(dut, live, total) == ref.state() | {"block_tables": ref.state()["block_tables"]}


@pytest.mark.parametrize("name", ["tiny", "llama8b", "llama70b", "prefix", "beam32k"])
def test_workload_traces_match_oracle(name):
    """Run each workload's trace on both allocators (no device work) and compare."""
    w = workloads.by_name(name)
    ref = scenario.run(w, with_data=False)
    dut = pa.BlockAllocator(w.num_blocks, w.block_size, w.initial_free_order())
    pairs, slots = [], []
    for op in w.trace:
        if op[0] == "allocate":
            dut.allocate_sequence(op[1], op[2])
        elif op[0] == "fork":
            dut.fork(op[1], op[2])
        elif op[0] == "append":
            for _ in range(op[2]):
                _, src, dst = dut.append_token(op[1])
                if src >= 0:
                    pairs.append((src, dst))
        elif op[0] == "write":
            slots.append(dut.slot_mapping(op[1], op[2], op[3]))
    assert pairs == ref["cow_pairs"]
    np.testing.assert_array_equal(np.concatenate(slots), ref["write_slots"])
    assert _state(dut, range(w.num_seqs), w.num_blocks) == ref["state"]
    tables, lens = dut.block_tables(list(range(w.num_seqs)), w.max_blocks_per_seq, pad=-1)
    np.testing.assert_array_equal(tables, ref["block_tables"])
    np.testing.assert_array_equal(lens, ref["context_lens"])


# -- pool statistics ------------------------------------------------------------------------

def _random_ops(seed, total=300):
    """The same random op stream applied to the oracle and to the C allocator; yields after each op."""
    rng = random.Random(seed)
    bs = rng.choice([1, 3, 16, 32])
    order = list(range(total))
    rng.shuffle(order)
    ref = PagePool(total, bs, order)
    dut = pa.BlockAllocator(total, bs, np.array(order, dtype=np.int32))
    live, next_id = [], 0
    for _ in range(250):
        op = rng.randrange(4)
        try:
            if op == 0 or not live:
                n = rng.randrange(0, 70)
                ref.admit(next_id, n)
                dut.allocate_sequence(next_id, n)
                live.append(next_id)
                next_id += 1
            elif op == 1:
                parent = rng.choice(live)
                ref.share(parent, next_id)
                dut.fork(parent, next_id)
                live.append(next_id)
                next_id += 1
            elif op == 2:
                s = rng.choice(live)
                for _ in range(rng.randrange(1, 9)):
                    ref.extend(s)
                    dut.append_token(s)
            else:
                s = rng.choice(live)
                ref.drop(s)
                dut.free_sequence(s)
                live.remove(s)
        except MemoryError:
            pass
        yield ref, dut


@pytest.mark.parametrize("seed", range(5))
def test_pool_stats_match_the_oracle_after_every_op(seed):
    from oracle import fragmentation
    for ref, dut in _random_ops(seed):
        for alarm in (0.10, 0.5):
            want = fragmentation.pool_stats(ref.state(), ref.num_pages, ref.block_size, alarm)
            assert dut.stats(alarm) == want


@pytest.mark.parametrize("name", ["llama8b", "prefix", "beam32k"])
def test_pool_stats_of_workload_traces(name):
    from oracle import fragmentation
    w = workloads.by_name(name)
    ref = scenario.run(w, with_data=False)
    dut = pa.BlockAllocator(w.num_blocks, w.block_size, w.initial_free_order())
    for op in w.trace:
        if op[0] == "allocate":
            dut.allocate_sequence(op[1], op[2])
        elif op[0] == "fork":
            dut.fork(op[1], op[2])
        elif op[0] == "append":
            for _ in range(op[2]):
                dut.append_token(op[1])
    assert dut.stats() == fragmentation.pool_stats(ref["state"], w.num_blocks, w.block_size)


def test_pool_stats_rejects_null():
    assert pa._lib.load().pa_block_alloc_stats(None, 0.1, None) == pa._lib.PA_ERR_INVALID


# -- batched appends ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(4))
def test_batched_appends_equal_sequential_ones_in_the_oracle(seed):
    """pa_block_alloc_append_tokens over a batch = the oracle's append_token for each sequence in order:
    the same slots, copy-on-write pairs and state, through forks and shared partial pages."""
    rng = random.Random(seed)
    bs = rng.choice([1, 4, 16])
    total = 500
    order = list(range(total))
    rng.shuffle(order)
    ref = PagePool(total, bs, order)
    dut = pa.BlockAllocator(total, bs, np.array(order, dtype=np.int32))
    live = []
    for s in range(6):
        n = rng.randrange(0, 40)
        ref.admit(s, n)
        dut.allocate_sequence(s, n)
        live.append(s)
    for child in range(6, 12):
        parent = rng.choice(live)
        ref.share(parent, child)
        dut.fork(parent, child)
        live.append(child)
    for _ in range(30):
        batch = [rng.choice(live) for _ in range(rng.randrange(1, 12))]
        want = [ref.extend(s) for s in batch]
        slots, pairs = dut.append_tokens(batch)
        assert [int(x) for x in slots] == [w[0] for w in want]
        assert [tuple(int(v) for v in p) for p in pairs] == [w[1] if w[1] else (-1, -1) for w in want]
    assert _state(dut, live, total) == ref.state()


def test_batched_appends_stop_at_the_first_failure():
    import ctypes
    a = pa.BlockAllocator(3, 4)
    a.allocate_sequence(0, 4)        # one full page
    a.allocate_sequence(1, 3)        # one page, room for one more
    # 0 needs a page (1 left), 1 fits, 0 fits, 0 fits, 0 fits, then 0 needs a page: none left
    seqs = np.array([0, 1, 0, 0, 0, 0], dtype=np.int64)
    slots = np.empty(6, dtype=np.int64)
    src = np.empty(6, dtype=np.int32)
    dst = np.empty(6, dtype=np.int32)
    done = ctypes.c_int32()
    lib = pa._lib.load()
    st = lib.pa_block_alloc_append_tokens(a.handle, pa._i64p(seqs), 6, pa._i64p(slots), pa._i32p(src),
                                          pa._i32p(dst), ctypes.byref(done))
    assert st == pa._lib.PA_ERR_OOM and done.value == 5
    assert a.num_tokens(0) == 8 and a.num_tokens(1) == 4 and a.num_free() == 0
    with pytest.raises(MemoryError):
        a.append_tokens([1, 0])      # 1 needs a page: fails first, nothing changes
    assert a.num_tokens(1) == 4 and a.num_tokens(0) == 8
    assert lib.pa_block_alloc_append_tokens(a.handle, None, 1, None, None, None, None) == pa._lib.PA_ERR_INVALID

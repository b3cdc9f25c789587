"""pa_block_alloc_prefix_plan on the CPU: the plan only claims partitions that
every member of a chunk really shares, page for page, and leaves each
member's last token to the per-sequence kernel."""
import random

import numpy as np
import pytest

from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads

PART = 512


def _run_trace(w):
    a = pa.BlockAllocator(w.num_blocks, w.block_size, w.initial_free_order())
    for op in w.trace:
        if op[0] == "allocate":
            a.allocate_sequence(op[1], op[2])
        elif op[0] == "fork":
            a.fork(op[1], op[2])
        elif op[0] == "append":
            for _ in range(op[2]):
                a.append_token(op[1])
    return a


def _check_plan(a, seqs, group_size, plan):
    bs = a.block_size
    tables = [a.block_table(s) for s in seqs]
    tokens = [a.num_tokens(s) for s in seqs]
    per_chunk = max(1, 128 // group_size)
    seen = set()
    first = plan["first_partition"]
    for leader, off, count, sp in plan["chunks"][:plan["num_chunks"]]:
        assert 1 <= count <= per_chunk and sp >= 1
        mem = plan["members"][off:off + count]
        assert leader in set(plan["members"][:plan["num_members"]])
        shared_blocks = -(-sp * PART // bs)
        for i in mem:
            assert i not in seen
            seen.add(i)
            assert first[i] == sp
            # every shared partition lies in pages identical to the leader's
            assert list(tables[i][:shared_blocks]) == list(tables[leader][:shared_blocks])
            assert sp * PART <= tokens[i] - 1
    for i in range(len(seqs)):
        if i not in seen:
            assert first[i] == 0


@pytest.mark.parametrize("name,chunks,sp", [("prefix", 4, 19), ("beam32k", 1, 64), ("llama70b", 0, 0),
                                            ("tiny", 0, 0)])
def test_workload_plans(name, chunks, sp):
    w = workloads.by_name(name)
    a = _run_trace(w)
    seqs = list(range(w.num_seqs))
    plan = a.prefix_plan(seqs, w.group_size)
    assert plan["num_chunks"] == chunks and plan["max_shared_partitions"] == sp
    _check_plan(a, seqs, w.group_size, plan)


@pytest.mark.parametrize("seed", range(10))
def test_random_fork_trees(seed):
    rnd = random.Random(seed)
    bs = rnd.choice([16, 32, 64])
    a = pa.BlockAllocator(4000, bs, rnd.sample(range(4000), 4000))
    live = []
    for root in range(rnd.randint(1, 4)):
        sid = 1000 * root
        a.allocate_sequence(sid, rnd.randint(0, 3000))
        live.append(sid)
        for k in range(rnd.randint(0, 9)):
            child = sid + k + 1
            a.fork(rnd.choice([x for x in live if x // 1000 == root]), child)
            live.append(child)
    for s in live:
        for _ in range(rnd.randint(0, 700)):
            a.append_token(s)
    rnd.shuffle(live)
    g = rnd.choice([1, 2, 4, 8, 16])
    plan = a.prefix_plan(live, g)
    _check_plan(a, live, g, plan)


def test_plan_rejects_bad_arguments():
    a = pa.BlockAllocator(10, 16)
    a.allocate_sequence(0, 20)
    with pytest.raises(pa.PagedAttentionError):
        a.prefix_plan([0], 0)
    with pytest.raises(KeyError):
        a.prefix_plan([0, 5], 4)
    plan = a.prefix_plan([], 4)
    assert plan["num_chunks"] == 0

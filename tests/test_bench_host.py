"""Host-side pieces of bench.py that need no GPU: the partition kernel's source hash resolves its
anchors, the committed ncu summary parses and still matches the sources, and the byte accounting of a
decode step counts shared pages once."""
import os

import numpy as np

import bench
from paged_kv_cache_356_b200 import workloads


def test_kernel_hash_and_committed_traffic_are_consistent():
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    traffic, rec = bench.profiled_traffic("decode_tc_kernel llama70b", h)
    assert rec is not None and len(rec["kernel_source_sha256"]) == 16
    assert rec["summary"].startswith("profiles/") and os.path.exists(os.path.join(bench.ROOT, rec["summary"]))
    if rec["kernel_source_sha256"] == h:   # counters taken on these sources: a plausible DRAM figure
        assert traffic is not None and 0.9 < traffic / rec["algorithmic_bytes_per_launch"] < 1.1
    else:                                   # the kernel changed since: the bench must report no traffic
        assert traffic is None
    assert bench.profiled_traffic("no such kernel", h) == (None, None)


def test_configs_cover_every_workload_and_kernel():
    """The default run carries every other workload, both verification sizes and both copy kernels."""
    names = set(bench.EXTRA_CONFIGS)
    assert {"llama8b", "prefix", "beam32k", "micro", "verify4", "verify8"} <= names
    assert bench.parse_args([]).no_configs is False and bench.parse_args(["--no-configs"]).no_configs


def test_unique_and_logical_kv_bytes():
    w = workloads.beam32k(num_beams=3, prompt_len=64, own=16)
    bs = w.block_size
    # three sequences sharing 4 pages of prompt, each with one page of its own
    tables = np.array([[0, 1, 2, 3, 4], [0, 1, 2, 3, 5], [0, 1, 2, 3, 6]], dtype=np.int32)
    ctx = np.array([80, 80, 80], dtype=np.int32)
    unique, logical = bench.kv_bytes(w, tables, ctx)
    per_token = 2 * w.num_kv_heads * w.head_dim * w.elem_bytes
    assert unique == (4 * bs + 3 * 16) * per_token
    assert logical == 3 * 80 * per_token


def test_fragmentation_rows_match_the_oracle_and_the_pages_bound():
    """bench --fragmentation: the C allocator's statistics equal the oracle's for the same trace; for
    independent sequences the paged waste is far under the pages' "under 4 percent", the contiguous
    reservation's far above it."""
    from oracle import fragmentation, scenario
    from paged_kv_cache_356_b200 import workloads
    rows = bench.fragmentation_rows(names=("llama8b", "beam32k"), block_sizes=(16, 32))
    assert len(rows) == 4
    for r in rows:
        w = workloads.by_name(r["workload"], block_size=r["block_size"])
        ref = fragmentation.pool_stats(scenario.run(w, with_data=False)["state"], w.num_blocks, w.block_size)
        assert r["paged_waste_fraction"] == ref["waste_fraction"]
        assert r["physical_tokens"] == ref["physical_tokens"] and r["used_pages"] == ref["used_pages"]
        assert not r["low_free_alarm"]
        assert r["tight_low_free_alarm"] and 0.04 < r["tight_free_fraction"] < 0.06
    ind = [r for r in rows if r["workload"] == "llama8b"]
    assert all(r["paged_waste_fraction"] < 0.04 < r["contiguous_waste_fraction"] for r in ind)
    beam = [r for r in rows if r["workload"] == "beam32k"]
    assert all(r["shared_pages"] > 0 and r["contiguous_over_paged_slots"] > 5 for r in beam)


def test_call_bytes_count_inputs_and_outputs_once():
    """A whole call's algorithmic bytes: unique KV + q + the tables' used entries + lengths + every
    output row once, with T query tokens per sequence; the partition kernel's own figure adds the
    partials it writes (and writes the rows of one-partition sequences directly)."""
    w = workloads.tiny()                      # 2 sequences of 36 and 42 tokens, 4 q / 1 kv heads, D 64, fp32
    ctx = np.array(w.context_lens)
    unique = 1234
    eb, rows_per_seq = w.elem_bytes, w.num_q_heads
    tables = 4 * sum(-(-int(c) // w.block_size) for c in ctx)
    for T in (1, 3):
        want = unique + 2 * (2 * T * rows_per_seq * w.head_dim * eb) + tables + 4 * w.num_seqs
        assert bench.call_bytes(w, ctx, unique, T) == want
    # both sequences fit one partition: the partition kernel writes their rows, no partials
    assert bench.partition_kernel_bytes(w, ctx, unique) == bench.call_bytes(w, ctx, unique, 1)

"""The four full-size workloads through the C ABI, in the launch configuration the
benchmark times (AUTO kernel choice, default tiling).

Allocator state (free pool order, reference counts, tables), write slots and
copy-on-write pairs are compared bit for bit with the oracle allocator, which
is cheap at any size.  Attention is compared on sampled sequences: the oracle
evaluates textbook attention over each sampled sequence's tokens in position
order, regenerated from the seeded generator -- so the check covers the
allocator's slots, the cache writes, the page copies and the block-table
translation end to end.
"""
import numpy as np
import pytest

from oracle import attention, scenario
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner
from tests.parity import assert_decode_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sampled_reference(w, seqs, heads=None):
    q64 = attention.to_float64(w.query(), w.dtype)
    g = w.group_size
    heads = range(w.num_q_heads) if heads is None else heads
    ref = np.zeros((len(seqs), len(heads), w.head_dim))
    for i, b in enumerate(seqs):
        k, v = w.sequence_kv(b)
        k64, v64 = attention.to_float64(k, w.dtype), attention.to_float64(v, w.dtype)
        for j, h in enumerate(heads):
            ref[i, j] = attention.softmax_attention(q64[b, h], k64[:, h // g], v64[:, h // g], w.scale)
    return ref


@pytest.fixture(scope="module", params=["llama8b", "llama70b", "prefix", "beam32k", "prefix+shared",
                                        "beam32k+shared"])
def full_run(request):
    import torch
    pa.pa_set_decode_kernel(pa.PA_DECODE_AUTO)
    pa.pa_set_decode_tiling(4, 2)
    name, _, shared = request.param.partition("+")
    w = workloads.by_name(name)
    run = TraceRunner(w, shared_prefix=bool(shared))
    out = run.run()
    torch.cuda.synchronize()
    yield w, run, out
    del run
    torch.cuda.empty_cache()


def test_allocator_state_and_slots(full_run):
    w, run, _ = full_run
    ref = scenario.run(w, with_data=False)
    assert run.allocator_state() == ref["state"]
    assert run.cow_pairs == ref["cow_pairs"]
    np.testing.assert_array_equal(np.concatenate(run.write_slots), ref["write_slots"])
    assert run.status() == 0
    if w.name == "prefix":
        assert len(run.cow_pairs) == 99


def test_sampled_sequences_match_oracle(full_run):
    w, run, out = full_run
    ctx = np.array(w.context_lens)
    rng = np.random.default_rng(0)
    pick = sorted({int(np.argmax(ctx)), int(np.argmin(ctx)), *rng.choice(w.num_seqs, min(6, w.num_seqs), False)})
    heads = list(range(w.num_q_heads)) if w.num_seqs <= 8 else sorted(rng.choice(w.num_q_heads, 16, False))
    ref = _sampled_reference(w, pick, heads)
    got = out[pick][:, heads]
    assert_decode_close(got, ref, w.dtype, w.name)


def test_step_replay_is_idempotent(full_run):
    """The benchmark's step (the step's cache write, then decode) reproduces the output bit for bit."""
    import torch
    w, run, out = full_run
    first = out.clone()
    run.step()
    torch.cuda.synchronize()
    assert torch.equal(run.out.view(torch.int16), first.view(torch.int16))

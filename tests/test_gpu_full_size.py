"""The four full-size workloads through the C ABI, in the launch configuration the
benchmark times (AUTO kernel choice, default tiling).

Allocator state (free pool order, reference counts, tables), write slots and
copy-on-write pairs are compared bit for bit with the oracle allocator, which
is cheap at any size.  Attention is regenerated from the seeds rather than read
back from the device cache, so the check covers the allocator's slots, the
cache writes, the page copies and the block-table translation end to end.  Every sequence and every query head of each decode
workload is compared (the oracle's textbook attention over each sequence's
tokens in position order, regenerated from the seeded generator); the
verification step, T times the work, is compared on sampled sequences.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

from oracle import attention, scenario
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner
from tests.parity import assert_decode_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


_FULL_REFERENCE = {}


def _full_reference(w):
    """fp64 output of every sequence and query head: the oracle's textbook attention over each
    sequence's tokens in position order, regenerated from the seeds (sequences in parallel threads)."""
    if w.name in _FULL_REFERENCE:
        return _FULL_REFERENCE[w.name]
    q64 = attention.to_float64(w.query(), w.dtype)
    g = w.group_size
    ref = np.zeros((w.num_seqs, w.num_q_heads, w.head_dim))

    def one(b):
        k, v = w.sequence_kv(b)
        k64, v64 = attention.to_float64(k, w.dtype), attention.to_float64(v, w.dtype)
        for kvh in range(w.num_kv_heads):
            kh, vh = np.ascontiguousarray(k64[:, kvh]), np.ascontiguousarray(v64[:, kvh])
            for h in range(kvh * g, (kvh + 1) * g):
                ref[b, h] = attention.softmax_attention(q64[b, h], kh, vh, w.scale)

    with ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1))) as ex:
        list(ex.map(one, range(w.num_seqs)))
    _FULL_REFERENCE.clear()   # one workload's reference at a time (the plain and shared runs share it)
    _FULL_REFERENCE[w.name] = ref
    return ref


@pytest.fixture(scope="module", params=["llama8b", "llama70b", "prefix", "prefix+auto", "prefix+balanced",
                                        "prefix+items", "beam32k", "beam32k+auto", "beam32k+balanced",
                                        "beam32k+items"])
def full_run(request):
    """A workload's whole trace, then its decode step: plain pa_decode, or pa_decode_shared_prefix with
    the joint kernel AUTO picks, the balanced kernel or the per-partition kernel."""
    import torch
    pa.pa_set_decode_kernel(pa.PA_DECODE_AUTO)
    pa.pa_set_decode_tiling(4, 2)
    name, _, joint = request.param.partition("+")
    pa.pa_set_shared_prefix_kernel({"": pa.PA_SHARED_PREFIX_AUTO, "auto": pa.PA_SHARED_PREFIX_AUTO,
                                    "balanced": pa.PA_SHARED_PREFIX_TCGEN05,
                                    "items": pa.PA_SHARED_PREFIX_TCGEN05_ITEMS}[joint])
    w = workloads.by_name(name)
    run = TraceRunner(w, shared_prefix=bool(joint))
    out = run.run()
    torch.cuda.synchronize()
    yield w, run, out
    pa.pa_set_shared_prefix_kernel(pa.PA_SHARED_PREFIX_AUTO)
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


def test_every_sequence_and_head_matches_oracle(full_run):
    """The whole batch, element by element, within the decode tolerance (ragged page tails and the
    shortest and longest contexts included)."""
    w, run, out = full_run
    assert_decode_close(out, _full_reference(w), w.dtype, w.name)


def test_step_replay_is_idempotent(full_run):
    """The benchmark's step (the step's cache write, then decode) reproduces the output bit for bit."""
    import torch
    w, run, out = full_run
    first = out.clone()
    run.step()
    torch.cuda.synchronize()
    assert torch.equal(run.out.view(torch.int16), first.view(torch.int16))


# -- draft verification at full size (the bench's --verify-tokens step) ------------------------------

@pytest.fixture(scope="module", params=["llama8b", "llama70b"])
def verify_run(request):
    import torch
    pa.pa_set_decode_kernel(pa.PA_DECODE_AUTO)
    w = workloads.by_name(request.param)
    run = TraceRunner(w)
    run.run(decode=False)
    torch.cuda.synchronize()
    yield w, run
    del run
    torch.cuda.empty_cache()


@pytest.mark.parametrize("num_tokens", [4, 8])
def test_verify_step_on_sampled_sequences(verify_run, num_tokens):
    """Draft tokens written at each sequence's last T positions, then pa_decode_verify (auto path) as
    the bench times it; sampled rows against textbook causal attention over the sequence's tokens,
    regenerated from the seeds with the draft tokens' K/V in place."""
    import torch
    w, run = verify_run
    T = num_tokens
    ctx = np.array(w.context_lens)
    slots = np.concatenate([run.alloc.slot_mapping(b, int(ctx[b]) - T, T) for b in range(w.num_seqs)])
    dk, dv = w.draft_kv(T)
    q = w.draft_query(T)
    pages = torch.from_numpy(slots // w.block_size).cuda()
    offs = torch.from_numpy(slots % w.block_size).cuda()
    saved = run.key_cache[pages, :, offs, :].clone(), run.value_cache[pages, :, offs, :].clone()
    pa.pa_reshape_and_cache(run._to_device(dk), run._to_device(dv), torch.from_numpy(slots.astype(np.int64)).cuda(),
                            run.key_cache, run.value_cache)
    # NaN bytes in the workspace: a partial that no kernel wrote shows up in the sampled rows
    need = pa.pa_decode_verify_workspace_size(w.num_seqs, T, w.num_q_heads, w.head_dim,
                                              run.block_tables.shape[1] * w.block_size)
    ws = torch.full((max(need, 1),), 0xFF, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = pa.pa_decode_verify(run._to_device(q), run.key_cache, run.value_cache, run.block_tables,
                              run.context_lens, w.scale, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, f"device status {status.item():#x}"
    del ws
    # the trace's own K/V back in place for the next case
    run.key_cache[pages, :, offs, :] = saved[0]
    run.value_cache[pages, :, offs, :] = saved[1]
    assert run.status() == 0
    rng = np.random.default_rng(T)
    pick = sorted({int(np.argmax(ctx)), int(np.argmin(ctx)), *rng.choice(w.num_seqs, 4, False)})
    heads = sorted(rng.choice(w.num_q_heads, 8, False))
    q64 = attention.to_float64(q, w.dtype)
    g = w.group_size
    ref = np.zeros((len(pick), T, len(heads), w.head_dim))
    for i, b in enumerate(pick):
        k, v = w.sequence_kv(b)
        k, v = k.copy(), v.copy()
        k[-T:], v[-T:] = dk[b * T:(b + 1) * T], dv[b * T:(b + 1) * T]
        k64, v64 = attention.to_float64(k, w.dtype), attention.to_float64(v, w.dtype)
        for t in range(T):
            n = attention.visible_keys(int(ctx[b]), T, t)
            for j, h in enumerate(heads):
                ref[i, t, j] = attention.softmax_attention(q64[b, t, h], k64[:n, h // g], v64[:n, h // g], w.scale)
    assert_decode_close(out[pick][:, :, heads], ref, w.dtype, f"{w.name} T={T}")

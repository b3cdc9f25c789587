"""pa_decode_shared_prefix on the GPU: same results as the oracle (and hence as
pa_decode) while shared partitions are read once per group."""
import numpy as np
import pytest

from oracle import scenario
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner
from tests.parity import assert_decode_close, bits_of, host_bits

pytestmark = pytest.mark.gpu

# auto: the balanced kernel with the members' tails folded in (few, short tails), or on the shared
# lanes only with the per-sequence kernel on the tails (many or long tails)
JOINT = {"auto": pa.PA_SHARED_PREFIX_AUTO,
         "tcgen05": pa.PA_SHARED_PREFIX_TCGEN05, "tcgen05_items": pa.PA_SHARED_PREFIX_TCGEN05_ITEMS,
         "tcgen05_2cta": pa.PA_SHARED_PREFIX_TCGEN05_2CTA, "tcgen05_serial": pa.PA_SHARED_PREFIX_TCGEN05_SERIAL,
         "mma_sync": pa.PA_SHARED_PREFIX_MMA_SYNC}


@pytest.fixture(params=list(JOINT))
def joint(request):
    pa.pa_set_shared_prefix_kernel(JOINT[request.param])
    yield request.param
    pa.pa_set_shared_prefix_kernel(pa.PA_SHARED_PREFIX_AUTO)


@pytest.mark.parametrize("make", [
    lambda: workloads.prefix(num_seqs=5, prefix_len=1700, max_tail=90),
    lambda: workloads.prefix(num_seqs=40, prefix_len=1100, max_tail=600),          # G=4: 3 chunks of <= 16
    lambda: workloads.beam32k(num_beams=3, prompt_len=2100, own=40),
    lambda: workloads.beam32k(num_beams=8, prompt_len=1536, own=1),               # prompt = 3 whole partitions
], ids=["prefix-5", "prefix-40", "beam-3", "beam-8-exact"])
def test_shared_flows_match_oracle(make, joint):
    w = make()
    run = TraceRunner(w, shared_prefix=True)
    out = run.run()
    assert run.plan["num_chunks"] > 0
    ref = scenario.run(w)
    assert run.allocator_state() == ref["state"]
    np.testing.assert_array_equal(bits_of(run.key_cache), host_bits(ref["key_cache"]))
    assert run.status() == 0
    assert_decode_close(out, ref["out"], w.dtype, w.name)


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", [(8, 8, 128, 16, "bf16"), (16, 8, 128, 32, "bf16"),
                                               (64, 8, 64, 16, "bf16"), (32, 2, 128, 16, "bf16"),
                                               (64, 4, 128, 64, "bf16"), (128, 8, 128, 16, "bf16"),
                                               (32, 8, 64, 32, "bf16"), (32, 8, 128, 48, "bf16"),
                                               (64, 8, 128, 16, "f16"), (16, 4, 64, 32, "f16")])
def test_shared_shapes(hq, hkv, d, bs, dtype, joint):
    """G = 1, 2, 4, 8, 16 with head_dim 64 / 128, block sizes 16 to 64 (48: pages not aligned to
    partitions), bf16 and f16."""
    import math
    import torch
    from oracle import attention
    rng = np.random.Generator(np.random.PCG64(hq + hkv + d + bs))
    nseq, prompt = 6, 1600 + bs
    own = [int(x) for x in rng.integers(1, 700, size=nseq)]
    nb = -(-prompt // bs) + sum(-(-o // bs) + 1 for o in own) + 4
    a = pa.BlockAllocator(nb, bs, rng.permutation(nb))
    a.allocate_sequence(0, prompt)
    for s in range(1, nseq):
        a.fork(0, s)
    pairs = []
    for s in range(nseq):
        for _ in range(own[s]):
            _, src, dst = a.append_token(s)
            if src >= 0:
                pairs.append((src, dst))
    ctx = [prompt + o for o in own]
    mb = max(-(-c // bs) for c in ctx)
    tables, lens = a.block_tables(list(range(nseq)), mb, pad=-1)
    def values(n):
        if dtype == "f16":
            return rng.standard_normal(n, dtype=np.float32).astype(np.float16).view(np.uint16)
        return workloads.normal_values(rng, n, "bf16")
    kc = values(nb * hkv * bs * d).reshape(nb, hkv, bs, d)
    vc = values(nb * hkv * bs * d).reshape(nb, hkv, bs, d)
    q = values(nseq * hq * d).reshape(nseq, hq, d)
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(tdt).cuda()  # noqa
    plan = pa.prefix_plan_to_device(a.prefix_plan(list(range(nseq)), hq // hkv))
    assert plan["num_chunks"] >= 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # NaN bytes in the workspace: a partial that no kernel wrote cannot pass for a stale one
    ws = torch.full((max(pa.pa_decode_workspace_size(nseq, hq, d, mb * bs), 256),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    out = pa.pa_decode_shared_prefix(dev(q), dev(kc), dev(vc), torch.from_numpy(tables).cuda(),
                                     torch.from_numpy(lens).cuda(), 1 / math.sqrt(d), plan, workspace=ws,
                                     dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = attention.decode_attention(q, kc, vc, tables, lens, 1 / math.sqrt(d), dtype)
    assert_decode_close(out, ref, dtype, f"shared {dtype} hq{hq} hkv{hkv} d{d} bs{bs}")


def test_bad_plan_entries_are_skipped_and_flagged(joint):
    """Out-of-range leader / member ranges / partitions are flagged, never dereferenced."""
    import math
    import torch
    w = workloads.beam32k(num_beams=3, prompt_len=1100, own=40)
    run = TraceRunner(w, shared_prefix=True)
    run.run(decode=False)
    plan = dict(run.plan)
    bad = torch.tensor([[w.num_seqs + 5, 0, 3, 2],      # leader outside the batch
                        [0, 1, 9, 2],                   # members past the array
                        [0, 0, 3, 40000]],              # partitions past the table
                       dtype=torch.int32, device="cuda")
    plan["chunks"], plan["num_chunks"] = bad, 3
    plan["max_shared_partitions"] = 3
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(run.q, run.key_cache, run.value_cache, run.block_tables, run.context_lens,
                               1 / math.sqrt(w.head_dim), plan, out=run.out, workspace=run.workspace,
                               dev_status=status)
    torch.cuda.synchronize()
    assert status.item() & pa.PA_DEV_BAD_PLAN


def test_wait_that_runs_out_reports_timeout_and_the_context_stays_usable():
    """Failure path of the tcgen05 joint kernel: with the first work item's hand-off withheld (test hook),
    the other roles' bounded waits run out after about a second; the call completes with PA_DEV_TIMEOUT
    instead of hanging, and the next ordinary call on the same context gives the oracle's result."""
    import math
    import time
    import torch
    pa.pa_set_shared_prefix_kernel(pa.PA_SHARED_PREFIX_TCGEN05)
    w = workloads.beam32k(num_beams=3, prompt_len=2100, own=40)
    run = TraceRunner(w, shared_prefix=True)
    run.run(decode=False)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        pa.pa_set_fault_injection(pa.PA_FAULT_WITHHOLD_FIRST_ITEM)
        t0 = time.perf_counter()
        pa.pa_decode_shared_prefix(run.q, run.key_cache, run.value_cache, run.block_tables, run.context_lens,
                                   1 / math.sqrt(w.head_dim), run.plan, out=run.out, workspace=run.workspace,
                                   dev_status=status)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        pa.pa_set_fault_injection(pa.PA_FAULT_NONE)
        pa.pa_set_shared_prefix_kernel(pa.PA_SHARED_PREFIX_AUTO)
    assert status.item() & pa.PA_DEV_TIMEOUT
    assert 0.2 < elapsed < 30
    status.zero_()
    out = pa.pa_decode_shared_prefix(run.q, run.key_cache, run.value_cache, run.block_tables, run.context_lens,
                                     1 / math.sqrt(w.head_dim), run.plan, out=run.out, workspace=run.workspace,
                                     dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert_decode_close(out, scenario.run(w)["out"], w.dtype, "after a timed-out call")


def test_fault_injection_rejects_unknown_modes():
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_set_fault_injection(7)

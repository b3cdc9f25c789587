"""pa_decode_fixed_scratch: paged decode for callers that cannot allocate device memory.

Such callers (a plugin inside an engine whose memory planner owns every device
allocation, or a serving loop that forbids allocation after start-up) pass
inputs and outputs only; the split-context partials live in the library's
fixed 32 MiB device array.  These tests call the entry point through the C
ABI (ctypes) and compare it with pa_decode, which takes a caller-provided
workspace, and with the fp64 oracle, within the bf16 decode tolerance used by
every decode test.  Two calls in a row on different inputs check that what
the array keeps from the previous call does not leak into the next; a call
after the first is checked to leave the device's free memory and torch's
allocated bytes unchanged.  This file is collected last, so a run that stops
at the first failure has run every other test before it.
"""
import ctypes
import math

import numpy as np
import pytest

from oracle import attention
from paged_kv_cache_356_b200 import _lib
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from tests.parity import BF16_ATOL, BF16_RTOL, assert_decode_close

pytestmark = pytest.mark.gpu


def _case(seed, ctx, hq=32, hkv=8, d=128, bs=16):
    import torch
    rng = np.random.Generator(np.random.PCG64(seed))
    need = [-(-c // bs) for c in ctx]
    nb = sum(need) + 4
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((len(ctx), max(need)), -1, dtype=np.int32)
    i = 0
    for b, n in enumerate(need):
        tables[b, :n] = perm[i:i + n]
        i += n

    def dev_bf16(n, shape):
        bits = workloads.normal_values(rng, n, "bf16").reshape(shape)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()

    kc = dev_bf16(nb * hkv * bs * d, (nb, hkv, bs, d))
    vc = dev_bf16(nb * hkv * bs * d, (nb, hkv, bs, d))
    q = dev_bf16(len(ctx) * hq * d, (len(ctx), hq, d))
    return dict(q=q, kc=kc, vc=vc, tables=torch.from_numpy(tables).cuda(), tables_np=tables,
                ctx=torch.tensor(ctx, dtype=torch.int32).cuda(), ctx_np=np.array(ctx, dtype=np.int32),
                scale=1.0 / math.sqrt(d))


def _fixed_scratch_call(c, out):
    """Call pa_decode_fixed_scratch through the C ABI; returns its status."""
    import torch
    lib = _lib.load()
    nb, hkv, bs, d = c["kc"].shape
    b, hq, _ = c["q"].shape
    return lib.pa_decode_fixed_scratch(
        c["q"].data_ptr(), c["kc"].data_ptr(), c["vc"].data_ptr(), c["tables"].data_ptr(), c["tables"].shape[1],
        c["ctx"].data_ptr(), b, hq, hkv, d, bs, nb, ctypes.c_float(c["scale"]), out.data_ptr(), _lib.PA_BF16,
        None, torch.cuda.current_stream().cuda_stream)


def _reference(c):
    return pa.pa_decode(c["q"], c["kc"], c["vc"], c["tables"], c["ctx"], c["scale"])


def _oracle(c):
    """fp64 textbook attention over the same stored bf16 bits."""
    bits = lambda t: t.view(__import__("torch").int16).cpu().numpy().view(np.uint16)
    return attention.decode_attention(bits(c["q"]), bits(c["kc"]), bits(c["vc"]), c["tables_np"], c["ctx_np"],
                                      c["scale"], "bf16")


def _assert_close(got, want):
    g = got.double().cpu().numpy()
    w = want.double().cpu().numpy()
    assert np.all(np.abs(g - w) <= BF16_ATOL + BF16_RTOL * np.abs(w))


def test_two_calls_in_a_row_match_pa_decode():
    import torch
    first = _case(1, [3000, 17, 1025, 2048, 511, 4000])       # up to 8 partitions: the scratch is used
    second = _case(2, [700, 2600, 1, 1900])                    # different shapes and data
    for c in (first, second):
        need = pa.pa_decode_workspace_size(c["q"].shape[0], c["q"].shape[1], 128, c["tables"].shape[1] * 16)
        assert 0 < need <= _lib.PA_FIXED_SCRATCH_BYTES
        out = torch.full_like(c["q"], float("nan"))
        assert _fixed_scratch_call(c, out) == 0, _lib.last_error()
        torch.cuda.synchronize()
        _assert_close(out, _reference(c))
        assert_decode_close(out, _oracle(c), "bf16", "pa_decode_fixed_scratch vs oracle")


def test_a_call_after_the_first_allocates_no_device_memory():
    """After the first call has done its one-time set-up, a call changes neither the device's free
    memory nor torch's allocated bytes; the same holds through the Python binding."""
    import torch
    c = _case(3, [1500, 40, 2600])
    out = torch.empty_like(c["q"])
    assert _fixed_scratch_call(c, out) == 0, _lib.last_error()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    assert _fixed_scratch_call(c, out) == 0, _lib.last_error()
    pa.pa_decode_fixed_scratch(c["q"], c["kc"], c["vc"], c["tables"], c["ctx"], c["scale"], out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert_decode_close(out, _oracle(c), "bf16", "binding pa_decode_fixed_scratch vs oracle")


def test_empty_batch_returns_before_any_work():
    import torch
    c = _case(4, [5])
    empty = dict(c, q=c["q"][:0], tables=c["tables"][:0], ctx=c["ctx"][:0])
    out = torch.empty_like(empty["q"])
    assert _fixed_scratch_call(empty, out) == 0, _lib.last_error()


def test_call_beyond_the_fixed_scratch_is_rejected():
    import torch
    # 256 sequences x 64 heads x 16 partitions needs ~136 MB of partials: over the limit.
    # Every buffer is real and every table entry points at page 0, so nothing could read
    # out of bounds even if a kernel were launched; none must be.
    c = dict(q=torch.zeros(256, 64, 128, dtype=torch.bfloat16, device="cuda"),
             kc=torch.zeros(1, 8, 16, 128, dtype=torch.bfloat16, device="cuda"),
             vc=torch.zeros(1, 8, 16, 128, dtype=torch.bfloat16, device="cuda"),
             tables=torch.zeros(256, 512, dtype=torch.int32, device="cuda"),
             ctx=torch.full((256,), 512 * 16, dtype=torch.int32, device="cuda"), scale=0.1)
    out = torch.full_like(c["q"], 7.0)
    assert _fixed_scratch_call(c, out) == _lib.PA_ERR_INVALID
    assert "fixed" in _lib.last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)

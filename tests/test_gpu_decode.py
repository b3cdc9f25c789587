"""pa_decode on the GPU against the fp64 oracle.

Both partition kernels (tensor-core and CUDA-core) are run on every case they
support.  Cases span several 16-token tiles, several 512-token partitions and
ragged tails; edge cases cover empty sequences, single tokens, lengths at and
around tile / page / partition boundaries, every GQA group size, head_dim and
block size the kernels accept, and out-of-range table entries and lengths,
which the kernels must skip and report instead of reading out of bounds.
"""
import math

import numpy as np
import pytest

from oracle import attention, scenario
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from paged_kv_cache_356_b200.runner import TraceRunner
from tests.parity import assert_decode_close, bits_of, host_bits

pytestmark = pytest.mark.gpu

KERNELS = {"tc": pa.PA_DECODE_TENSOR_CORES, "cc": pa.PA_DECODE_CUDA_CORES, "auto": pa.PA_DECODE_AUTO}


@pytest.fixture(autouse=True)
def _reset_kernel():
    yield
    pa.pa_set_decode_kernel(pa.PA_DECODE_AUTO)
    pa.pa_set_decode_tiling(4, 2)


def _values(rng, n, dtype):
    if dtype == "f16":
        return rng.standard_normal(n, dtype=np.float32).astype(np.float16).view(np.uint16)
    return workloads.normal_values(rng, n, dtype)


def _paged_case(seed, ctx, hq, hkv, d, bs, dtype, extra=3):
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(ctx, dtype=np.int32)
    need = [max(1, -(-int(c) // bs)) for c in ctx]
    nb = sum(need) + extra
    mb = max(need)
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((len(ctx), mb), -1, dtype=np.int32)
    i = 0
    for b, n in enumerate(need):
        tables[b, :n] = perm[i:i + n]
        i += n
    shape = (nb, hkv, bs, d)
    kc = _values(rng, int(np.prod(shape)), dtype).reshape(shape)
    vc = _values(rng, int(np.prod(shape)), dtype).reshape(shape)
    q = _values(rng, len(ctx) * hq * d, dtype).reshape(len(ctx), hq, d)
    return dict(q=q, kc=kc, vc=vc, tables=tables, ctx=ctx, scale=1.0 / math.sqrt(d), dtype=dtype)


def _dev(a, dtype):
    import torch
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(tdt).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run_gpu(case, kernel="auto", tables=None, ctx=None, workspace=None, status=None):
    import torch
    pa.pa_set_decode_kernel(KERNELS[kernel])
    dt = case["dtype"]
    t = case["tables"] if tables is None else tables
    c = case["ctx"] if ctx is None else ctx
    if workspace is None:  # NaN bytes: a partial that no kernel wrote cannot pass for a stale one
        q = case["q"]
        need = pa.pa_decode_workspace_size(q.shape[0], q.shape[1], q.shape[2], t.shape[1] * case["kc"].shape[2])
        workspace = torch.full((max(need, 256),), 0xFF, dtype=torch.uint8, device="cuda")
    out = pa.pa_decode(_dev(case["q"], dt), _dev(case["kc"], dt), _dev(case["vc"], dt),
                       torch.from_numpy(t).cuda(), torch.from_numpy(np.asarray(c, np.int32)).cuda(), case["scale"],
                       workspace=workspace, dev_status=status)
    torch.cuda.synchronize()
    return out


def _oracle(case, tables=None, ctx=None):
    t = case["tables"] if tables is None else tables
    c = case["ctx"] if ctx is None else ctx
    return attention.decode_attention(case["q"], case["kc"], case["vc"], t, c, case["scale"], case["dtype"])


# -- full flows through the C ABI (allocator + cache write + copy + decode) -------------------

def _compare_flow(w, kernel):
    pa.pa_set_decode_kernel(KERNELS[kernel])
    run = TraceRunner(w)
    out = run.run()
    ref = scenario.run(w)
    assert run.allocator_state() == ref["state"]
    assert run.cow_pairs == ref["cow_pairs"]
    np.testing.assert_array_equal(bits_of(run.key_cache), host_bits(ref["key_cache"]))
    np.testing.assert_array_equal(bits_of(run.value_cache), host_bits(ref["value_cache"]))
    assert run.status() == 0
    return assert_decode_close(out, ref["out"], w.dtype, w.name)


def test_tiny_workload_full_flow():
    """36- and 42-token sequences, 16-token pages from a shuffled pool of 16, fp32."""
    _compare_flow(workloads.tiny(), "auto")


@pytest.mark.parametrize("kernel", ["tc", "cc"])
@pytest.mark.parametrize("make", [
    lambda: workloads.llama8b(num_seqs=8, lo=100, hi=1300),
    lambda: workloads.llama70b(num_seqs=6, lo=512, hi=2600),
    lambda: workloads.prefix(num_seqs=5, prefix_len=700, max_tail=90),
    lambda: workloads.beam32k(num_beams=3, prompt_len=1100, own=40),
], ids=["llama8b-small", "llama70b-small", "prefix-small", "beam-small"])
def test_small_flows(make, kernel):
    _compare_flow(make(), kernel)


# -- kernel-level cases -------------------------------------------------------------------------

EDGE_LENGTHS = [1, 2, 15, 16, 17, 31, 32, 33, 255, 511, 512, 513, 1023, 1024, 1025, 1536, 2049]


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_edge_lengths(kernel):
    case = _paged_case(1, EDGE_LENGTHS, 64, 8, 128, 16, "bf16")
    assert_decode_close(_run_gpu(case, kernel), _oracle(case), "bf16", kernel)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("bs", [16, 32, 128])
def test_tensor_core_shapes(dtype, d, group, bs):
    hkv = 2
    case = _paged_case(d + group + bs, [7, 300, 777, 1300], group * hkv, hkv, d, bs, dtype)
    out = _run_gpu(case, "tc")
    assert_decode_close(out, _oracle(case), dtype, f"tc {dtype} d{d} g{group} bs{bs}")
    out_cc = _run_gpu(case, "cc")
    assert_decode_close(out_cc, _oracle(case), dtype, f"cc {dtype} d{d} g{group} bs{bs}")


@pytest.mark.parametrize("dtype,d,group,bs", [("f32", 64, 4, 16), ("f32", 128, 8, 1), ("f32", 256, 3, 8),
                                              ("bf16", 128, 16, 16), ("bf16", 64, 5, 24), ("f16", 128, 8, 8),
                                              ("bf16", 128, 8, 256), ("bf16", 128, 2, 1)])
def test_cuda_core_shapes(dtype, d, group, bs):
    hkv = 2
    case = _paged_case(d * group + bs, [1, 40, 513, 1100], group * hkv, hkv, d, bs, dtype)
    assert_decode_close(_run_gpu(case, "auto"), _oracle(case), dtype, f"auto {dtype} d{d} g{group} bs{bs}")
    assert_decode_close(_run_gpu(case, "cc"), _oracle(case), dtype, f"cc {dtype} d{d} g{group} bs{bs}")


@pytest.mark.parametrize("kernel", ["tc", "cc"])
@pytest.mark.parametrize("ctx", [[9000, 15000, 700], [9000, 20000, 700], [30000, 1, 513],
                                 [70000, 40000, 1, 513], [140000, 3, 2000]],
                         ids=["p30", "p40", "p59", "p137", "p274"])
def test_long_contexts_merge_many_partitions(kernel, ctx):
    """Merges of 30 to 274 partitions: the merge kernel's 2- and 4-warp forms, the
    latter over more than one group of 128 partitions (32 per warp)."""
    case = _paged_case(31 + len(ctx), ctx, 4, 1, 128, 16, "bf16")
    assert_decode_close(_run_gpu(case, kernel), _oracle(case), "bf16", f"{kernel} ctx{ctx}")


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_empty_sequences_give_zeros(kernel):
    case = _paged_case(4, [0, 600, 0, 3, 0], 16, 2, 128, 16, "bf16")
    out = _run_gpu(case, kernel)
    ref = _oracle(case)
    assert_decode_close(out, ref, "bf16", kernel)
    assert not out[0].float().abs().sum().item() and not out[2].float().abs().sum().item()


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_partition_partials_in_workspace(kernel):
    """The workspace holds each 512-token partition's (o_p / l_p, m_p, l_p) as documented."""
    import torch
    ctx = [1300, 513, 100]
    case = _paged_case(9, ctx, 8, 2, 128, 32, "bf16")
    mb = case["tables"].shape[1]
    need = pa.pa_decode_workspace_size(3, 8, 128, mb * 32)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    _run_gpu(case, kernel, workspace=ws)
    parts = -(-mb * 32 // 512)
    rows = 3 * 8 * parts
    align = lambda x: (x + 255) // 256 * 256  # noqa: E731
    raw = ws.cpu().numpy()
    o_part = raw[:rows * 128 * 4].view(np.float32).reshape(3, 8, parts, 128)
    m_off = align(rows * 128 * 4)
    m_part = raw[m_off:m_off + rows * 4].view(np.float32).reshape(3, 8, parts)
    l_off = m_off + align(rows * 4)
    l_part = raw[l_off:l_off + rows * 4].view(np.float32).reshape(3, 8, parts)
    q64 = attention.to_float64(case["q"], "bf16")
    for b in (0, 1):   # sequence 2 has one partition and writes its output directly
        keys = attention.to_float64(attention.gather_sequence(case["kc"], case["tables"][b], ctx[b]), "bf16")
        values = attention.to_float64(attention.gather_sequence(case["vc"], case["tables"][b], ctx[b]), "bf16")
        for h in range(8):
            ref = attention.partition_attention(q64[b, h], keys[:, h // 4], values[:, h // 4], case["scale"])
            for p, (o_ref, m_ref, l_ref) in enumerate(ref):
                np.testing.assert_allclose(o_part[b, h, p], o_ref, atol=2e-3, rtol=1e-2)
                np.testing.assert_allclose(m_part[b, h, p], m_ref, atol=1e-3, rtol=1e-3)
                np.testing.assert_allclose(l_part[b, h, p], l_ref, rtol=1e-2)


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_out_of_range_pages_are_skipped_and_flagged(kernel):
    import torch
    case = _paged_case(12, [100, 700, 64], 16, 2, 128, 16, "bf16")
    tables = case["tables"].copy()
    nb = case["kc"].shape[0]
    tables[0, 2] = nb + 3          # tokens 32..47 of sequence 0
    tables[1, 40] = -5             # tokens 640..655 of sequence 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run_gpu(case, kernel, tables=tables, status=status)
    assert status.item() & pa.PA_DEV_BAD_PAGE
    # reference: attention over the tokens whose pages are valid
    q64 = attention.to_float64(case["q"], "bf16")
    ref = _oracle(case)
    for b, bad_block in ((0, 2), (1, 40)):
        keep = [j for j in range(case["ctx"][b]) if j // 16 != bad_block]
        keys = attention.to_float64(attention.gather_sequence(case["kc"], case["tables"][b], case["ctx"][b]), "bf16")
        vals = attention.to_float64(attention.gather_sequence(case["vc"], case["tables"][b], case["ctx"][b]), "bf16")
        for h in range(16):
            ref[b, h] = attention.softmax_attention(q64[b, h], keys[keep, h // 8], vals[keep, h // 8], case["scale"])
    assert_decode_close(out, ref, "bf16", kernel)


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_out_of_range_context_is_clamped_and_flagged(kernel):
    import torch
    case = _paged_case(13, [64, 50], 8, 1, 64, 16, "bf16")
    mb = case["tables"].shape[1]
    assert mb == 4
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run_gpu(case, kernel, ctx=np.array([mb * 16 + 100, -3], np.int32), status=status)
    assert status.item() == pa.PA_DEV_BAD_CTX
    # sequence 0 is clamped to what its (full) table addresses; sequence 1 gives zeros
    assert_decode_close(out, _oracle(case, ctx=[mb * 16, 0]), "bf16", kernel)


def test_forcing_tensor_cores_on_fp32_is_rejected():
    case = _paged_case(2, [10], 4, 1, 64, 16, "f32")
    with pytest.raises(pa.PagedAttentionError):
        _run_gpu(case, "tc")


@pytest.mark.parametrize("warps,stages", [(4, 2), (4, 3), (4, 4), (2, 4), (8, 2)])
def test_every_built_tiling_matches(warps, stages):
    case = _paged_case(21, [5, 16, 333, 512, 900, 2100], 32, 4, 128, 16, "bf16")
    pa.pa_set_decode_tiling(warps, stages)
    assert_decode_close(_run_gpu(case, "tc"), _oracle(case), "bf16", f"tiling {warps}x{stages}")


def test_repeat_calls_are_bit_identical():
    case = _paged_case(22, [700, 1500, 3], 16, 2, 128, 16, "bf16")
    a = bits_of(_run_gpu(case, "tc"))
    b = bits_of(_run_gpu(case, "tc"))
    np.testing.assert_array_equal(a, b)

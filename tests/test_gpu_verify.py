"""pa_decode_verify (several causal query tokens per sequence) on the GPU against the fp64 oracle.

Both partition kernels run on every case they support.  Cases cover one to
several row tiles per CTA and several CTAs per kv head, GQA groups above 8,
padding rows, every head_dim, contexts shorter than the query count, at and
around tile / page / partition boundaries, several partitions with the
log-sum-exp merge, empty sequences, and out-of-range pages and lengths.
"""
import math

import numpy as np
import pytest

from oracle import attention
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from tests.parity import assert_decode_close, bits_of

pytestmark = pytest.mark.gpu

KERNELS = {"tc": pa.PA_DECODE_TENSOR_CORES, "cc": pa.PA_DECODE_CUDA_CORES, "auto": pa.PA_DECODE_AUTO}
PATHS = {"auto": pa.PA_VERIFY_AUTO, "per_sequence": pa.PA_VERIFY_PER_SEQUENCE, "joint": pa.PA_VERIFY_JOINT}
# (partition kernel, path): the joint path runs the tcgen05 shared-prefix kernel on the partitions
# every token sees in full and the tensor-core verify kernel on the rest
ROUTES = [("tc", "per_sequence"), ("tc", "joint"), ("cc", "per_sequence")]


@pytest.fixture(autouse=True)
def _reset_kernel():
    yield
    pa.pa_set_decode_kernel(pa.PA_DECODE_AUTO)
    pa.pa_set_verify_path(pa.PA_VERIFY_AUTO)
    pa.pa_set_shared_prefix_kernel(pa.PA_SHARED_PREFIX_AUTO)
    pa.pa_set_verify_tiling(0)


def _values(rng, n, dtype):
    if dtype == "f16":
        return rng.standard_normal(n, dtype=np.float32).astype(np.float16).view(np.uint16)
    return workloads.normal_values(rng, n, dtype)


def _case(seed, ctx, num_tokens, hq, hkv, d, bs, dtype, extra=3):
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(ctx, dtype=np.int32)
    need = [max(1, -(-int(c) // bs)) for c in ctx]
    nb = sum(need) + extra
    perm = rng.permutation(nb).astype(np.int32)
    tables = np.full((len(ctx), max(need)), -1, dtype=np.int32)
    i = 0
    for b, n in enumerate(need):
        tables[b, :n] = perm[i:i + n]
        i += n
    shape = (nb, hkv, bs, d)
    kc = _values(rng, int(np.prod(shape)), dtype).reshape(shape)
    vc = _values(rng, int(np.prod(shape)), dtype).reshape(shape)
    q = _values(rng, len(ctx) * num_tokens * hq * d, dtype).reshape(len(ctx), num_tokens, hq, d)
    return dict(q=q, kc=kc, vc=vc, tables=tables, ctx=ctx, scale=1.0 / math.sqrt(d), dtype=dtype)


def _dev(a, dtype):
    import torch
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(tdt).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(case, kernel, tables=None, ctx=None, status=None, path="auto"):
    import torch
    pa.pa_set_decode_kernel(KERNELS[kernel])
    pa.pa_set_verify_path(PATHS[path])
    dt = case["dtype"]
    t = case["tables"] if tables is None else tables
    c = case["ctx"] if ctx is None else ctx
    q = _dev(case["q"], dt)
    # The workspace starts as NaN bytes, so a partial that no kernel wrote cannot pass for a stale
    # correct one left by an earlier call.
    need = pa.pa_decode_verify_workspace_size(q.shape[0], q.shape[1], q.shape[2], q.shape[3],
                                              t.shape[1] * case["kc"].shape[2])
    ws = torch.full((max(need, 1),), 0xFF, dtype=torch.uint8, device="cuda")
    own_status = status is None
    if own_status:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = pa.pa_decode_verify(q, _dev(case["kc"], dt), _dev(case["vc"], dt),
                              torch.from_numpy(t).cuda(), torch.from_numpy(np.asarray(c, np.int32)).cuda(),
                              case["scale"], workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    if own_status:
        assert status.item() == 0, f"device status {status.item():#x}"
    return out


def _oracle(case, ctx=None):
    c = case["ctx"] if ctx is None else ctx
    return attention.verify_attention(case["q"], case["kc"], case["vc"], case["tables"], c, case["scale"],
                                      case["dtype"])


CONTEXTS = [1, 3, 4, 15, 16, 17, 33, 100, 511, 512, 513, 515, 1040, 1700]

# (query tokens, q heads, kv heads, head_dim, block_size, dtype): rows per kv head = T * G
SHAPES = [
    (1, 8, 1, 128, 16, "bf16"),     # 8 rows: one n8 tile (a decode step)
    (2, 32, 8, 128, 16, "bf16"),    # 8 rows, G = 4
    (4, 32, 8, 128, 16, "bf16"),    # 16 rows: two tiles
    (4, 64, 8, 128, 16, "bf16"),    # 32 rows: four tiles
    (5, 32, 8, 128, 16, "bf16"),    # 20 rows: four tiles, 12 padding rows
    (8, 64, 8, 128, 16, "bf16"),    # 64 rows: two CTAs per kv head
    (7, 8, 8, 128, 32, "bf16"),     # G = 1
    (2, 24, 2, 128, 16, "bf16"),    # G = 12
    (3, 8, 2, 64, 16, "f16"),
    (6, 16, 2, 64, 48, "bf16"),     # 48 rows at head_dim 64, 48-token pages
    (3, 16, 2, 256, 16, "bf16"),    # 24 rows at head_dim 256: two CTAs of 16
]


@pytest.mark.parametrize("route", ROUTES, ids=["-".join(r) for r in ROUTES])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"T{s[0]}-hq{s[1]}-hkv{s[2]}-d{s[3]}-bs{s[4]}-{s[5]}" for s in SHAPES])
def test_verify_matches_oracle(shape, route):
    num_tokens, hq, hkv, d, bs, dtype = shape
    kernel, path = route
    if path == "joint" and d == 256:
        pytest.skip("the joint kernel serves head_dim 64 and 128")
    case = _case(100 + num_tokens * 7 + d, CONTEXTS, num_tokens, hq, hkv, d, bs, dtype)
    assert_decode_close(_run(case, kernel, path=path), _oracle(case), dtype, f"{route} {shape}")


# Contexts around the edge of the partitions all T tokens see: ctx - T + 1 at, just below and just
# above a multiple of 512, one-partition sequences beside multi-partition ones.
def _edge_contexts(num_tokens):
    out = [5, 512, 513]
    for k in (1, 2, 3):
        out += [512 * k + num_tokens - 2, 512 * k + num_tokens - 1, 512 * k + num_tokens]
    return [c for c in out if c > 0]


@pytest.mark.parametrize("joint_kernel", ["tcgen05", "tcgen05_items", "mma_sync"])
@pytest.mark.parametrize("num_tokens,hq,hkv,d", [(4, 64, 8, 128), (3, 8, 2, 64), (5, 32, 1, 128), (9, 16, 1, 64)],
                         ids=["T4-G8", "T3-G4-d64", "T5-G32-two-chunks", "T9-G16-two-chunks"])
def test_joint_path_partition_edges(num_tokens, hq, hkv, d, joint_kernel):
    """The joint kernel's plan (built on the device) against the causal limits; G * T above 128
    splits a sequence's tokens over several chunks.  tcgen05 is the balanced kernel (equal ranges of
    steps per CTA), tcgen05_items the one-CTA-per-partition kernel."""
    pa.pa_set_shared_prefix_kernel({"tcgen05": pa.PA_SHARED_PREFIX_TCGEN05,
                                    "tcgen05_items": pa.PA_SHARED_PREFIX_TCGEN05_ITEMS,
                                    "mma_sync": pa.PA_SHARED_PREFIX_MMA_SYNC}[joint_kernel])
    case = _case(300 + num_tokens, _edge_contexts(num_tokens), num_tokens, hq, hkv, d, 16, "bf16")
    assert_decode_close(_run(case, "tc", path="joint"), _oracle(case), "bf16", joint_kernel)


@pytest.mark.parametrize("path", ["per_sequence", "joint"])
@pytest.mark.parametrize("rows_per_cta", [8, 16, 32])
def test_every_built_row_tiling_matches(rows_per_cta, path):
    """32 rows per kv head served by 4, 2 or 1 CTAs of 8, 16 or 32 rows."""
    pa.pa_set_verify_tiling(rows_per_cta)
    case = _case(400 + rows_per_cta, CONTEXTS, 4, 64, 8, 128, 16, "bf16")
    assert_decode_close(_run(case, "tc", path=path), _oracle(case), "bf16", f"{rows_per_cta} {path}")


def test_unbuilt_row_tiling_is_rejected():
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_set_verify_tiling(24)


@pytest.mark.parametrize("route", ROUTES, ids=["-".join(r) for r in ROUTES])
def test_prefill_chunk_of_many_tokens(route):
    """A chunk of 100 new tokens at the end of each context (chunked prefill is the same computation):
    400 rows per kv head, many row groups and joint-kernel chunks per sequence."""
    case = _case(500, [100, 101, 700, 1537, 2100], 100, 16, 4, 64, 16, "bf16")
    assert_decode_close(_run(case, route[0], path=route[1]), _oracle(case), "bf16", str(route))


def test_joint_path_that_cannot_run_is_rejected():
    case = _case(17, [10, 20], 2, 8, 2, 64, 16, "bf16")      # one partition: nothing for the joint kernel
    with pytest.raises(pa.PagedAttentionError):
        _run(case, "tc", path="joint")


@pytest.mark.parametrize("num_tokens,bs", [(3, 16), (4, 8), (2, 5)])
def test_verify_fp32_and_odd_pages_on_cuda_cores(num_tokens, bs):
    """fp32 or pages off the 16-token tile run on the CUDA-core kernel (auto picks it)."""
    for dtype in ("f32", "bf16"):
        case = _case(200 + bs, [1, 2, 9, 40, 530], num_tokens, 8, 2, 64, bs, dtype)
        if dtype == "bf16" and bs % 16 == 0:
            continue
        assert_decode_close(_run(case, "auto"), _oracle(case), dtype, f"{dtype} bs{bs}")


def test_forcing_tensor_cores_on_fp32_is_rejected():
    case = _case(3, [10], 2, 4, 1, 64, 16, "f32")
    with pytest.raises(pa.PagedAttentionError):
        _run(case, "tc")


@pytest.mark.parametrize("route", ROUTES, ids=["-".join(r) for r in ROUTES])
def test_long_contexts_merge_partitions(route):
    case = _case(7, [4100, 9000, 2], 4, 32, 8, 128, 16, "bf16")
    assert_decode_close(_run(case, route[0], path=route[1]), _oracle(case), "bf16", str(route))


@pytest.mark.parametrize("route", ROUTES, ids=["-".join(r) for r in ROUTES])
def test_empty_sequences_and_tokens_before_the_context_give_zeros(route):
    case = _case(8, [0, 2, 700], 5, 16, 2, 128, 16, "bf16")
    out = _run(case, route[0], path=route[1])
    ref = _oracle(case)
    assert np.all(ref[0] == 0) and np.all(ref[1, :3] == 0)
    assert np.all(bits_of(out[0]) == 0) and np.all(bits_of(out[1, :3]) == 0)
    assert_decode_close(out, ref, "bf16", str(route))


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_out_of_range_pages_are_skipped_and_flagged(kernel):
    import torch
    num_tokens, hq, hkv = 3, 16, 2
    case = _case(12, [100, 700], num_tokens, hq, hkv, 128, 16, "bf16")
    tables = case["tables"].copy()
    nb = case["kc"].shape[0]
    tables[0, 2] = nb + 3          # tokens 32..47 of sequence 0
    tables[1, 40] = -5             # tokens 640..655 of sequence 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(case, kernel, tables=tables, status=status)
    assert status.item() & pa.PA_DEV_BAD_PAGE
    q64 = attention.to_float64(case["q"], "bf16")
    ref = np.zeros(q64.shape)
    g = hq // hkv
    for b, bad_block in ((0, 2), (1, 40)):
        c = int(case["ctx"][b])
        keys = attention.to_float64(attention.gather_sequence(case["kc"], case["tables"][b], c), "bf16")
        vals = attention.to_float64(attention.gather_sequence(case["vc"], case["tables"][b], c), "bf16")
        for t in range(num_tokens):
            keep = [j for j in range(attention.visible_keys(c, num_tokens, t)) if j // 16 != bad_block]
            for h in range(hq):
                ref[b, t, h] = attention.softmax_attention(q64[b, t, h], keys[keep, h // g], vals[keep, h // g],
                                                           case["scale"])
    assert_decode_close(out, ref, "bf16", kernel)


@pytest.mark.parametrize("kernel", ["tc", "cc"])
def test_out_of_range_context_is_clamped_and_flagged(kernel):
    import torch
    case = _case(13, [64, 50], 2, 8, 1, 64, 16, "bf16")
    mb = case["tables"].shape[1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _run(case, kernel, ctx=np.array([mb * 16 + 100, -3], np.int32), status=status)
    assert status.item() == pa.PA_DEV_BAD_CTX
    assert_decode_close(out, _oracle(case, ctx=[mb * 16, 0]), "bf16", kernel)


def test_one_query_token_matches_decode():
    """T = 1 computes what pa_decode computes (both within tolerance of the same oracle rows)."""
    import torch
    case = _case(14, CONTEXTS, 1, 64, 8, 128, 16, "bf16")
    out = _run(case, "auto")
    q3 = _dev(case["q"][:, 0], "bf16")
    dec = pa.pa_decode(q3, _dev(case["kc"], "bf16"), _dev(case["vc"], "bf16"),
                       torch.from_numpy(case["tables"]).cuda(), torch.from_numpy(case["ctx"]).cuda(), case["scale"])
    ref = _oracle(case)[:, 0]
    assert_decode_close(out[:, 0], ref, "bf16", "verify")
    assert_decode_close(dec, ref, "bf16", "decode")


@pytest.mark.parametrize("path", ["per_sequence", "joint"])
def test_repeat_calls_are_bit_identical(path):
    case = _case(15, [300, 1300, 5], 4, 64, 8, 128, 16, "bf16")
    a = bits_of(_run(case, "auto", path=path))
    b = bits_of(_run(case, "auto", path=path))
    assert np.array_equal(a, b)


def test_bad_arguments_are_rejected():
    import torch
    case = _case(16, [10], 2, 8, 2, 64, 16, "bf16")
    dev = lambda a: _dev(a, "bf16")
    kc, vc = dev(case["kc"]), dev(case["vc"])
    tables = torch.from_numpy(case["tables"]).cuda()
    ctx = torch.from_numpy(case["ctx"]).cuda()
    with pytest.raises(ValueError):
        pa.pa_decode_verify(dev(case["q"][:, 0]), kc, vc, tables, ctx, 0.1)        # 3-D q
    q = dev(case["q"])
    lib = pa._lib.load()
    st = lib.pa_decode_verify(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), tables.data_ptr(), 1, ctx.data_ptr(),
                              1, 0, 8, 2, 64, 16, case["kc"].shape[0], 0.1, q.data_ptr(), pa.PA_BF16, None, 0,
                              None, None)
    assert st == pa._lib.PA_ERR_INVALID

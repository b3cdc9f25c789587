"""pa_reshape_and_cache and pa_copy_blocks on the GPU: bit-exact against the oracle."""
import numpy as np
import pytest

from oracle import cache_ops
from paged_kv_cache_356_b200 import binding as pa
from paged_kv_cache_356_b200 import workloads
from tests.parity import bits_of, host_bits

pytestmark = pytest.mark.gpu

DTYPES = {"bf16": ("bfloat16", np.uint16), "f16": ("float16", np.uint16), "f32": ("float32", np.float32)}


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _values(rng, shape, dtype):
    n = int(np.prod(shape))
    if dtype == "f32":
        return rng.standard_normal(n, dtype=np.float32).reshape(shape)
    # arbitrary 16-bit patterns (NaN/Inf patterns included): the copy must move bits
    return rng.integers(0, 65536, size=n, dtype=np.uint16).reshape(shape)


def _dev(a, dtype):
    import torch
    tdt = getattr(torch, DTYPES[dtype][0])
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(tdt).cuda()
    return torch.from_numpy(a).cuda()


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("num_tokens,hkv,bs,d", [(1, 1, 16, 64), (37, 2, 16, 128), (300, 8, 32, 128),
                                                 (129, 4, 1, 64), (70, 3, 8, 256)])
def test_reshape_and_cache_bit_exact(dtype, num_tokens, hkv, bs, d):
    import torch
    rng = _rng(num_tokens * 7 + hkv)
    nb = (num_tokens + bs - 1) // bs + 5
    kc = _values(rng, (nb, hkv, bs, d), dtype)
    vc = _values(rng, (nb, hkv, bs, d), dtype)
    key = _values(rng, (num_tokens, hkv, d), dtype)
    value = _values(rng, (num_tokens, hkv, d), dtype)
    slots = rng.permutation(nb * bs)[:num_tokens].astype(np.int64)
    slots[rng.random(num_tokens) < 0.1] = -1          # padding tokens
    kd, vd = _dev(kc, dtype), _dev(vc, dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(_dev(key, dtype), _dev(value, dtype), torch.from_numpy(slots).cuda(), kd, vd,
                            dev_status=status)
    cache_ops.reshape_and_cache(key, value, slots, kc, vc)
    np.testing.assert_array_equal(bits_of(kd), host_bits(kc))
    np.testing.assert_array_equal(bits_of(vd), host_bits(vc))
    assert status.item() == 0


def test_reshape_and_cache_strided_rows():
    """K and V as views into a fused [T, 3, Hkv, D] projection output."""
    import torch
    rng = _rng(11)
    t, hkv, d, bs, nb = 50, 4, 128, 16, 8
    fused = _values(rng, (t, 3, hkv, d), "bf16")
    fd = _dev(fused, "bf16")
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    kd, vd = _dev(kc, "bf16"), _dev(vc, "bf16")
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    pa.pa_reshape_and_cache(fd[:, 1], fd[:, 2], torch.from_numpy(slots).cuda(), kd, vd)
    cache_ops.reshape_and_cache(fused[:, 1], fused[:, 2], slots, kc, vc)
    np.testing.assert_array_equal(bits_of(kd), kc)
    np.testing.assert_array_equal(bits_of(vd), vc)


def test_reshape_and_cache_out_of_range_slot_is_skipped_and_flagged():
    import torch
    rng = _rng(3)
    nb, hkv, bs, d = 4, 2, 16, 64
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    key = _values(rng, (3, hkv, d), "bf16")
    slots = np.array([5, nb * bs, 2 ** 40], dtype=np.int64)     # one good, two past the pool
    kd, vd = _dev(kc, "bf16"), _dev(vc, "bf16")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(_dev(key, "bf16"), _dev(key, "bf16"), torch.from_numpy(slots).cuda(), kd, vd,
                            dev_status=status)
    cache_ops.reshape_and_cache(key[:1], key[:1], slots[:1], kc, vc)
    np.testing.assert_array_equal(bits_of(kd), kc)
    assert status.item() == pa.PA_DEV_BAD_SLOT


def test_reshape_and_cache_large_batch():
    """The 65,536-token write used for the kernel's bandwidth measurement."""
    import torch
    t, hkv, d, bs = 65536, 8, 128, 16
    nb = t // bs + 64
    rng = _rng(99)
    key = workloads.normal_values(rng, t * hkv * d, "bf16").reshape(t, hkv, d)
    value = workloads.normal_values(rng, t * hkv * d, "bf16").reshape(t, hkv, d)
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    kd = torch.zeros((nb, hkv, bs, d), dtype=torch.bfloat16, device="cuda")
    vd = torch.zeros_like(kd)
    pa.pa_reshape_and_cache(_dev(key, "bf16"), _dev(value, "bf16"), torch.from_numpy(slots).cuda(), kd, vd)
    kc = np.zeros((nb, hkv, bs, d), np.uint16)
    vc = np.zeros_like(kc)
    # oracle on a sample of tokens (the full loop is slow in Python): check those slots
    pick = rng.choice(t, 512, replace=False)
    cache_ops.reshape_and_cache(key[pick], value[pick], slots[pick], kc, vc)
    kb, vb = bits_of(kd), bits_of(vd)
    for i in pick:
        page, off = divmod(int(slots[i]), bs)
        np.testing.assert_array_equal(kb[page, :, off], kc[page, :, off])
        np.testing.assert_array_equal(vb[page, :, off], vc[page, :, off])
    # every written slot holds its token; no other slot was touched
    written = np.zeros(nb * bs, bool)
    written[slots] = True
    flat_k = kb.transpose(0, 2, 1, 3).reshape(nb * bs, hkv, d)
    np.testing.assert_array_equal(flat_k[slots], key)
    assert not flat_k[~written].any()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hkv,bs,d,pairs", [(1, 16, 64, 1), (8, 16, 128, 37), (8, 32, 128, 99), (2, 1, 64, 5)])
def test_copy_blocks_bit_exact(dtype, hkv, bs, d, pairs):
    import torch
    rng = _rng(pairs * 3 + bs)
    nb = 2 * pairs + 7
    kc = _values(rng, (nb, hkv, bs, d), dtype)
    vc = _values(rng, (nb, hkv, bs, d), dtype)
    perm = rng.permutation(nb)
    mapping = np.stack([perm[:pairs], perm[pairs:2 * pairs]], axis=1).astype(np.int64)
    kd, vd = _dev(kc, dtype), _dev(vc, dtype)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(mapping).cuda(), dev_status=status)
    cache_ops.copy_blocks(kc, vc, mapping)
    np.testing.assert_array_equal(bits_of(kd), host_bits(kc))
    np.testing.assert_array_equal(bits_of(vd), host_bits(vc))
    assert status.item() == 0


def test_copy_blocks_bad_pair_is_skipped_and_flagged():
    import torch
    rng = _rng(5)
    nb, hkv, bs, d = 6, 2, 16, 64
    kc = _values(rng, (nb, hkv, bs, d), "bf16")
    vc = _values(rng, (nb, hkv, bs, d), "bf16")
    mapping = np.array([[0, 1], [2, nb], [-1, 3], [4, 5]], dtype=np.int64)
    kd, vd = _dev(kc, "bf16"), _dev(vc, "bf16")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(mapping).cuda(), dev_status=status)
    cache_ops.copy_blocks(kc, vc, mapping[[0, 3]])
    np.testing.assert_array_equal(bits_of(kd), kc)
    np.testing.assert_array_equal(bits_of(vd), vc)
    assert status.item() == pa.PA_DEV_BAD_PAIR


def test_copy_blocks_many_pairs():
    """More pairs than one grid dimension holds (grid-stride over pairs)."""
    import torch
    nb, hkv, bs, d = 140_000, 1, 1, 64
    rng = _rng(8)
    kc = _values(rng, (nb, hkv, bs, d), "bf16")
    perm = rng.permutation(nb)
    mapping = np.stack([perm[:70_000], perm[70_000:]], axis=1).astype(np.int64)
    kd, vd = _dev(kc, "bf16"), _dev(kc, "bf16")
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(mapping).cuda())
    ref = kc.copy()
    ref[mapping[:, 1]] = kc[mapping[:, 0]]
    np.testing.assert_array_equal(bits_of(kd), ref)
    np.testing.assert_array_equal(bits_of(vd), ref)


# -- block-table updates --------------------------------------------------------------------------

def test_block_tables_apply_writes_each_update():
    """Distinct random (row, column, page) triples, more than one CTA of them, against numpy."""
    import torch
    rng = _rng(11)
    rows, mb = 300, 70
    tables = rng.integers(-5, 10_000, size=(rows, mb)).astype(np.int32)
    flat = rng.choice(rows * mb, size=5_000, replace=False)
    upd = np.stack([flat // mb, flat % mb, rng.integers(0, 10_000, size=len(flat))], axis=1).astype(np.int32)
    dt = torch.from_numpy(tables.copy()).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_block_tables_apply(dt, torch.from_numpy(upd).cuda(), dev_status=status)
    tables[upd[:, 0], upd[:, 1]] = upd[:, 2]
    np.testing.assert_array_equal(dt.cpu().numpy(), tables)
    assert status.item() == 0
    pa.pa_block_tables_apply(dt, torch.from_numpy(upd).cuda(), num_updates=0)   # nothing to do
    np.testing.assert_array_equal(dt.cpu().numpy(), tables)


def test_block_tables_apply_bad_update_is_skipped_and_flagged():
    import torch
    tables = np.zeros((4, 5), np.int32)
    upd = np.array([[0, 0, 7], [4, 0, 9], [1, 5, 9], [-2, 2, 9], [3, 4, 8], [2, -3, 9]], np.int32)
    dt = torch.from_numpy(tables.copy()).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_block_tables_apply(dt, torch.from_numpy(upd).cuda(), dev_status=status)
    tables[0, 0], tables[3, 4] = 7, 8
    np.testing.assert_array_equal(dt.cpu().numpy(), tables)
    assert status.item() == pa.PA_DEV_BAD_UPDATE


def test_block_tables_apply_skips_padding_rows():
    """Row -1 is padding: skipped without a flag, whatever the column and page."""
    import torch
    tables = np.arange(12, dtype=np.int32).reshape(3, 4)
    upd = np.array([[-1, 0, 50], [1, 2, 60], [-1, 99, 70], [-1, -1, -1]], np.int32)
    dt = torch.from_numpy(tables.copy()).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_block_tables_apply(dt, torch.from_numpy(upd).cuda(), dev_status=status)
    tables[1, 2] = 60
    np.testing.assert_array_equal(dt.cpu().numpy(), tables)
    assert status.item() == 0


def test_device_tables_follow_decode_steps():
    """The allocator's updates, applied on the device step after step (new blocks, a fork with
    copy-on-write, a freed and replaced sequence), keep the device copy equal to the full export."""
    import torch
    bs, mb = 16, 32
    alloc = pa.BlockAllocator(2_000, bs, _rng(3).permutation(2_000))
    for s, n in enumerate([5, 16, 200, 31, 47]):
        alloc.allocate_sequence(s, n)
    batch = list(range(5))
    dev = torch.full((len(batch), mb), 12345, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(60):
        if step == 20:
            alloc.fork(2, 9)
            batch[4] = 9            # row 4 now holds the fork
        if step == 40:
            alloc.free_sequence(1)
            alloc.allocate_sequence(1, 3)
        for s in batch:
            alloc.append_token(s)
        upd, lens = alloc.table_updates(batch, mb)
        pa.pa_block_tables_apply(dev, torch.from_numpy(upd.copy()).cuda(), dev_status=status)
        full, _ = alloc.block_tables(batch, mb)
        np.testing.assert_array_equal(dev.cpu().numpy(), full)
    assert status.item() == 0

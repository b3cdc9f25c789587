"""Pins of oracle/attention.py and oracle/cache_ops.py.

Each pin ties the oracle to something other than itself: the pages' printed
block tables, closed forms of softmax attention, torch's own
scaled_dot_product_attention (fp64, CPU), brute force over tiny inputs with
explicit page walking, and exact invariances (page relabelling, identity
tables).  ``test_planted_mistakes_are_caught`` plants plausible mistakes in
the oracle and checks that these pins fail on them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention, cache_ops


def _rand_case(rng, num_seqs, hq, hkv, d, bs, ctx_max, pages=None):
    """fp64 cache with random pages per sequence; returns tables, ctx, q, caches."""
    ctx = rng.integers(1, ctx_max + 1, size=num_seqs)
    need = sum(-(-int(c) // bs) for c in ctx)
    pages = pages or need + 3
    perm = rng.permutation(pages)
    mb = max(-(-int(c) // bs) for c in ctx)
    tables = np.full((num_seqs, mb), -1, dtype=np.int64)
    i = 0
    for b, c in enumerate(ctx):
        n = -(-int(c) // bs)
        tables[b, :n] = perm[i:i + n]
        i += n
    kc = rng.standard_normal((pages, hkv, bs, d))
    vc = rng.standard_normal((pages, hkv, bs, d))
    q = rng.standard_normal((num_seqs, hq, d))
    return q, kc, vc, tables, ctx


def _sdpa(q, keys, values, scale):
    """torch SDPA in fp64 on CPU, kv heads repeated for the query-head groups."""
    hq = q.shape[0]
    g = hq // keys.shape[1]
    qt = torch.from_numpy(q)[None, :, None, :]                                   # [1, Hq, 1, D]
    kt = torch.from_numpy(keys).permute(1, 0, 2).repeat_interleave(g, 0)[None]   # [1, Hq, ctx, D]
    vt = torch.from_numpy(values).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[0, :, 0, :].numpy()


def _brute(q_row, kc, vc, table, ctx, kvh, scale):
    """Pure-Python attention walking the table block by block, slot by slot."""
    bs = kc.shape[2]
    scores, rows = [], []
    for blk, page in enumerate(table):
        for off in range(bs):
            if blk * bs + off >= ctx:
                break
            k = kc[page][kvh][off]
            scores.append(scale * sum(float(q_row[i]) * float(k[i]) for i in range(len(q_row))))
            rows.append(vc[page][kvh][off])
    if not scores:
        return [0.0] * len(q_row)
    top = max(scores)
    w = [math.exp(s - top) for s in scores]
    tot = sum(w)
    return [sum(w[j] * float(rows[j][i]) for j in range(len(w))) / tot for i in range(len(q_row))]


# -- block-table translation --------------------------------------------------

@pytest.mark.parametrize("fixture", ["glossary_36_token_diagram.txt", "internals_block_table_flowchart.txt"])
def test_gather_follows_printed_table(golden, fixture):
    g = golden(fixture)
    bs = g["block_size"]
    table = [page for _, _, _, page in g["blocks"]]
    pages = max(table) + 1
    # each slot holds a marker encoding (page, offset)
    cache = np.zeros((pages, 1, bs, 2))
    for p in range(pages):
        for o in range(bs):
            cache[p, 0, o] = (p, o)
    rows = attention.gather_sequence(cache, table, g["num_tokens"])
    assert rows.shape == (g["num_tokens"], 1, 2)
    for _, first, last, page in g["blocks"]:
        for tok in range(first, last + 1):
            assert tuple(rows[tok, 0]) == (page, tok - first)


def test_reshape_and_cache_lands_where_gather_reads(golden):
    g = golden("glossary_36_token_diagram.txt")
    bs = g["block_size"]
    table = [page for _, _, _, page in g["blocks"]]
    n = g["num_tokens"]
    kc = np.zeros((16, 2, bs, 3))
    vc = np.zeros_like(kc)
    key = np.arange(n * 2 * 3, dtype=np.float64).reshape(n, 2, 3)
    value = -key
    # slot of token t: its block's page times bs plus its offset inside the block (the diagram)
    slots = []
    for _, first, last, page in g["blocks"]:
        slots += [page * bs + (t - first) for t in range(first, last + 1)]
    cache_ops.reshape_and_cache(key, value, np.array(slots), kc, vc)
    np.testing.assert_array_equal(attention.gather_sequence(kc, table, n), key)
    np.testing.assert_array_equal(attention.gather_sequence(vc, table, n), value)
    # token 35 sits at page 2, offset 3; token 20 at page 14, offset 4
    np.testing.assert_array_equal(kc[2, :, 3], key[35])
    np.testing.assert_array_equal(kc[14, :, 4], key[20])


def test_reshape_and_cache_skips_negative_slots():
    kc = np.zeros((2, 1, 4, 2))
    vc = np.zeros_like(kc)
    key = np.ones((3, 1, 2))
    cache_ops.reshape_and_cache(key, key * 2, np.array([-1, 5, -7]), kc, vc)
    assert kc.sum() == 2 and kc[1, 0, 1].tolist() == [1, 1] and vc[1, 0, 1].tolist() == [2, 2]


def test_copy_blocks_copies_whole_pages():
    rng = np.random.default_rng(0)
    kc = rng.integers(0, 65535, size=(6, 2, 4, 8)).astype(np.uint16)
    vc = rng.integers(0, 65535, size=(6, 2, 4, 8)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    cache_ops.copy_blocks(kc, vc, [(1, 4), (3, 0)])
    np.testing.assert_array_equal(kc[4], k0[1])
    np.testing.assert_array_equal(vc[0], v0[3])
    for p in (1, 2, 3, 5):
        np.testing.assert_array_equal(kc[p], k0[p])
        np.testing.assert_array_equal(vc[p], v0[p])


# -- attention: closed forms -----------------------------------------------------

def test_single_token_returns_its_value():
    rng = np.random.default_rng(1)
    q, kc, vc, tables, _ = _rand_case(rng, 3, 4, 2, 8, 4, 10)
    ctx = np.array([1, 1, 1])
    out = attention.decode_attention(q.astype(np.float32), kc.astype(np.float32), vc.astype(np.float32),
                                     tables, ctx, 0.3, "f32")
    for b in range(3):
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], vc.astype(np.float32)[tables[b, 0], h // 2, 0])


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    bs, ctx = 4, 11
    kc = np.tile(rng.standard_normal((1, 1, 1, 8)), (4, 1, bs, 1)).astype(np.float32)
    vc = rng.standard_normal((4, 1, bs, 8)).astype(np.float32)
    table = np.array([[2, 0, 3]])
    q = rng.standard_normal((1, 2, 8)).astype(np.float32)
    out = attention.decode_attention(q, kc, vc, table, [ctx], 0.7, "f32")
    rows = attention.to_float64(attention.gather_sequence(vc, table[0], ctx), "f32")[:, 0]
    np.testing.assert_allclose(out[0, 0], rows.mean(axis=0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0, 1], rows.mean(axis=0), rtol=0, atol=1e-14)


def test_equal_values_give_that_value():
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((5, 2, 4, 6)).astype(np.float32)
    vc = np.full((5, 2, 4, 6), 0.375, dtype=np.float32)
    tables = np.array([[4, 1, 0, 2], [3, -1, -1, -1]])
    q = rng.standard_normal((2, 4, 6)).astype(np.float32)
    out = attention.decode_attention(q, kc, vc, tables, [14, 3], 0.5, "f32")
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-15)


def test_empty_sequence_gives_zeros():
    kc = np.ones((2, 1, 4, 3), dtype=np.float32)
    out = attention.decode_attention(np.ones((1, 2, 3), np.float32), kc, kc, np.array([[0]]), [0], 1.0, "f32")
    assert not out.any()


def test_two_tokens_closed_form():
    # ctx 2: out = sigmoid(s0 - s1) v0 + sigmoid(s1 - s0) v1
    kc = np.zeros((2, 1, 1, 2))
    vc = np.zeros((2, 1, 1, 2))
    kc[1, 0, 0] = [1.0, 0.0]    # logical 0 -> page 1
    kc[0, 0, 0] = [0.0, 2.0]    # logical 1 -> page 0
    vc[1, 0, 0] = [3.0, -1.0]
    vc[0, 0, 0] = [0.5, 4.0]
    q = np.array([[[0.25, 0.5]]])
    s0, s1 = 2.0 * 0.25, 2.0 * 1.0
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    expect = w0 * np.array([3.0, -1.0]) + (1 - w0) * np.array([0.5, 4.0])
    out = attention.decode_attention(q.astype(np.float32), kc.astype(np.float32), vc.astype(np.float32),
                                     np.array([[1, 0]]), [2], 2.0, "f32")
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-15, atol=1e-15)


# -- attention: library routine, brute force, invariances ----------------------------

@pytest.mark.parametrize("hq,hkv,bs", [(4, 1, 16), (8, 2, 4), (6, 3, 1), (8, 8, 32)])
def test_matches_torch_sdpa_fp64(hq, hkv, bs):
    rng = np.random.default_rng(hq * 10 + hkv + bs)
    q, kc, vc, tables, ctx = _rand_case(rng, 4, hq, hkv, 16, bs, 70)
    out = attention.decode_attention(q, kc, vc, tables, ctx, 0.25, "f32")
    q32 = q.astype(np.float32).astype(np.float64)
    for b in range(4):
        keys = attention.gather_sequence(kc.astype(np.float32).astype(np.float64), tables[b], ctx[b])
        values = attention.gather_sequence(vc.astype(np.float32).astype(np.float64), tables[b], ctx[b])
        np.testing.assert_allclose(out[b], _sdpa(q32[b], keys, values, 0.25), rtol=1e-12, atol=1e-12)


def test_identity_table_equals_contiguous_attention():
    rng = np.random.default_rng(7)
    bs, ctx, hkv, hq, d = 4, 23, 2, 4, 8
    keys = rng.standard_normal((ctx, hkv, d))
    values = rng.standard_normal((ctx, hkv, d))
    pages = -(-ctx // bs)
    kc = np.zeros((pages, hkv, bs, d))
    vc = np.zeros_like(kc)
    for j in range(ctx):          # contiguous storage: token j in page j // bs
        kc[j // bs, :, j % bs] = keys[j]
        vc[j // bs, :, j % bs] = values[j]
    q = rng.standard_normal((1, hq, d))
    out = attention.decode_attention(q, kc, vc, np.arange(pages)[None], [ctx], 0.5, "f32")
    q32 = q.astype(np.float32).astype(np.float64)[0]
    k32 = keys.astype(np.float32).astype(np.float64)
    v32 = values.astype(np.float32).astype(np.float64)
    np.testing.assert_allclose(out[0], _sdpa(q32, k32, v32, 0.5), rtol=1e-12, atol=1e-12)


def test_page_relabelling_leaves_output_unchanged():
    rng = np.random.default_rng(8)
    q, kc, vc, tables, ctx = _rand_case(rng, 5, 8, 2, 8, 4, 40)
    base = attention.decode_attention(q, kc, vc, tables, ctx, 0.4, "f32")
    for trial in range(3):
        perm = rng.permutation(kc.shape[0])          # physical page p moves to perm[p]
        kc2 = np.empty_like(kc)
        vc2 = np.empty_like(vc)
        kc2[perm] = kc
        vc2[perm] = vc
        tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
        out = attention.decode_attention(q, kc2, vc2, tables2, ctx, 0.4, "f32")
        np.testing.assert_array_equal(out, base)


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    bs = int(rng.integers(2, 5))
    q, kc, vc, tables, ctx = _rand_case(rng, 2, 4, 2, 4, bs, 10)
    scale = 0.6
    out = attention.decode_attention(q, kc, vc, tables, ctx, scale, "f32")
    k32, v32, q32 = (a.astype(np.float32).astype(np.float64) for a in (kc, vc, q))
    for b in range(2):
        for h in range(4):
            ref = _brute(q32[b, h], k32, v32, [int(p) for p in tables[b] if p >= 0], int(ctx[b]), h // 2, scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("ctx", [1, 511, 512, 513, 1024, 1500, 4097])
def test_partition_merge_equals_unsplit(ctx):
    rng = np.random.default_rng(ctx)
    keys = rng.standard_normal((ctx, 32))
    values = rng.standard_normal((ctx, 32))
    q = rng.standard_normal(32) * 3.0
    parts = attention.partition_attention(q, keys, values, 0.3)
    assert len(parts) == -(-ctx // 512)
    np.testing.assert_allclose(attention.lse_merge(parts), attention.softmax_attention(q, keys, values, 0.3),
                               rtol=1e-12, atol=1e-13)
    # each partial is itself the attention over its partition
    for i, (o, m, l) in enumerate(parts):
        kp = keys[i * 512:(i + 1) * 512]
        s = 0.3 * kp @ q
        np.testing.assert_allclose(m, s.max(), rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(l, np.exp(s - s.max()).sum(), rtol=1e-13)
        np.testing.assert_allclose(o, attention.softmax_attention(q, kp, values[i * 512:(i + 1) * 512], 0.3),
                                   rtol=1e-12, atol=1e-13)


def test_bf16_widening_is_exact():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F7F, 0x0001], dtype=np.uint16)
    vals = attention.to_float64(bits, "bf16")
    assert vals.tolist()[:5] == [1.0, -2.0, 1.0078125, 0.0, -0.0]
    assert vals[5] == (2 - 2 ** -7) * 2.0 ** 127
    assert vals[6] == 2.0 ** -133
    f16 = np.array([0x3C00, 0xC500], dtype=np.uint16)
    assert attention.to_float64(f16, "f16").tolist() == [1.0, -5.0]


# -- the pins have teeth -------------------------------------------------------------

def _wrong_offset_gather(cache, block_table, context_len):
    bs = cache.shape[2]
    pos = np.arange(context_len)
    pages = np.asarray(block_table)[pos // bs]
    return cache[pages, :, (pos + 1) % bs, :]


def _ignores_table_gather(cache, block_table, context_len):
    bs = cache.shape[2]
    pos = np.arange(context_len)
    return cache[pos // bs, :, pos % bs, :]


def _drops_last_token_gather(cache, block_table, context_len):
    bs = cache.shape[2]
    pos = np.arange(max(context_len - 1, 0))
    return cache[np.asarray(block_table)[pos // bs], :, pos % bs, :]


def _negated_scores(q, keys, values, scale):
    s = -scale * (keys @ q)
    e = np.exp(s - s.max())
    return (e / e.sum()) @ values


def _unscaled(q, keys, values, scale):
    s = keys @ q
    e = np.exp(s - s.max())
    return (e / e.sum()) @ values


def _keys_as_values(q, keys, values, scale):
    s = scale * (keys @ q)
    e = np.exp(s - s.max())
    return (e / e.sum()) @ keys


@pytest.mark.parametrize("where,mutant", [
    ("gather_sequence", _wrong_offset_gather),
    ("gather_sequence", _ignores_table_gather),
    ("gather_sequence", _drops_last_token_gather),
    ("softmax_attention", _negated_scores),
    ("softmax_attention", _unscaled),
    ("softmax_attention", _keys_as_values),
])
def test_planted_mistakes_are_caught(monkeypatch, where, mutant):
    """A plausible mistake planted in the oracle must fail the library or brute-force pin."""
    rng = np.random.default_rng(5)
    q, kc, vc, tables, ctx = _rand_case(rng, 3, 4, 2, 8, 4, 30)
    monkeypatch.setattr(attention, where, mutant)
    out = attention.decode_attention(q, kc, vc, tables, ctx, 0.5, "f32")
    k32, v32, q32 = (a.astype(np.float32).astype(np.float64) for a in (kc, vc, q))
    worst = 0.0
    for b in range(3):
        for h in range(4):
            ref = _brute(q32[b, h], k32, v32, [int(p) for p in tables[b] if p >= 0], int(ctx[b]), h // 2, 0.5)
            worst = max(worst, float(np.max(np.abs(out[b, h] - np.array(ref)))))
    assert worst > 1e-6


def test_planted_grouping_mistake_is_caught(monkeypatch):
    """Reading kv head h % H_kv instead of h // G must fail the torch-SDPA pin."""
    rng = np.random.default_rng(6)
    q, kc, vc, tables, ctx = _rand_case(rng, 2, 8, 2, 8, 4, 30)
    good = attention.decode_attention(q, kc, vc, tables, ctx, 0.5, "f32")

    def wrong_grouping(q_, kcache, vcache, tabs, clens, scale, dtype, seqs=None):
        q64 = attention.to_float64(q_, dtype)
        out = np.zeros(q64.shape)
        hkv = kcache.shape[1]
        for b in range(q64.shape[0]):
            keys = attention.to_float64(attention.gather_sequence(kcache, tabs[b], int(clens[b])), dtype)
            values = attention.to_float64(attention.gather_sequence(vcache, tabs[b], int(clens[b])), dtype)
            for h in range(q64.shape[1]):
                out[b, h] = attention.softmax_attention(q64[b, h], keys[:, h % hkv], values[:, h % hkv], scale)
        return out

    bad = wrong_grouping(q, kc, vc, tables, ctx, 0.5, "f32")
    q32 = q.astype(np.float32).astype(np.float64)
    keys = attention.gather_sequence(kc.astype(np.float32).astype(np.float64), tables[0], ctx[0])
    values = attention.gather_sequence(vc.astype(np.float32).astype(np.float64), tables[0], ctx[0])
    lib = _sdpa(q32[0], keys, values, 0.5)
    np.testing.assert_allclose(good[0], lib, rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(bad[0] - lib)) > 1e-6

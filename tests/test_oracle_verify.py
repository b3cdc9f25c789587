"""Pins of oracle/attention.py's several-query-tokens form (draft verification).

The oracle's ``verify_attention`` is tied to textbook causal self-attention
(torch's own fp64 scaled_dot_product_attention with ``is_causal=True`` over the
whole contiguous sequence: its last T rows), to pure-Python brute force that
walks the block table, and to exact invariances of the causal mask (keys after
a token's position never matter, its own key does).  Planted mistakes in the
mask must fail these pins.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention


def _scatter_case(rng, ctxs, hq, hkv, d, bs, extra_pages=3):
    """Contiguous per-sequence K/V and the same rows scattered into random pages."""
    need = [-(-c // bs) for c in ctxs]
    pages = sum(need) + extra_pages
    perm = rng.permutation(pages)
    mb = max(max(need), 1)
    tables = np.full((len(ctxs), mb), -1, dtype=np.int64)
    kc = rng.standard_normal((pages, hkv, bs, d))
    vc = rng.standard_normal((pages, hkv, bs, d))
    seq_k, seq_v = [], []
    i = 0
    for b, c in enumerate(ctxs):
        tables[b, :need[b]] = perm[i:i + need[b]]
        i += need[b]
        k = rng.standard_normal((c, hkv, d))
        v = rng.standard_normal((c, hkv, d))
        for j in range(c):
            kc[tables[b, j // bs], :, j % bs, :] = k[j]
            vc[tables[b, j // bs], :, j % bs, :] = v[j]
        seq_k.append(k)
        seq_v.append(v)
    return kc, vc, tables, seq_k, seq_v


def _causal_sdpa_last_rows(q_all, k, v, scale, num_tokens):
    """torch fp64 causal self-attention over the whole sequence; its last rows."""
    g = q_all.shape[1] // k.shape[1]
    qt = torch.from_numpy(q_all).permute(1, 0, 2)[None]                         # [1, Hq, ctx, D]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(g, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()[-num_tokens:]                          # [T, Hq, D]


@pytest.mark.parametrize("num_tokens,hq,hkv,bs", [(1, 4, 2, 4), (3, 8, 2, 4), (5, 4, 1, 16), (8, 6, 3, 2)])
def test_verify_is_the_last_rows_of_causal_self_attention(num_tokens, hq, hkv, bs):
    rng = np.random.default_rng(10 + num_tokens)
    ctxs = [num_tokens, num_tokens + 1, 17, 40, 63]
    d = 8
    kc, vc, tables, seq_k, seq_v = _scatter_case(rng, ctxs, hq, hkv, d, bs)
    q_all = [rng.standard_normal((c, hq, d)) for c in ctxs]
    q = np.stack([qa[-num_tokens:] for qa in q_all])
    out = attention.verify_attention(q, kc, vc, tables, np.array(ctxs), 0.37, "f32")
    for b, c in enumerate(ctxs):
        ref = _causal_sdpa_last_rows(q_all[b].astype(np.float32).astype(np.float64),
                                     seq_k[b].astype(np.float32).astype(np.float64),
                                     seq_v[b].astype(np.float32).astype(np.float64), 0.37, num_tokens)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def _brute_row(q_row, kc, vc, table, visible, kvh, scale):
    bs = kc.shape[2]
    scores, rows = [], []
    for j in range(visible):
        page = int(table[j // bs])
        k = kc[page][kvh][j % bs]
        scores.append(scale * sum(float(q_row[i]) * float(k[i]) for i in range(len(q_row))))
        rows.append(vc[page][kvh][j % bs])
    if not scores:
        return [0.0] * len(q_row)
    top = max(scores)
    w = [math.exp(s - top) for s in scores]
    return [sum(w[j] * float(rows[j][i]) for j in range(len(w))) / sum(w) for i in range(len(q_row))]


def test_verify_matches_brute_force_walk_of_the_table():
    rng = np.random.default_rng(21)
    ctxs = [2, 9, 14]
    kc, vc, tables, _, _ = _scatter_case(rng, ctxs, 4, 2, 4, 4)
    num_tokens = 4
    q = rng.standard_normal((3, num_tokens, 4, 4))
    out = attention.verify_attention(q, kc, vc, tables, np.array(ctxs), 0.5, "f32")
    f = lambda a: a.astype(np.float32).astype(np.float64)
    for b, c in enumerate(ctxs):
        for t in range(num_tokens):
            pos = c - num_tokens + t                  # this token's own position
            for h in range(4):
                ref = _brute_row(f(q[b, t, h]), f(kc), f(vc), tables[b], max(0, pos + 1), h // 2, 0.5)
                np.testing.assert_allclose(out[b, t, h], ref, rtol=0, atol=1e-12)


def test_tokens_before_the_context_see_nothing():
    """More query tokens than context: the ones with a negative position give zeros."""
    rng = np.random.default_rng(22)
    kc, vc, tables, seq_k, seq_v = _scatter_case(rng, [3], 2, 1, 8, 4)
    q = rng.standard_normal((1, 5, 2, 8))
    out = attention.verify_attention(q, kc, vc, tables, np.array([3]), 0.3, "f32")
    assert np.all(out[0, :2] == 0.0)
    f = lambda a: a.astype(np.float32).astype(np.float64)
    q_all = f(q[0, 2:])
    ref = _causal_sdpa_last_rows(q_all, f(seq_k[0]), f(seq_v[0]), 0.3, 3)
    np.testing.assert_allclose(out[0, 2:], ref, rtol=0, atol=1e-12)


def test_keys_after_a_token_never_matter_and_its_own_key_does():
    rng = np.random.default_rng(23)
    ctx, num_tokens, bs = 21, 4, 4
    kc, vc, tables, _, _ = _scatter_case(rng, [ctx], 4, 2, 8, bs)
    q = rng.standard_normal((1, num_tokens, 4, 8))
    base = attention.verify_attention(q, kc, vc, tables, np.array([ctx]), 0.4, "f32")
    for t in range(num_tokens):
        pos = ctx - num_tokens + t
        later = kc.copy(), vc.copy()
        for j in range(pos + 1, ctx):
            later[0][tables[0, j // bs], :, j % bs, :] += 5.0
            later[1][tables[0, j // bs], :, j % bs, :] -= 3.0
        moved = attention.verify_attention(q, later[0], later[1], tables, np.array([ctx]), 0.4, "f32")
        assert np.array_equal(moved[0, t], base[0, t])
        own = kc.copy()
        own[tables[0, pos // bs], :, pos % bs, :] += 1.0
        moved = attention.verify_attention(q, own, vc, tables, np.array([ctx]), 0.4, "f32")
        assert np.max(np.abs(moved[0, t] - base[0, t])) > 1e-6


def test_one_query_token_is_a_decode_step():
    rng = np.random.default_rng(24)
    ctxs = [1, 30, 47]
    kc, vc, tables, _, _ = _scatter_case(rng, ctxs, 8, 2, 16, 8)
    q = rng.standard_normal((3, 1, 8, 16))
    out = attention.verify_attention(q, kc, vc, tables, np.array(ctxs), 0.25, "f32")
    dec = attention.decode_attention(q[:, 0], kc, vc, tables, np.array(ctxs), 0.25, "f32")
    np.testing.assert_allclose(out[:, 0], dec, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mutant", [
    lambda c, n, t: max(0, c - n + t),          # a token misses its own key
    lambda c, n, t: max(0, c - t),              # tokens in reverse order
    lambda c, n, t: c,                          # no causal mask
    lambda c, n, t: max(0, c - n + t + 2),      # a token sees the next one
])
def test_planted_mask_mistakes_are_caught(monkeypatch, mutant):
    rng = np.random.default_rng(25)
    ctxs = [9, 26]
    num_tokens = 3
    kc, vc, tables, seq_k, seq_v = _scatter_case(rng, ctxs, 4, 2, 8, 4)
    q_all = [rng.standard_normal((c, 4, 8)) for c in ctxs]
    q = np.stack([qa[-num_tokens:] for qa in q_all])
    monkeypatch.setattr(attention, "visible_keys", lambda c, n, t: min(c, mutant(c, n, t)))
    out = attention.verify_attention(q, kc, vc, tables, np.array(ctxs), 0.5, "f32")
    f = lambda a: a.astype(np.float32).astype(np.float64)
    worst = max(float(np.max(np.abs(out[b] - _causal_sdpa_last_rows(f(q_all[b]), f(seq_k[b]), f(seq_v[b]), 0.5,
                                                                    num_tokens))))
                for b in range(2))
    assert worst > 1e-6

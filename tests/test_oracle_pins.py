"""Pins for the oracle: checks against things other than the oracle itself.

Each test would fail for a plausible mistake in the oracle: a dropped scale,
an off-by-one causal bound, a wrong GQA group index, a transposed operand,
a wrong page/slot index or a misaligned chunk.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _f64(t):
    return t.to(torch.float64).numpy()


def _tiny(seqlens, H, G, d, seed, bs=16, scale=None):
    return W.make_workload(seqlens, H, G, d, block_size=bs, seed=seed, scale=scale)


# ---------------------------------------------------------------- P1
@pytest.mark.parametrize("seqlens,H,G,d", [([37], 4, 2, 16), ([5, 70, 1], 6, 3, 32)])
def test_softmax_rows_sum_to_one(seqlens, H, G, d):
    w = _tiny(seqlens, H, G, d, seed=11)
    for row in [0, 1, w.total_tokens // 2, w.total_tokens - 1]:
        for h in range(H):
            p = oracle.softmax_weights(w.q, w.k, w.v, w.cu_seqlens, H, G, d, w.scale, row, h)
            assert abs(p.sum() - 1.0) < 1e-12
            assert (p >= 0).all()


def test_softmax_weights_chunked_sum_to_one():
    w = _tiny([200], 4, 2, 16, seed=12, bs=16)
    cache = oracle.kv_write(w.k[:120], w.v[:120], torch.tensor([0, 120], dtype=torch.int32),
                            w.empty_cache(), w.block_table, 16)
    q, k, v = w.q[120:], w.k[120:], w.v[120:]
    cu = torch.tensor([0, 80], dtype=torch.int32)
    for row in (0, 79):
        p = oracle.softmax_weights(q, k, v, cu, 4, 2, 16, w.scale, row, 3,
                                   context_lens=[120], kv_cache=cache, block_table=w.block_table)
        assert len(p) == 120 + row + 1
        assert abs(p.sum() - 1.0) < 1e-12


# ---------------------------------------------------------------- P2
def test_first_row_outputs_v0_exactly():
    w = _tiny([9, 33, 1, 64], 8, 2, 64, seed=13)
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 8, 2, 64, w.scale)
    v = _f64(w.v)
    for i in range(w.num_seqs):
        t = int(w.cu_seqlens[i])
        for h in range(8):
            assert np.array_equal(out[t, h], v[t, h // 4])


# ---------------------------------------------------------------- P3
def test_identical_keys_give_prefix_mean():
    w = _tiny([50], 4, 4, 32, seed=14)
    k = w.k.clone()
    k[:] = k[0:1]  # every key equal
    out = oracle.attention(w.q, k, w.v, w.cu_seqlens, 4, 4, 32, w.scale)
    v = _f64(w.v)
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, 51)[:, None, None]
    assert np.max(np.abs(out - prefix_mean)) < 1e-12


def test_zero_query_gives_prefix_mean():
    w = _tiny([40, 23], 4, 2, 16, seed=15)
    q = torch.zeros_like(w.q)
    out = oracle.attention(q, w.k, w.v, w.cu_seqlens, 4, 2, 16, w.scale)
    v = _f64(w.v)
    for i in range(2):
        a, b = int(w.cu_seqlens[i]), int(w.cu_seqlens[i + 1])
        pm = np.cumsum(v[a:b], axis=0) / np.arange(1, b - a + 1)[:, None, None]
        for h in range(4):
            assert np.max(np.abs(out[a:b, h] - pm[:, h // 2])) < 1e-12


# ---------------------------------------------------------------- P4
@pytest.mark.parametrize("H,G", [(8, 2), (6, 3), (4, 1)])
def test_gqa_equals_mha_with_repeated_kv(H, G):
    w = _tiny([45, 17], H, G, 16, seed=16)
    r = H // G
    k_rep = w.k.repeat_interleave(r, dim=1)
    v_rep = w.v.repeat_interleave(r, dim=1)
    out_gqa = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, H, G, 16, w.scale)
    out_mha = oracle.attention(w.q, k_rep, v_rep, w.cu_seqlens, H, H, 16, w.scale)
    assert np.array_equal(out_gqa, out_mha)


# ---------------------------------------------------------------- P5
def _brute_force(q, k, v, cu, H, G, scale):
    """Independent per-element loop: no max subtraction, exp directly."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, _, d = q.shape
    out = np.zeros((T, H, d))
    for i in range(len(cu) - 1):
        a0, a1 = int(cu[i]), int(cu[i + 1])
        for h in range(H):
            g = h * G // H
            for a in range(a0, a1):
                num = np.zeros(d)
                den = 0.0
                for b in range(a0, a + 1):
                    s = 0.0
                    for x in range(d):
                        s += q[a, h, x] * k[b, g, x]
                    e = math.exp(s * scale)
                    den += e
                    for x in range(d):
                        num[x] += e * v[b, g, x]
                out[a, h] = num / den
    return out


@pytest.mark.parametrize("seqlens,H,G,d", [([9], 4, 2, 4), ([3, 7, 1], 2, 1, 3), ([8], 4, 4, 4)])
def test_brute_force_tiny(seqlens, H, G, d):
    w = _tiny(seqlens, H, G, d, seed=17, scale=0.37)
    # small magnitudes so exp() without max subtraction is safe
    q = (w.q.float() * 0.5).to(torch.bfloat16)
    out = oracle.attention(q, w.k, w.v, w.cu_seqlens, H, G, d, 0.37)
    ref = _brute_force(q, w.k, w.v, w.cu_seqlens, H, G, 0.37)
    assert np.max(np.abs(out - ref)) < 1e-12


# ---------------------------------------------------------------- P6
@pytest.mark.parametrize("seqlens,H,G,d", [([128], 4, 4, 64), ([300, 129, 2], 8, 2, 32)])
def test_matches_torch_sdpa_fp64(seqlens, H, G, d):
    w = _tiny(seqlens, H, G, d, seed=18)
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, H, G, d, w.scale)
    for i in range(w.num_seqs):
        a, b = int(w.cu_seqlens[i]), int(w.cu_seqlens[i + 1])
        q = w.q[a:b].to(torch.float64).transpose(0, 1)  # [H, s, d]
        k = w.k[a:b].to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
        v = w.v[a:b].to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=w.scale)
        assert np.max(np.abs(out[a:b] - ref.transpose(0, 1).numpy())) < 1e-10


def test_chunk_matches_torch_sdpa_with_explicit_mask():
    """Bottom-right alignment: chunk row a sees keys 0..ctx+a."""
    H, G, d, ctx, L = 4, 2, 32, 70, 45
    w = _tiny([ctx + L], H, G, d, seed=19, bs=16)
    cache = oracle.kv_write(w.k[:ctx], w.v[:ctx], torch.tensor([0, ctx], dtype=torch.int32),
                            w.empty_cache(), w.block_table, 16)
    out = oracle.attention(w.q[ctx:], w.k[ctx:], w.v[ctx:], torch.tensor([0, L], dtype=torch.int32),
                           H, G, d, w.scale, context_lens=[ctx], kv_cache=cache,
                           block_table=w.block_table, block_size=16)
    q = w.q[ctx:].to(torch.float64).transpose(0, 1)
    k = w.k.to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
    v = w.v.to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
    mask = torch.arange(ctx + L)[None, :] <= (ctx + torch.arange(L))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=w.scale)
    assert np.max(np.abs(out - ref.transpose(0, 1).numpy())) < 1e-10


# ---------------------------------------------------------------- P7
@pytest.mark.parametrize("chunk,bs", [(64, 16), (100, 16), (37, 32)])
def test_chunked_equals_unchunked(chunk, bs):
    H, G, d, s = 4, 2, 32, 260
    w = _tiny([s], H, G, d, seed=20, bs=bs)
    full_out, full_cache = oracle.prefill(w)
    cache = w.empty_cache()
    outs = []
    for q, k, v, cu, ctx, bt in W.chunk_views(w, chunk):
        out = oracle.attention(q, k, v, cu, H, G, d, w.scale, context_lens=ctx, kv_cache=cache,
                               block_table=bt, block_size=bs)
        cache = oracle.kv_write(k, v, cu, cache, bt, bs, context_lens=ctx)
        outs.append(out)
    out = np.concatenate(outs, axis=0)
    assert np.max(np.abs(out - full_out)) < 1e-12
    assert torch.equal(cache.view(torch.int16), full_cache.view(torch.int16))


# ---------------------------------------------------------------- P8
def test_varlen_equals_separate_calls():
    lens = [33, 1, 80, 17]
    H, G, d = 4, 2, 16
    w = _tiny(lens, H, G, d, seed=21)
    out, _ = oracle.prefill(w)
    for i, n in enumerate(lens):
        a, b = int(w.cu_seqlens[i]), int(w.cu_seqlens[i + 1])
        o1 = oracle.attention(w.q[a:b], w.k[a:b], w.v[a:b], torch.tensor([0, n], dtype=torch.int32),
                              H, G, d, w.scale)
        assert np.array_equal(out[a:b], o1)


# ---------------------------------------------------------------- P9
def test_block_table_invariance_and_gather():
    lens = [40, 75]
    H, G, d, bs = 4, 2, 16, 16
    w1 = _tiny(lens, H, G, d, seed=22, bs=bs)
    out1, cache1 = oracle.prefill(w1)
    # same tensors, another page assignment with spare pages in the pool
    w2 = W.make_workload(lens, H, G, d, block_size=bs, seed=22, extra_pages=5)
    assert torch.equal(w2.q, w1.q) and not torch.equal(w2.block_table, w1.block_table)
    out2, cache2 = oracle.prefill(w2)
    assert np.array_equal(out1, out2)
    # gather the cache through the table: bit-exact K/V; unused pages keep the sentinel
    for w, cache in ((w1, cache1), (w2, cache2)):
        c16 = cache.view(torch.int16)
        used = set()
        for i, n in enumerate(lens):
            a = int(w.cu_seqlens[i])
            for t in range(n):
                page = int(w.block_table[i, t // bs])
                used.add(page)
                assert torch.equal(c16[page, 0, t % bs], w.k[a + t].view(torch.int16))
                assert torch.equal(c16[page, 1, t % bs], w.v[a + t].view(torch.int16))
            # slots past the end of a partially filled last page stay untouched
            last = int(w.block_table[i, (n - 1) // bs])
            tail = c16[last, :, n % bs:] if n % bs else c16[last, :, bs:]
            assert (tail == W.sentinel_value_int16()).all()
        for p in range(w.num_blocks):
            if p not in used:
                assert (c16[p] == W.sentinel_value_int16()).all()


def test_chunk_prefix_read_through_table():
    """Prefix keys come from the cache through the table, not the input rows."""
    H, G, d, bs, ctx, L = 2, 1, 8, 16, 48, 20
    w = _tiny([ctx + L], H, G, d, seed=23, bs=bs)
    cache = oracle.kv_write(w.k[:ctx], w.v[:ctx], torch.tensor([0, ctx], dtype=torch.int32),
                            w.empty_cache(), w.block_table, bs)
    args = (w.q[ctx:], w.k[ctx:], w.v[ctx:], torch.tensor([0, L], dtype=torch.int32), H, G, d, w.scale)
    base = oracle.attention(*args, context_lens=[ctx], kv_cache=cache, block_table=w.block_table, block_size=bs)
    # corrupt one prefix V row in the cache -> every output row must move
    c2 = cache.clone()
    page = int(w.block_table[0, 5 // bs])
    c2[page, 1, 5 % bs] = c2[page, 1, 5 % bs] + 1.0
    moved = oracle.attention(*args, context_lens=[ctx], kv_cache=c2, block_table=w.block_table, block_size=bs)
    assert (np.abs(moved - base).max(axis=2) > 0).all()


# ---------------------------------------------------------------- P10
def test_kv_write_bytes_match_page_figures():
    g = json.load(open(GOLDEN))
    for key, H, G in (("kv_bytes_per_token_per_layer_mha", 32, 32),
                      ("kv_bytes_per_token_per_layer_gqa8", 32, 8)):
        T = 2048 if G == 32 else 8192
        w = W.make_workload([T], H, G, 128, block_size=16, seed=24)
        before = w.empty_cache().view(torch.int16)
        after = oracle.kv_write(w.k, w.v, w.cu_seqlens, w.empty_cache(), w.block_table, 16).view(torch.int16)
        changed_bytes = int((after != before).sum()) * 2
        assert changed_bytes == T * g[key]["value"]
        assert changed_bytes == 32 * 2**20  # both shapes write 32 MiB


def test_page_size_figures():
    g = json.load(open(GOLDEN))
    gib = 2**30
    assert 32 * 32768 * g["kv_bytes_per_token_per_layer_mha"]["value"] == g["kv_cache_32_layers_32k_ctx_mha_gib"]["value"] * gib
    assert 32 * 32768 * g["kv_bytes_per_token_per_layer_gqa8"]["value"] == g["kv_cache_32_layers_32k_ctx_gqa8_gib"]["value"] * gib
    assert 8192 * 8192 * 32 * 2 == g["score_matrix_8k_32_heads_fp16_gib"]["value"] * gib
    assert 3 * 128 * 128 * 2 == g["qkv_block_128_d128_fp16_kib"]["value"] * 1024
    e = g["kv_formula_28_layers_40_heads_4096_tokens_gb"]
    assert abs(2 * 28 * 40 * 128 * 4096 * 2 / 1e9 - e["value"]) < e["tolerance"]


def test_scale_of_named_workloads_matches_page():
    g = json.load(open(GOLDEN))["inverse_scale_head_dim_128"]
    w = W.make_workload([4], 4, 4, 128, seed=1)
    assert abs(1.0 / w.scale - g["value"]) < g["tolerance"]


# ---------------------------------------------------------------- misc
def test_scale_enters_scores():
    """Doubling the scale must change the output (a dropped scale would not)."""
    w = _tiny([30], 2, 2, 16, seed=25)
    o1 = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 2, 2, 16, 0.25)
    o2 = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 2, 2, 16, 0.5)
    assert np.abs(o1 - o2)[1:].max() > 1e-3


def test_rows_api_matches_full():
    w = _tiny([77, 51], 4, 2, 32, seed=26)
    full = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 32, w.scale)
    rows = [0, 5, 76, 77, 127]
    heads = [0, 3, 1, 2, 3]
    sel = oracle.attention_rows(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 32, w.scale, rows, heads)
    for s, (r, h) in enumerate(zip(rows, heads)):
        assert np.array_equal(sel[s], full[r, h])


def test_bad_block_table_is_reported():
    w = _tiny([20], 2, 2, 8, seed=27)
    bt = w.block_table.clone()
    bt[0, 1] = w.num_blocks + 3
    with pytest.raises(RuntimeError):
        oracle.kv_write(w.k, w.v, w.cu_seqlens, w.empty_cache(), bt, 16)


# ---------------------------------------------------------------- sliding window
# A window of W keys (lnwmold.com/news/496245 §4.1): row P sees keys
# max(0, P-W+1) .. P.  Pinned by closed forms (W = 1; identical keys), by
# reduction to plain causal attention (a wide window; a truncated sequence),
# by torch's fp64 SDPA with an explicit band mask, and by a brute-force loop.

def test_window_one_outputs_own_value_exactly():
    w = _tiny([9, 33, 1, 64], 8, 2, 64, seed=40)
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 8, 2, 64, w.scale, window=1)
    v = _f64(w.v)
    for h in range(8):
        assert np.array_equal(out[:, h], v[:, h // 4])


def test_wide_window_equals_plain_causal():
    w = _tiny([70, 5, 129], 4, 2, 32, seed=41)
    plain = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 32, w.scale)
    for win in (129, 130, 10_000):
        out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 32, w.scale, window=win)
        assert np.array_equal(out, plain)
    # one key too narrow changes the last row of the longest sequence
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 32, w.scale, window=128)
    assert not np.array_equal(out[-1], plain[-1])
    assert np.array_equal(out[:-1], plain[:-1])


def test_window_equals_causal_on_truncated_sequence():
    """Row a under window W is the last row of plain causal attention over
    tokens a-W+1 .. a alone (positions only enter through the mask)."""
    H, G, d, s, win = 4, 2, 16, 90, 23
    w = _tiny([s], H, G, d, seed=42)
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, H, G, d, w.scale, window=win)
    for a in (0, 5, 21, 22, 23, 50, 89):
        b0 = max(0, a - win + 1)
        n = a + 1 - b0
        o1 = oracle.attention(w.q[b0:a + 1], w.k[b0:a + 1], w.v[b0:a + 1], torch.tensor([0, n], dtype=torch.int32),
                              H, G, d, w.scale)
        assert np.max(np.abs(out[a] - o1[-1])) < 1e-13


def _band_mask(q_pos, n_keys, win):
    j = torch.arange(n_keys)[None, :]
    P = q_pos[:, None]
    return (j <= P) & (j > P - win)


@pytest.mark.parametrize("seqlens,win", [([300, 129, 2], 64), ([200], 1), ([150], 149)])
def test_window_matches_torch_sdpa_band_mask(seqlens, win):
    H, G, d = 8, 2, 32
    w = _tiny(seqlens, H, G, d, seed=43)
    out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, H, G, d, w.scale, window=win)
    for i in range(w.num_seqs):
        a, b = int(w.cu_seqlens[i]), int(w.cu_seqlens[i + 1])
        q = w.q[a:b].to(torch.float64).transpose(0, 1)
        k = w.k[a:b].to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
        v = w.v[a:b].to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
        mask = _band_mask(torch.arange(b - a), b - a, win)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=w.scale)
        assert np.max(np.abs(out[a:b] - ref.transpose(0, 1).numpy())) < 1e-10


def test_window_chunk_matches_torch_sdpa_band_mask():
    """Chunked mode: the window is counted in absolute positions, so it
    reaches back into the cached prefix."""
    H, G, d, ctx, L, win = 4, 2, 32, 70, 45, 50
    w = _tiny([ctx + L], H, G, d, seed=44, bs=16)
    cache = oracle.kv_write(w.k[:ctx], w.v[:ctx], torch.tensor([0, ctx], dtype=torch.int32),
                            w.empty_cache(), w.block_table, 16)
    out = oracle.attention(w.q[ctx:], w.k[ctx:], w.v[ctx:], torch.tensor([0, L], dtype=torch.int32),
                           H, G, d, w.scale, context_lens=[ctx], kv_cache=cache,
                           block_table=w.block_table, block_size=16, window=win)
    q = w.q[ctx:].to(torch.float64).transpose(0, 1)
    k = w.k.to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
    v = w.v.to(torch.float64).repeat_interleave(H // G, 1).transpose(0, 1)
    mask = _band_mask(ctx + torch.arange(L), ctx + L, win)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=w.scale)
    assert np.max(np.abs(out - ref.transpose(0, 1).numpy())) < 1e-10


def test_window_brute_force_tiny():
    H, G, d, win = 4, 2, 3, 3
    w = _tiny([9, 4], H, G, d, seed=45, scale=0.41)
    q = (w.q.float() * 0.5).to(torch.bfloat16)
    out = oracle.attention(q, w.k, w.v, w.cu_seqlens, H, G, d, 0.41, window=win)
    qq, kk, vv = _f64(q), _f64(w.k), _f64(w.v)
    for i in range(w.num_seqs):
        a0, a1 = int(w.cu_seqlens[i]), int(w.cu_seqlens[i + 1])
        for h in range(H):
            g = h * G // H
            for a in range(a0, a1):
                num, den = np.zeros(d), 0.0
                for b in range(a0, a + 1):
                    if a - b >= win:
                        continue
                    e = math.exp(0.41 * sum(qq[a, h, x] * kk[b, g, x] for x in range(d)))
                    den += e
                    num += e * vv[b, g]
                assert np.max(np.abs(out[a, h] - num / den)) < 1e-12


def test_window_weights_and_identical_keys():
    H, G, d, win = 4, 4, 32, 7
    w = _tiny([50], H, G, d, seed=46)
    for row in (0, 3, 6, 7, 49):
        p = oracle.softmax_weights(w.q, w.k, w.v, w.cu_seqlens, H, G, d, w.scale, row, 2, window=win)
        assert len(p) == row + 1
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.count_nonzero(p) == min(row + 1, win)
        assert (p[: max(0, row - win + 1)] == 0).all()
    k = w.k.clone()
    k[:] = k[0:1]
    out = oracle.attention(w.q, k, w.v, w.cu_seqlens, H, G, d, w.scale, window=win)
    v = _f64(w.v)
    for a in range(50):
        b0 = max(0, a - win + 1)
        assert np.max(np.abs(out[a] - v[b0:a + 1].mean(axis=0))) < 1e-12


def test_window_chunked_equals_unchunked():
    H, G, d, s, bs, win = 4, 2, 32, 260, 16, 75
    w = _tiny([s], H, G, d, seed=47, bs=bs)
    full_out, full_cache = oracle.prefill(w, window=win)
    cache = w.empty_cache()
    outs = []
    for q, k, v, cu, ctx, bt in W.chunk_views(w, 64):
        outs.append(oracle.attention(q, k, v, cu, H, G, d, w.scale, context_lens=ctx, kv_cache=cache,
                                     block_table=bt, block_size=bs, window=win))
        cache = oracle.kv_write(k, v, cu, cache, bt, bs, context_lens=ctx)
    assert np.max(np.abs(np.concatenate(outs, axis=0) - full_out)) < 1e-12
    assert torch.equal(cache.view(torch.int16), full_cache.view(torch.int16))


# ---------------------------------------------------------------- fused QKV projection
# hncyxsy.com/news/270449 §4.1 / §2.2: y = x W^T with W = [W_q; W_k; W_v] (one row
# per output feature), cut by columns into Q, K, V, each reshaped head-dim last.

def test_qkv_projection_brute_force_tiny():
    g = torch.Generator().manual_seed(50)
    T, hid, H, G, d = 3, 5, 2, 1, 2
    x = torch.randn(T, hid, generator=g).to(torch.bfloat16)
    w = torch.randn((H + 2 * G) * d, hid, generator=g).to(torch.bfloat16)
    q, k, v = oracle.qkv_projection(x, w, H, G, d)
    xs, ws = _f64(x), _f64(w)
    for t in range(T):
        for n in range((H + 2 * G) * d):
            y = sum(xs[t, c] * ws[n, c] for c in range(hid))
            if n < H * d:
                got = q[t, n // d, n % d]
            elif n < (H + G) * d:
                got = k[t, (n - H * d) // d, (n - H * d) % d]
            else:
                got = v[t, (n - (H + G) * d) // d, (n - (H + G) * d) % d]
            assert abs(got - y) < 1e-12


def test_qkv_projection_one_hot_weights_select_features():
    """W rows one-hot: output feature n copies input feature perm[n], so every
    element of Q, K and V is a known input element (checks the column order
    Q | K | V and the head-dim-last reshape)."""
    g = torch.Generator().manual_seed(51)
    T, H, G, d = 4, 4, 2, 8
    N = (H + 2 * G) * d
    hid = N
    x = torch.randn(T, hid, generator=g).to(torch.bfloat16)
    perm = torch.randperm(hid, generator=g)
    w = torch.zeros(N, hid)
    w[torch.arange(N), perm] = 1.0
    q, k, v = oracle.qkv_projection(x, w.to(torch.bfloat16), H, G, d)
    xs = _f64(x)
    for h in range(H):
        for e in range(d):
            assert np.array_equal(q[:, h, e], xs[:, perm[h * d + e]])
    for gg in range(G):
        for e in range(d):
            assert np.array_equal(k[:, gg, e], xs[:, perm[H * d + gg * d + e]])
            assert np.array_equal(v[:, gg, e], xs[:, perm[(H + G) * d + gg * d + e]])


def test_qkv_projection_matches_torch_linear_fp64():
    g = torch.Generator().manual_seed(52)
    T, hid, H, G, d = 37, 96, 4, 2, 16
    x = torch.randn(T, hid, generator=g).to(torch.bfloat16)
    w = torch.randn((H + 2 * G) * d, hid, generator=g).to(torch.bfloat16)
    q, k, v = oracle.qkv_projection(x, w, H, G, d)
    ref = torch.nn.functional.linear(x.to(torch.float64), w.to(torch.float64)).numpy()
    got = np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], axis=1)
    assert np.max(np.abs(got - ref)) < 1e-12


# ---------------------------------------------------------------- output projection
# hncyxsy.com/news/270449 §3.3: the heads' outputs (s, n_head, head_dim) are
# flattened back to (s, h) head after head, then one plain GEMM with W_o.

def test_out_projection_brute_force_tiny():
    g = torch.Generator().manual_seed(53)
    T, H, d, hid = 3, 2, 3, 4
    o = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    w = torch.randn(hid, H * d, generator=g).to(torch.bfloat16)
    y = oracle.out_projection(o, w)
    os_, ws = _f64(o), _f64(w)
    for t in range(T):
        for n in range(hid):
            ref = sum(os_[t, h, e] * ws[n, h * d + e] for h in range(H) for e in range(d))
            assert abs(y[t, n] - ref) < 1e-12


def test_out_projection_head_block_selects_that_head():
    """W_o zero except an identity block under head h's input features: y is
    head h's output exactly (checks that merged feature h*d + e is (h, e))."""
    g = torch.Generator().manual_seed(54)
    T, H, d = 5, 3, 4
    o = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    for h in range(H):
        w = torch.zeros(d, H * d)
        w[:, h * d:(h + 1) * d] = torch.eye(d)
        y = oracle.out_projection(o, w.to(torch.bfloat16))
        assert np.array_equal(y, _f64(o)[:, h, :])

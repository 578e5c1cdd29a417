"""Pins for the FP8 (e4m3) KV-cache oracle: the code table, rounding to the
nearest code with ties to even, saturation, a cross-check against torch's own
float8_e4m3fn conversion, the paged FP8 write, and decode over an FP8 cache
reducing to the bf16 definition when every value is exactly representable."""
import math

import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import workloads as W

FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_code_table_values():
    cases = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x3F: 1.875, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9,
             0x08: 2.0 ** -6, 0x30: 0.5, 0x46: 3.5, 0xC0: -2.0, 0xFE: -448.0}
    for c, v in cases.items():
        assert oracle.e4m3_decode(c) == v, hex(c)
    assert math.copysign(1.0, oracle.e4m3_decode(0x80)) == -1.0 and oracle.e4m3_decode(0x80) == 0.0
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))


def test_every_finite_code_round_trips():
    for c in FINITE:
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c, hex(c)


def test_midpoints_round_to_the_even_code():
    pos = sorted((oracle.e4m3_decode(c), c) for c in FINITE if c < 0x80)
    for (a, ca), (b, cb) in zip(pos, pos[1:]):
        mid = np.float32((a + b) / 2)  # exact in fp32: codes have at most 4 significant bits
        assert float(mid) == (a + b) / 2
        want = ca if ca % 2 == 0 else cb
        assert oracle.e4m3_encode(float(mid)) == want, (a, b)
        assert oracle.e4m3_encode(-float(mid)) == want | 0x80
        assert oracle.e4m3_encode(float(np.nextafter(mid, np.float32(0)))) == ca
        assert oracle.e4m3_encode(float(np.nextafter(mid, np.float32(1e9)))) == cb


def test_saturation():
    for x, c in [(448.0, 0x7E), (460.0, 0x7E), (464.0, 0x7E), (1e6, 0x7E), (float("inf"), 0x7E), (-1e6, 0xFE),
                 (-470.0, 0xFE)]:
        assert oracle.e4m3_encode(x) == c, x


def test_matches_torch_float8_e4m3fn_in_range():
    g = torch.Generator().manual_seed(60)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 120.0)])
    x = x.clamp(-448, 448).to(torch.float32)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x.numpy()], dtype=np.uint8)
    assert np.array_equal(got, ref)


def _fp8_cache(w):
    return torch.full((w.num_blocks, 2, w.block_size, w.n_kv_head, w.head_dim), 0xA5, dtype=torch.uint8)


def test_kv_write_fp8_bytes_and_untouched_slots():
    w = W.make_workload([37, 5], 4, 2, 16, block_size=16, seed=61, extra_pages=2)
    ks, vs = torch.tensor([0.02, 0.5]), torch.tensor([0.1, 1.5])
    cache = oracle.kv_write_fp8(w.k, w.v, w.cu_seqlens, _fp8_cache(w), w.block_table, 16, ks, vs)
    touched = np.zeros(cache.shape, dtype=bool)
    for i, n in enumerate(w.seqlens):
        for t in range(n):
            page, slot = int(w.block_table[i, t // 16]), t % 16
            row = int(w.cu_seqlens[i]) + t
            for g in range(2):
                for which, src, sc in ((0, w.k, ks), (1, w.v, vs)):
                    vals = src[row, g].to(torch.float32)
                    want = [oracle.e4m3_encode(float(np.float32(x) / np.float32(sc[g]))) for x in vals.numpy()]
                    assert cache[page, which, slot, g].tolist() == want
                    touched[page, which, slot, g] = True
    assert (cache.numpy()[~touched] == 0xA5).all()


def _decode_inputs(lens, H, G, d, seed, exact):
    w = W.make_workload(lens, H, G, d, block_size=16, seed=seed, extra_pages=2)
    pq, pk, pv, pcu, q, k, v, ctx = W.decode_views(w)
    ks = torch.full((G,), 0.125) if exact else torch.linspace(0.01, 0.03, G)
    vs = torch.full((G,), 0.25) if exact else torch.linspace(0.02, 0.05, G)
    if exact:  # values that are e4m3 codes times a power-of-two scale: quantization is exact
        gen = torch.Generator().manual_seed(seed + 1)
        codes_k = torch.randint(0, 0x7F, pk.shape, generator=gen).to(torch.float64)
        pk = torch.tensor([[[oracle.e4m3_decode(int(c)) for c in row] for row in blk] for blk in codes_k.tolist()],
                          dtype=torch.float64)
        pk = (pk * 0.125).to(torch.bfloat16)
        pv = (pk.to(torch.float64) * 2.0).to(torch.bfloat16)  # codes times 0.25
        k = (torch.tensor([[[oracle.e4m3_decode(int(c)) for c in row] for row in blk]
                           for blk in torch.randint(0, 0x7F, k.shape, generator=gen).tolist()]) * 0.125).to(torch.bfloat16)
        v = (k.to(torch.float64) * 2.0).to(torch.bfloat16)
    return w, pq, pk, pv, pcu, q, k, v, ctx, ks, vs


def test_decode_fp8_equals_bf16_definition_when_values_are_exact():
    H, G, d = 4, 2, 16
    w, pq, pk, pv, pcu, q, k, v, ctx, ks, vs = _decode_inputs([40, 1, 17], H, G, d, seed=62, exact=True)
    cache8 = oracle.kv_write_fp8(pk, pv, pcu, _fp8_cache(w), w.block_table, 16, ks, vs)
    out8 = oracle.decode_fp8(q, k, v, ctx, H, G, d, w.scale, ks, vs, cache8, w.block_table, 16)
    cache = oracle.kv_write(pk, pv, pcu, w.empty_cache(), w.block_table, 16)
    B = len(w.seqlens)
    ref = oracle.attention(q, k, v, torch.arange(B + 1, dtype=torch.int32), H, G, d, w.scale, context_lens=ctx,
                           kv_cache=cache, block_table=w.block_table, block_size=16)
    assert np.max(np.abs(out8 - ref)) < 1e-12


def test_decode_fp8_empty_context_returns_dequantized_value():
    H, G, d = 4, 2, 16
    w, pq, pk, pv, pcu, q, k, v, ctx, ks, vs = _decode_inputs([1, 1], H, G, d, seed=63, exact=False)
    out8 = oracle.decode_fp8(q, k, v, ctx, H, G, d, w.scale, ks, vs, _fp8_cache(w), w.block_table, 16)
    for i in range(2):
        for h in range(H):
            g = h // (H // G)
            want = [oracle.e4m3_decode(oracle.e4m3_encode(float(np.float32(x) / np.float32(vs[g])))) * float(vs[g])
                    for x in v[i, g].to(torch.float32).numpy()]
            assert np.allclose(out8[i, h], want, rtol=0, atol=1e-15)


def test_decode_fp8_close_to_bf16_attention():
    """Quantization changes the keys and values by at most half a code step
    (relative 2^-4): the outputs stay close to the unquantized definition."""
    H, G, d = 8, 2, 64
    w, pq, pk, pv, pcu, q, k, v, ctx, ks, vs = _decode_inputs([300, 2, 129], H, G, d, seed=64, exact=False)
    ks = torch.full((G,), 4.0 / 448)
    vs = torch.full((G,), 6.0 / 448)
    cache8 = oracle.kv_write_fp8(pk, pv, pcu, _fp8_cache(w), w.block_table, 16, ks, vs)
    out8 = oracle.decode_fp8(q, k, v, ctx, H, G, d, w.scale, ks, vs, cache8, w.block_table, 16)
    cache = oracle.kv_write(pk, pv, pcu, w.empty_cache(), w.block_table, 16)
    B = len(w.seqlens)
    ref = oracle.attention(q, k, v, torch.arange(B + 1, dtype=torch.int32), H, G, d, w.scale, context_lens=ctx,
                           kv_cache=cache, block_table=w.block_table, block_size=16)
    err = np.abs(out8 - ref)
    assert err.max() < 0.15 and err.mean() < 0.02


# ---------------------------------------------------------------- chunked prefill over an FP8 cache
def _exact_kv(shape, seed):
    """K with values e4m3 code x 0.125 and V = 2 K (codes x 0.25): quantization
    with scales 0.125 / 0.25 is exact for them."""
    gen = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 0x7F, shape, generator=gen).reshape(-1).tolist()
    k = (torch.tensor([oracle.e4m3_decode(int(c)) for c in codes], dtype=torch.float64).reshape(shape) * 0.125)
    k = k.to(torch.bfloat16)
    return k, (k.to(torch.float64) * 2.0).to(torch.bfloat16)


def _fp8_chunk_case(lens, ctxs, H, G, d, seed, exact=False):
    """Sequences of ctx + n tokens: the first ctx of each are already in the FP8
    cache (the oracle's FP8 write), the last n are the call's chunk rows."""
    w = W.make_workload([c + n for c, n in zip(ctxs, lens)], H, G, d, block_size=16, seed=seed, extra_pages=2)
    k, v = w.k, w.v
    if exact:
        k, v = _exact_kv(tuple(w.k.shape), seed + 1)
        ks, vs = torch.full((G,), 0.125), torch.full((G,), 0.25)
    else:
        ks, vs = torch.linspace(0.01, 0.03, G), torch.linspace(0.02, 0.05, G)
    starts = w.cu_seqlens.tolist()
    pre = torch.cat([torch.arange(s, s + c) for s, c in zip(starts, ctxs)]).long()
    chk = torch.cat([torch.arange(s + c, s + c + n) for s, c, n in zip(starts, ctxs, lens)]).long()
    pcu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    cache8 = oracle.kv_write_fp8(k[pre], v[pre], pcu, _fp8_cache(w), w.block_table, 16, ks, vs)
    return dict(w=w, q=w.q[chk], k=k[chk], v=v[chk], cu=cu, ctx=torch.tensor(ctxs, dtype=torch.int32),
                cache8=cache8, ks=ks, vs=vs, k_all=k, v_all=v, pre=pre, pcu=pcu)


def _chunked(c, H, G, d, **kw):
    return oracle.chunked_fp8(c["q"], c["k"], c["v"], c["cu"], c["ctx"], H, G, d, c["w"].scale, c["ks"], c["vs"],
                              c["cache8"], c["w"].block_table, 16, **kw)


def test_chunked_fp8_one_row_chunks_equal_decode():
    H, G, d = 4, 2, 16
    w, pq, pk, pv, pcu, q, k, v, ctx, ks, vs = _decode_inputs([40, 1, 17], H, G, d, seed=65, exact=False)
    cache8 = oracle.kv_write_fp8(pk, pv, pcu, _fp8_cache(w), w.block_table, 16, ks, vs)
    B = len(w.seqlens)
    dec = oracle.decode_fp8(q, k, v, ctx, H, G, d, w.scale, ks, vs, cache8, w.block_table, 16)
    chk = oracle.chunked_fp8(q, k, v, torch.arange(B + 1, dtype=torch.int32), ctx, H, G, d, w.scale, ks, vs, cache8,
                             w.block_table, 16)
    assert np.max(np.abs(dec - chk)) < 1e-12


def test_chunked_fp8_exact_values_equal_bf16_definition():
    """Values that quantize exactly: the chunked FP8 attention equals the bf16
    chunked definition over a bf16 cache holding the same prefix."""
    H, G, d = 4, 2, 16
    c = _fp8_chunk_case([37, 50, 1], [40, 0, 17], H, G, d, seed=66, exact=True)
    out8 = _chunked(c, H, G, d)
    cache = oracle.kv_write(c["k_all"][c["pre"]], c["v_all"][c["pre"]], c["pcu"], c["w"].empty_cache(),
                            c["w"].block_table, 16)
    ref = oracle.attention(c["q"], c["k"], c["v"], c["cu"], H, G, d, c["w"].scale, context_lens=c["ctx"],
                           kv_cache=cache, block_table=c["w"].block_table, block_size=16)
    assert np.max(np.abs(out8 - ref)) < 1e-12


def test_chunked_fp8_split_invariance():
    """One chunk of a sequence, or two chunks with the first one's codes in the
    cache: the same outputs (a chunk's own keys are quantized as they are stored)."""
    H, G, d = 4, 2, 16
    lens, cut = [300, 77], [170, 30]
    w = W.make_workload(lens, H, G, d, block_size=16, seed=67, extra_pages=2)
    ks, vs = torch.linspace(0.01, 0.03, G), torch.linspace(0.02, 0.05, G)
    zero = torch.zeros(2, dtype=torch.int32)
    whole = oracle.chunked_fp8(w.q, w.k, w.v, w.cu_seqlens, zero, H, G, d, w.scale, ks, vs, _fp8_cache(w),
                               w.block_table, 16)
    s = w.cu_seqlens.tolist()
    first = torch.cat([torch.arange(s[i], s[i] + cut[i]) for i in range(2)]).long()
    second = torch.cat([torch.arange(s[i] + cut[i], s[i + 1]) for i in range(2)]).long()
    cu1 = torch.tensor([0, cut[0], sum(cut)], dtype=torch.int32)
    cu2 = torch.tensor([0, lens[0] - cut[0], sum(lens) - sum(cut)], dtype=torch.int32)
    out1 = oracle.chunked_fp8(w.q[first], w.k[first], w.v[first], cu1, zero, H, G, d, w.scale, ks, vs, _fp8_cache(w),
                              w.block_table, 16)
    cache8 = oracle.kv_write_fp8(w.k[first], w.v[first], cu1, _fp8_cache(w), w.block_table, 16, ks, vs)
    out2 = oracle.chunked_fp8(w.q[second], w.k[second], w.v[second], cu2, torch.tensor(cut, dtype=torch.int32), H, G,
                              d, w.scale, ks, vs, cache8, w.block_table, 16)
    assert np.max(np.abs(out1 - whole[first.numpy()])) < 1e-12
    assert np.max(np.abs(out2 - whole[second.numpy()])) < 1e-12


def test_chunked_fp8_selected_rows_match_full():
    H, G, d = 4, 2, 16
    c = _fp8_chunk_case([37, 50], [40, 3], H, G, d, seed=68)
    full = _chunked(c, H, G, d)
    rows, heads = [0, 36, 37, 86, 5], [0, 3, 1, 2, 3]
    sel = _chunked(c, H, G, d, rows=rows, heads=heads)
    for n, (r, h) in enumerate(zip(rows, heads)):
        assert np.array_equal(sel[n], full[r, h])

"""GPU parity of the FP8 (e4m3) KV cache against the oracle: kv_cache_store_fp8
writes exactly the oracle's codes (the whole pool compared byte for byte, the
sentinel bytes elsewhere untouched), and paged_decode_attn_fp8 matches the
oracle's decode over the dequantized cache within the suite's tolerance, with
the new token's codes in its slot."""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5


def _scales(t: torch.Tensor) -> torch.Tensor:
    """One scale per kv head: the head's largest magnitude maps to 448."""
    return (t.float().abs().amax(dim=(0, 2)).clamp(min=1e-6) / 448.0).contiguous()


def _fp8_pool(w: W.Workload) -> torch.Tensor:
    return torch.full((w.num_blocks, 2, w.block_size, w.n_kv_head, w.head_dim), SENTINEL, dtype=torch.uint8)


def _assert_bytes_equal(a: torch.Tensor, b: torch.Tensor, what: str):
    if not torch.equal(a, b):
        bad = (a != b).nonzero()
        raise AssertionError(f"{what}: {bad.shape[0]} bytes differ, first at {bad[0].tolist()}")


@pytest.mark.parametrize("lens,ctxs,G,d,bs", [
    ([37, 5, 300], None, 2, 128, 16),
    ([100, 1], [50, 300], 8, 128, 32),
    ([129, 64], [0, 17], 4, 64, 64),
    ([1000], [3], 2, 128, 128),
])
def test_store_fp8_matches_oracle_codes(lens, ctxs, G, d, bs):
    full = [(c or 0) + n for c, n in zip(ctxs or [0] * len(lens), lens)]
    w = W.make_workload(full, 2 * G, G, d, block_size=bs, seed=600 + sum(lens), extra_pages=3)
    starts = w.cu_seqlens.tolist()
    ctx_list = ctxs or [0] * len(lens)
    sel = torch.cat([torch.arange(s + c, s + c + n) for s, c, n in zip(starts, ctx_list, lens)])
    k, v = w.k[sel].contiguous(), w.v[sel].contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ctx = torch.tensor(ctx_list, dtype=torch.int32) if ctxs else None
    ks, vs = _scales(k), _scales(v)
    ref = oracle.kv_write_fp8(k, v, cu, _fp8_pool(w), w.block_table, bs, ks, vs, context_lens=ctx)
    cache = _fp8_pool(w).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.kv_cache_store_fp8(k.cuda(), v.cuda(), cu.cuda(), None if ctx is None else ctx.cuda(), ks.cuda(), vs.cuda(),
                            cache, w.block_table.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _assert_bytes_equal(cache.cpu(), ref, "fp8 pool")


def _decode_case(lens, H, G, d, bs=16, seed=0, fill_on_gpu=False, fill_by_prefill=False):
    """lens: tokens per sequence including the decode token.  The prompts'
    codes come from the oracle, or from kv_cache_store_fp8 (fill_on_gpu), or
    from prefill_attn_fp8_cache (fill_by_prefill), checked byte for byte."""
    w = W.make_workload(lens, H, G, d, block_size=bs, seed=seed, extra_pages=2)
    pq, pk, pv, pcu, q, k, v, ctx = W.decode_views(w)
    ks, vs = _scales(torch.cat([pk, k])), _scales(torch.cat([pv, v]))
    B = len(lens)
    pool = oracle.kv_write_fp8(pk, pv, pcu, _fp8_pool(w), w.block_table, bs, ks, vs)
    ref_out = oracle.decode_fp8(q, k, v, ctx, H, G, d, w.scale, ks, vs, pool, w.block_table, bs)
    ref_pool = oracle.kv_write_fp8(k, v, torch.arange(B + 1, dtype=torch.int32), pool, w.block_table, bs, ks, vs,
                                   context_lens=ctx)
    bt = w.block_table.cuda()
    ks_d, vs_d = ks.cuda(), vs.cuda()
    if fill_on_gpu:
        cache = _fp8_pool(w).cuda()
        _lib.kv_cache_store_fp8(pk.cuda(), pv.cuda(), pcu.cuda(), None, ks_d, vs_d, cache, bt)
        torch.cuda.synchronize()
        _assert_bytes_equal(cache.cpu(), pool, "prompts stored on the GPU")
    elif fill_by_prefill:
        cache = _fp8_pool(w).cuda()
        pout = torch.empty(pq.shape, dtype=torch.bfloat16, device="cuda")
        _lib.prefill_attn_fp8_cache(pq.cuda(), pk.cuda(), pv.cuda(), pcu.cuda(), max(int(c) for c in ctx) or 1,
                                    w.scale, ks_d, vs_d, pout, cache, bt)
        torch.cuda.synchronize()
        _assert_bytes_equal(cache.cpu(), pool, "prompts written by prefill_attn_fp8_cache")
    else:
        cache = pool.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.paged_decode_attn_fp8(q.cuda(), k.cuda(), v.cuda(), ctx.cuda(), int(ctx.max()), w.scale, ks_d, vs_d, out,
                               cache, bt, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _assert_bytes_equal(cache.cpu(), ref_pool, "fp8 pool after decode")
    return U.compare_out(out.cpu(), ref_out, f"fp8 decode {lens[:4]}")


@pytest.mark.parametrize("n", [1, 2, 16, 17, 65, 129, 513, 3000])
def test_decode_fp8_context_lengths(n):
    _decode_case([n], 8, 2, 128, seed=620 + n)


@pytest.mark.parametrize("H,G,d", [(4, 4, 128), (8, 1, 128), (6, 2, 64), (16, 2, 64)])
def test_decode_fp8_head_shapes(H, G, d):
    _decode_case([700, 37], H, G, d, seed=640 + H + G + d)


@pytest.mark.parametrize("bs", [16, 32, 128])
def test_decode_fp8_block_sizes(bs):
    _decode_case([1, 300, 129, 1000], 8, 2, 128, bs=bs, seed=650 + bs)


def test_decode_fp8_varlen64_prompts_stored_on_gpu():
    base = W.named_workload("varlen64_gqa_h32g8_d128")
    _decode_case([n + 1 for n in base.seqlens], 32, 8, 128, seed=660, fill_on_gpu=True)


def test_decode_fp8_after_fp8_prefill():
    _decode_case([1, 300, 129, 1000, 2], 8, 2, 128, seed=670, fill_by_prefill=True)


# ---------------------------------------------------------------- prefill writing the FP8 cache
def _prefill_fp8(w: W.Workload, ks, vs):
    t = U.to_dev(w)
    cache = _fp8_pool(w).cuda()
    out = torch.full_like(t["q"], float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_fp8_cache(t["q"], t["k"], t["v"], t["cu"], w.max_seqlen, w.scale, ks.cuda(), vs.cuda(), out,
                                cache, t["bt"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu(), cache.cpu()


def _check_prefill_fp8(w: W.Workload, full_output: bool, what: str):
    """The codes byte-exact against the oracle (whole pool, sentinel included),
    the output against the oracle's attention, and bit-equal to prefill_attn's
    (the FP8 write leaves the attention arithmetic alone)."""
    ks, vs = _scales(w.k), _scales(w.v)
    out, cache = _prefill_fp8(w, ks, vs)
    ref_pool = oracle.kv_write_fp8(w.k, w.v, w.cu_seqlens, _fp8_pool(w), w.block_table, w.block_size, ks, vs)
    _assert_bytes_equal(cache, ref_pool, f"{what}: fp8 pool")
    if full_output:
        ref = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim, w.scale)
        U.compare_out(out, ref, what)
    else:
        rows, heads = U.sample_rows(w, 96, seed=7)
        ref = oracle.attention_rows(w.q, w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim, w.scale, rows,
                                    heads)
        U.compare_out(out[rows, heads], ref, what)
    bf16_out, _, st = U.run_prefill(w)
    assert st == 0
    assert torch.equal(out.view(torch.int16), bf16_out.view(torch.int16)), f"{what}: output differs from prefill_attn"


@pytest.mark.parametrize("lens,H,G,d,bs", [
    ([37, 5, 300], 4, 2, 128, 16),        # few work items: split-KV
    ([1000], 8, 2, 64, 32),
    ([129, 64, 0, 700], 8, 8, 128, 128),  # an empty sequence
    ([768, 255, 1], 16, 4, 128, 64),
])
def test_prefill_fp8_cache_matches_oracle(lens, H, G, d, bs):
    w = W.make_workload(lens, H, G, d, block_size=bs, seed=680 + sum(lens), extra_pages=3)
    _check_prefill_fp8(w, True, f"fp8 prefill {lens}")


@pytest.mark.parametrize("name", ["gqa_s8192_h32g8_d128", "varlen64_gqa_h32g8_d128"])
def test_prefill_fp8_cache_full_size(name):
    _check_prefill_fp8(W.named_workload(name), False, name)


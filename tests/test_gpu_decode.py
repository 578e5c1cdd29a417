"""GPU parity of paged decode attention (paged_decode_attn) against the
oracle: each sequence's prompt is in the paged cache, and its one new token
attends to the prompt and itself (the oracle's chunked definition with
one-row chunks); the new K/V land in their slot.  Output within the suite's
tolerance, the whole pool bit-exact (sentinel slots included)."""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _case(lens, H, G, d, bs=16, seed=0, max_ctx=None, fill_with_prefill=False):
    """lens: tokens per sequence including the decode token."""
    w = W.make_workload(lens, H, G, d, block_size=bs, seed=seed, extra_pages=2)
    pq, pk, pv, pcu, q, k, v, ctx = W.decode_views(w)
    B = len(lens)
    cu1 = torch.arange(B + 1, dtype=torch.int32)
    cache = oracle.kv_write(pk, pv, pcu, w.empty_cache(), w.block_table, bs)
    ref_out = oracle.attention(q, k, v, cu1, H, G, d, w.scale, context_lens=ctx, kv_cache=cache,
                               block_table=w.block_table, block_size=bs)
    ref_cache = oracle.kv_write(k, v, cu1, cache, w.block_table, bs, context_lens=ctx)
    bt = w.block_table.cuda()
    if fill_with_prefill:  # the prompts' K/V written by this library's own prefill call
        cache_d = w.empty_cache().cuda()
        pout = torch.empty(pq.shape, dtype=torch.bfloat16, device="cuda")
        _lib.prefill_attn(pq.cuda(), pk.cuda(), pv.cuda(), pcu.cuda(), max(int(c) for c in ctx) or 1, w.scale, pout,
                          cache_d, bt)
        torch.cuda.synchronize()
        U.assert_cache_bits_equal(cache_d.cpu(), cache, "prompt cache written by prefill_attn")
    else:
        cache_d = cache.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mc = int(ctx.max()) if max_ctx is None else max_ctx
    _lib.paged_decode_attn(q.cuda(), k.cuda(), v.cuda(), ctx.cuda(), mc, w.scale, out, cache_d, bt, status=status)
    torch.cuda.synchronize()
    return dict(w=w, q=q, k=k, v=v, ctx=ctx, out=out.cpu(), cache=cache_d.cpu(), status=int(status.item()),
                ref_out=ref_out, ref_cache=ref_cache, prompt_cache=cache)


def _check(c, what):
    assert c["status"] == 0, f"{what}: status {c['status']}"
    U.assert_cache_bits_equal(c["cache"], c["ref_cache"], what)
    return U.compare_out(c["out"], c["ref_out"], what)


@pytest.mark.parametrize("n", [1, 2, 16, 17, 64, 65, 66, 129, 512, 513, 514, 1025, 3000, 5001])
def test_decode_context_lengths(n):
    _check(_case([n], 8, 2, 128, seed=400 + n), f"len={n}")


@pytest.mark.parametrize("n", [1, 65, 600, 2100])
def test_decode_head_dim_64(n):
    _check(_case([n], 8, 2, 64, seed=420 + n), f"d=64 len={n}")


@pytest.mark.parametrize("H,G", [(4, 4), (8, 4), (6, 2), (8, 2), (8, 1), (16, 2), (16, 1), (30, 2)])
def test_decode_head_groupings(H, G):
    _check(_case([700, 37], H, G, 128, seed=430 + H * 10 + G), f"H={H} G={G}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
def test_decode_block_sizes(bs):
    _check(_case([1, 300, 129, 1000], 8, 2, 128, bs=bs, seed=440 + bs), f"bs={bs}")


def test_decode_varlen_batch():
    _check(_case([1, 300, 17, 2049, 64, 513, 4100, 2], 32, 8, 128, seed=450), "varlen decode")


def test_decode_long_context_uses_longer_units():
    """40001 keys: more than 64 units of 512 keys, so units of 1024 keys."""
    _check(_case([40001], 8, 2, 128, seed=451), "long context")


def test_decode_empty_context_returns_own_value_bit_exact():
    c = _case([1, 1, 1], 8, 2, 128, seed=452)
    assert c["status"] == 0
    v_rep = c["v"].repeat_interleave(4, dim=1)
    assert torch.equal(c["out"].view(torch.int16), v_rep.view(torch.int16))
    U.assert_cache_bits_equal(c["cache"], c["ref_cache"], "ctx 0 cache")


def test_decode_equals_one_row_chunked_prefill():
    c = _case([900, 5, 260], 8, 2, 128, seed=453)
    w, q, k, v, ctx = c["w"], c["q"], c["k"], c["v"], c["ctx"]
    B = len(w.seqlens)
    cache_d = c["prompt_cache"].cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    _lib.prefill_attn_chunked(q.cuda(), k.cuda(), v.cuda(), torch.arange(B + 1, dtype=torch.int32).cuda(), ctx.cuda(),
                              1, int(ctx.max()), w.scale, out, cache_d, w.block_table.cuda())
    torch.cuda.synchronize()
    U.assert_cache_bits_equal(cache_d.cpu(), c["cache"], "same cache")
    U.compare_out(out.cpu(), c["out"].to(torch.float64).numpy(), "decode vs one-row chunks")


def test_decode_full_size_varlen64_after_prefill():
    """The 64 prompts of the varlen workload prefilled by prefill_attn, then one
    decode token each; every output row against the oracle."""
    w = W.named_workload("varlen64_gqa_h32g8_d128")
    lens = [n + 1 for n in w.seqlens]
    c = _case(lens, 32, 8, 128, seed=454, fill_with_prefill=True)
    _check(c, "varlen64 decode")


def test_decode_bad_block_table_entry_is_reported():
    w = W.make_workload([300], 4, 2, 128, seed=455, extra_pages=1)
    pq, pk, pv, pcu, q, k, v, ctx = W.decode_views(w)
    bt = w.block_table.clone()
    bt[0, 3] = w.num_blocks + 7
    cache = w.empty_cache().cuda()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.paged_decode_attn(q.cuda(), k.cuda(), v.cuda(), ctx.cuda(), int(ctx.max()), w.scale, out, cache, bt.cuda(),
                           status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4


def test_decode_context_above_bound_is_reported():
    c = _case([200, 50], 4, 2, 128, seed=456, max_ctx=100)
    assert c["status"] == 2  # sequence 0 (context 199 > 100) skipped and reported
    U.compare_out(c["out"][1:], c["ref_out"][1:], "the sequence within the bound")

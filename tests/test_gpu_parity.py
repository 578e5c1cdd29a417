"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same
seeded inputs.  Output within max|d| <= 2e-2 and mean|d| <= 2e-3 (bf16 inputs,
fp32 accumulation); the whole KV pool bit-exact, sentinel slots included."""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _native():
    _lib.load()  # the in-tree libprefill.so must be present: no fallback exists
    assert torch.cuda.is_available()


def _full_check(w: W.Workload, what: str):
    out, cache, status = U.run_prefill(w)
    assert status == 0, f"{what}: device status {status}"
    ref_out, ref_cache = oracle.prefill(w)
    U.assert_cache_bits_equal(cache, ref_cache, what)
    if w.total_tokens:
        return U.compare_out(out, ref_out, what)


# ------------------------------------------------------------ small, every element
def test_named_small_workload():
    _full_check(W.named_workload("mha_s128_h4_d64"), "mha_s128_h4_d64")


@pytest.mark.parametrize("n", [1, 2, 3, 15, 16, 17, 127, 128, 129, 255, 256, 300])
@pytest.mark.parametrize("d", [64, 128])
def test_single_sequence_lengths(n, d):
    _full_check(W.make_workload([n], 4, 2, d, seed=100 + n), f"n={n} d={d}")


@pytest.mark.parametrize("H,G", [(8, 8), (8, 2), (8, 1), (6, 3)])
def test_head_groupings(H, G):
    _full_check(W.make_workload([200, 70], H, G, 128, seed=7), f"H={H} G={G}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
def test_block_sizes(bs):
    _full_check(W.make_workload([150, 300, 33], 4, 2, 128, block_size=bs, seed=8, extra_pages=3), f"bs={bs}")


def test_varlen_with_empty_and_ragged_sequences():
    _full_check(W.make_workload([5, 0, 257, 1, 130, 0, 64], 4, 1, 128, seed=9, extra_pages=4), "varlen")


def test_many_work_items_every_element():
    """More work items than SMs, checked element by element: 8 sequences of
    about 1k tokens (ragged tails) at 32 query / 8 kv heads give 1120 items
    (pair of 128-row query blocks x head) over the 148 persistent CTAs, so
    every CTA runs several items back to back (K/V ring phases carried across
    items, TMEM and Q buffers reused, the zigzag deal)."""
    w = W.make_workload([1024, 1000, 1100, 777, 1024, 1300, 900, 1024], 32, 8, 128, seed=15, extra_pages=2)
    _full_check(w, "many items")


def test_idempotent_rerun_rewrites_same_bits():
    w = W.make_workload([333], 8, 2, 128, seed=10)
    out1, cache1, s1 = U.run_prefill(w)
    out2, cache2, s2 = U.run_prefill(w, cache=cache1)
    assert s1 == s2 == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    U.assert_cache_bits_equal(cache1, cache2, "rerun")


# ------------------------------------------------------------ chunked, every element
@pytest.mark.parametrize("s,chunk,bs", [(700, 256, 16), (333, 100, 32), (512, 128, 16), (260, 37, 64)])
def test_chunked_matches_oracle(s, chunk, bs):
    w = W.make_workload([s], 4, 2, 128, block_size=bs, seed=30 + s)
    out, cache, statuses = U.run_chunked(w, chunk)
    assert all(st == 0 for st in statuses), statuses
    ref_out, ref_cache = oracle.prefill(w)  # chunked == unchunked is pinned on the oracle
    U.assert_cache_bits_equal(cache, ref_cache, f"chunked s={s}")
    U.compare_out(out, ref_out, f"chunked s={s} chunk={chunk}")


def test_chunked_batch_with_different_contexts():
    """One call, three sequences with different cached prefixes (not block aligned)."""
    ctxs, lens, bs = [50, 300, 0], [100, 1, 260], 16
    H, G, d = 8, 2, 128
    full = W.make_workload([c + L for c, L in zip(ctxs, lens)], H, G, d, block_size=bs, seed=41, extra_pages=2)
    cache = full.empty_cache()
    starts = full.cu_seqlens.tolist()
    pre_k = torch.cat([full.k[s:s + c] for s, c in zip(starts, ctxs)])
    pre_v = torch.cat([full.v[s:s + c] for s, c in zip(starts, ctxs)])
    pre_cu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cache = oracle.kv_write(pre_k, pre_v, pre_cu, cache, full.block_table, bs)  # the cached prefixes
    sel = torch.cat([torch.arange(s + c, s + c + L) for s, c, L in zip(starts, ctxs, lens)])
    q, k, v = full.q[sel].contiguous(), full.k[sel].contiguous(), full.v[sel].contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ctx = torch.tensor(ctxs, dtype=torch.int32)

    ref_out = oracle.attention(q, k, v, cu, H, G, d, full.scale, context_lens=ctx, kv_cache=cache,
                               block_table=full.block_table, block_size=bs)
    ref_cache = oracle.kv_write(k, v, cu, cache, full.block_table, bs, context_lens=ctx)

    cache_d = cache.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_chunked(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), ctx.cuda(), max(lens), max(ctxs), full.scale,
                              out, cache_d, full.block_table.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.assert_cache_bits_equal(cache_d.cpu(), ref_cache, "chunked batch")
    U.compare_out(out.cpu(), ref_out, "chunked batch")


# ------------------------------------------------------------ special values on the device
def test_first_row_is_v0_bit_exact():
    w = W.make_workload([64, 200], 8, 2, 128, seed=12)
    out, _, status = U.run_prefill(w)
    assert status == 0
    for i in range(2):
        t = int(w.cu_seqlens[i])
        for h in range(8):
            assert torch.equal(out[t, h].view(torch.int16), w.v[t, h // 4].view(torch.int16))


# ------------------------------------------------------------ device-detected errors
def test_bad_block_table_entry_sets_status_and_skips():
    w = W.make_workload([100, 40], 4, 2, 128, seed=13)
    bt = w.block_table.clone()
    bt[1, 1] = w.num_blocks + 7  # tokens 16..31 of sequence 1 have no valid page
    w.block_table = bt
    out, cache, status = U.run_prefill(w)
    assert status == 4
    # sequence 0 and the valid pages of sequence 1 are still written correctly
    ref_out = oracle.attention(w.q, w.k, w.v, w.cu_seqlens, 4, 2, 128, w.scale)
    U.compare_out(out, ref_out, "attention unaffected by the cache")


def test_sequence_longer_than_bound_sets_status():
    w = W.make_workload([100, 300], 4, 2, 128, seed=14)
    t = U.to_dev(w)
    cache = w.empty_cache().cuda()
    out = torch.zeros_like(t["q"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn(t["q"], t["k"], t["v"], t["cu"], 256, w.scale, out, cache, t["bt"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2


# ------------------------------------------------------------ full sizes, sampled rows
def _sampled_check(w: W.Workload, what: str, n_random=96):
    out, cache, status = U.run_prefill(w)
    assert status == 0, f"{what}: status {status}"
    ref_cache = oracle.kv_write(w.k, w.v, w.cu_seqlens, w.empty_cache(), w.block_table, w.block_size)
    U.assert_cache_bits_equal(cache, ref_cache, what)
    rows, heads = U.sample_rows(w, n_random, seed=1)
    ref = oracle.attention_rows(w.q, w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim, w.scale, rows, heads)
    U.compare_out(out[rows, heads], ref, what)
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("name", ["mha_s2048_h32_d128", "gqa_s8192_h32g8_d128", "varlen64_gqa_h32g8_d128"])
def test_named_full_size(name):
    _sampled_check(W.named_workload(name), name)


def test_named_chunked_full_size():
    w = W.named_workload("chunked512_gqa_s8192_h32g8_d128")
    out, cache, statuses = U.run_chunked(w, 512)
    assert all(s == 0 for s in statuses)
    ref_cache = oracle.kv_write(w.k, w.v, w.cu_seqlens, w.empty_cache(), w.block_table, w.block_size)
    U.assert_cache_bits_equal(cache, ref_cache, "chunked full")
    rows, heads = U.sample_rows(w, 96, seed=2)
    rows += [511, 512, 513, 4095, 4096, 8191]
    heads += [0, 5, 31, 7, 8, 2]
    # rows are checked with the chunked oracle: prefix gathered from the oracle's own cache
    ref = np.zeros((len(rows), 128))
    for c in sorted({r // 512 for r in rows}):
        ctx = 512 * c
        pre = oracle.kv_write(w.k[:ctx], w.v[:ctx], torch.tensor([0, ctx], dtype=torch.int32), w.empty_cache(),
                              w.block_table, 16) if ctx else w.empty_cache()
        idx = [s for s, r in enumerate(rows) if r // 512 == c]
        ref[idx] = oracle.attention_rows(w.q[ctx:ctx + 512], w.k[ctx:ctx + 512], w.v[ctx:ctx + 512],
                                         torch.tensor([0, 512], dtype=torch.int32), 32, 8, 128, w.scale,
                                         [rows[s] - ctx for s in idx], [heads[s] for s in idx],
                                         context_lens=[ctx], kv_cache=pre, block_table=w.block_table,
                                         block_size=16)
    U.compare_out(out[rows, heads], ref, "chunked full")


# ------------------------------------------------------------ split-KV (few work items, long prefix)
def _chunked_call(ctxs, lens, H, G, d, bs, seed):
    full = W.make_workload([c + L for c, L in zip(ctxs, lens)], H, G, d, block_size=bs, seed=seed, extra_pages=2)
    cache = full.empty_cache()
    starts = full.cu_seqlens.tolist()
    pre_k = torch.cat([full.k[s:s + c] for s, c in zip(starts, ctxs)])
    pre_v = torch.cat([full.v[s:s + c] for s, c in zip(starts, ctxs)])
    pre_cu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cache = oracle.kv_write(pre_k, pre_v, pre_cu, cache, full.block_table, bs)
    sel = torch.cat([torch.arange(s + c, s + c + L) for s, c, L in zip(starts, ctxs, lens)])
    q, k, v = full.q[sel].contiguous(), full.k[sel].contiguous(), full.v[sel].contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ctx = torch.tensor(ctxs, dtype=torch.int32)
    ref_out = oracle.attention(q, k, v, cu, H, G, d, full.scale, context_lens=ctx, kv_cache=cache,
                               block_table=full.block_table, block_size=bs)
    ref_cache = oracle.kv_write(k, v, cu, cache, full.block_table, bs, context_lens=ctx)
    cache_d = cache.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_chunked(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), ctx.cuda(), max(lens), max(ctxs), full.scale,
                              out, cache_d, full.block_table.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.assert_cache_bits_equal(cache_d.cpu(), ref_cache, "split-kv cache")
    return U.compare_out(out.cpu(), ref_out, f"split-kv ctx={ctxs} lens={lens} d={d}")


@pytest.mark.parametrize("d", [64, 128])
def test_split_kv_long_prefix(d):
    """4 work items against a ~3k prefix: the kv range is split and merged."""
    _chunked_call([3000], [300], 8, 2, d, 16, seed=71)


def test_chunked_many_work_items_every_element():
    """A chunked call with more work items than SMs (8 sequences x 2 pairs x
    32 heads = 512, so no split-KV), every element against the oracle: each
    CTA gathers several prefixes through the block table, back to back."""
    _chunked_call([1000, 1537, 512, 2000, 0, 700, 1300, 64], [512, 500, 512, 300, 512, 511, 512, 257], 32, 8, 128, 16,
                  seed=73)


def test_split_kv_mixed_batch():
    """Pairs with long ranges split, short ones do not; both paths in one call."""
    _chunked_call([2000, 50, 1500, 0], [200, 30, 129, 5], 4, 1, 128, 32, seed=72)

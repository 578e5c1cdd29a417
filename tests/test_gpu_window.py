"""GPU parity of the sliding-window call (prefill_attn_sliding_window) against
the oracle with the same window: every output element within the suite's
tolerance and the whole KV pool bit-exact.  Covers windows narrower than,
equal to and wider than a tile, windows that cut a cached prefix (including
a partly filled last prefix page), varlen batches, split-KV, and the two
exact reductions: window 1 returns each row's own V, and a window wider than
every sequence reproduces prefill_attn bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def run_window(w: W.Workload, window: int, cache: torch.Tensor | None = None):
    t = U.to_dev(w)
    cache_d = (w.empty_cache() if cache is None else cache).cuda()
    out = torch.full_like(t["q"], float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_sliding_window(t["q"], t["k"], t["v"], t["cu"], None, w.max_seqlen, 0, w.scale, window, out,
                                     cache_d, t["bt"], status=status)
    torch.cuda.synchronize()
    return out.cpu(), cache_d.cpu(), int(status.item())


def _full_check(w: W.Workload, window: int, what: str):
    out, cache, status = run_window(w, window)
    assert status == 0, f"{what}: device status {status}"
    ref_out, ref_cache = oracle.prefill(w, window=window)
    U.assert_cache_bits_equal(cache, ref_cache, what)
    return U.compare_out(out, ref_out, what)


@pytest.mark.parametrize("window", [1, 2, 64, 127, 128, 129, 200, 256, 300, 699, 5000])
@pytest.mark.parametrize("d", [64, 128])
def test_window_single_sequence(window, d):
    _full_check(W.make_workload([700], 4, 2, d, seed=300 + window), window, f"window={window} d={d}")


@pytest.mark.parametrize("n", [1, 129, 255, 256, 257, 520])
def test_window_lengths(n):
    _full_check(W.make_workload([n], 8, 2, 128, seed=320 + n), 150, f"n={n}")


def test_window_varlen_gqa():
    w = W.make_workload([5, 0, 700, 1, 130, 0, 389], 8, 2, 128, seed=330, extra_pages=4)
    _full_check(w, 100, "varlen window")


@pytest.mark.parametrize("bs", [16, 64])
def test_window_block_sizes(bs):
    _full_check(W.make_workload([600, 150], 4, 1, 128, block_size=bs, seed=331), 333, f"bs={bs}")


def test_window_one_returns_own_value_bit_exact():
    w = W.make_workload([300, 17], 8, 2, 128, seed=332)
    out, _, status = run_window(w, 1)
    assert status == 0
    v_rep = w.v.repeat_interleave(4, dim=1)
    assert torch.equal(out.view(torch.int16), v_rep.view(torch.int16))


def test_wide_window_equals_prefill_attn_bit_exact():
    w = W.make_workload([700, 129, 3], 8, 2, 128, seed=333)
    out_w, cache_w, s1 = run_window(w, 701)
    out_p, cache_p, s2 = U.run_prefill(w)
    assert s1 == s2 == 0
    assert torch.equal(out_w.view(torch.int16), out_p.view(torch.int16))
    U.assert_cache_bits_equal(cache_w, cache_p, "wide window cache")


# ------------------------------------------------------------ chunked with a window
def _chunked_window(ctxs, lens, H, G, d, bs, window, seed):
    """One chunked call: each sequence's chunk after its cached prefix."""
    full = W.make_workload([c + L for c, L in zip(ctxs, lens)], H, G, d, block_size=bs, seed=seed, extra_pages=2)
    starts = full.cu_seqlens.tolist()
    pre_k = torch.cat([full.k[s:s + c] for s, c in zip(starts, ctxs)])
    pre_v = torch.cat([full.v[s:s + c] for s, c in zip(starts, ctxs)])
    pre_cu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cache = oracle.kv_write(pre_k, pre_v, pre_cu, full.empty_cache(), full.block_table, bs)
    sel = torch.cat([torch.arange(s + c, s + c + L) for s, c, L in zip(starts, ctxs, lens)])
    q, k, v = full.q[sel].contiguous(), full.k[sel].contiguous(), full.v[sel].contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ctx = torch.tensor(ctxs, dtype=torch.int32)
    ref_out = oracle.attention(q, k, v, cu, H, G, d, full.scale, context_lens=ctx, kv_cache=cache,
                               block_table=full.block_table, block_size=bs, window=window)
    ref_cache = oracle.kv_write(k, v, cu, cache, full.block_table, bs, context_lens=ctx)
    cache_d = cache.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_sliding_window(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), ctx.cuda(), max(lens), max(ctxs),
                                     full.scale, window, out, cache_d, full.block_table.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.assert_cache_bits_equal(cache_d.cpu(), ref_cache, "window chunked cache")
    return U.compare_out(out.cpu(), ref_out, f"window chunked ctx={ctxs} lens={lens} window={window}")


@pytest.mark.parametrize("window", [1, 60, 128, 201, 450, 2000])
def test_window_chunked(window):
    """A prefix of 333 tokens (last page partly filled at bs 16, last prefix
    tile partial): the window reaches into it by various amounts."""
    _chunked_window([333], [300], 4, 2, 128, 16, window, seed=340)


def test_window_chunked_batch():
    _chunked_window([50, 300, 0, 1000], [100, 1, 260, 200], 8, 2, 128, 16, 257, seed=341)


@pytest.mark.parametrize("d", [64, 128])
def test_window_split_kv(d):
    """Few work items against a long prefix (not a multiple of the tile): the
    windowed kv range is split and merged."""
    _chunked_window([3001], [300], 8, 2, d, 16, 1500, seed=342)


def test_window_split_kv_mixed():
    _chunked_window([2000, 50, 4100, 0], [200, 30, 129, 5], 4, 1, 128, 32, 1100, seed=343)


# ------------------------------------------------------------ full size, sampled rows
def test_window_full_size_sampled():
    w = W.named_workload("gqa_s8192_h32g8_d128")
    window = 4096
    out, cache, status = run_window(w, window)
    assert status == 0
    ref_cache = oracle.kv_write(w.k, w.v, w.cu_seqlens, w.empty_cache(), w.block_table, w.block_size)
    U.assert_cache_bits_equal(cache, ref_cache, "window full")
    rows, heads = U.sample_rows(w, 96, seed=3)
    rows += [4094, 4095, 4096, 4097, 8191]
    heads += [0, 9, 17, 31, 30]
    ref = oracle.attention_rows(w.q, w.k, w.v, w.cu_seqlens, 32, 8, 128, w.scale, rows, heads, window=window)
    U.compare_out(out[rows, heads], ref, "window full")
    assert torch.isfinite(out.float()).all()


def test_window_rejects_bad_arguments():
    w = W.make_workload([10], 4, 2, 128, seed=344)
    t = U.to_dev(w)
    out = torch.empty_like(t["q"])
    cache = w.empty_cache().cuda()
    for bad in (0, -5):
        rc = _lib.prefill_attn_sliding_window(t["q"], t["k"], t["v"], t["cu"], None, 10, 0, w.scale, bad, out, cache,
                                              t["bt"], raise_on_error=False)
        assert rc == 2


def test_window_split_kv_start_in_partial_prefix_tile():
    """Split-KV with query block 10's window starting inside the partly filled
    last prefix tile (positions 2944..3000 of a 3001-token prefix), so its pair
    partner starts two tiles later, at the chunk's first tile."""
    _chunked_window([3001], [1536], 8, 2, 128, 16, 1400, seed=345)

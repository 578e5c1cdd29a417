"""GPU parity of chunked prefill over an FP8 (e4m3) cache
(prefill_attn_chunked_fp8) against the oracle: each chunk attends to its
dequantized cached prefix and to its own rows quantized the same way (every
key and value the attention sees is a dequantized cache value), and its codes
are appended.  The pool is compared byte for byte (sentinel bytes elsewhere
untouched), the output within the suite's tolerance.

This file is collected last, so that a run stopping at its first failure has
already run every other GPU test.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U
from tests.test_gpu_fp8 import _assert_bytes_equal, _fp8_pool, _scales

pytestmark = pytest.mark.gpu


def _compare(gpu_out: torch.Tensor, ref: np.ndarray, vs: torch.Tensor, what: str):
    """The suite's tolerance (max 2e-2, mean 2e-3).  The call stages the e4m3
    code values, which bf16 holds exactly, and applies the per-kv-head scales
    in fp32 inside the attention (K's to the scores, V's to the output), so
    the only departures from the fp64 oracle are the fp32 accumulation and the
    bf16 P and output roundings of the bf16 path."""
    return U.compare_out(gpu_out, ref, what)


def _chunk_case(lens, ctxs, H, G, d, bs, seed):
    """Sequences of ctx + n tokens whose first ctx are already in the FP8 cache
    (the oracle's codes); the last n are the call's chunk rows."""
    w = W.make_workload([c + n for c, n in zip(ctxs, lens)], H, G, d, block_size=bs, seed=seed, extra_pages=3)
    ks, vs = _scales(w.k), _scales(w.v)
    starts = w.cu_seqlens.tolist()
    pre = torch.cat([torch.arange(s, s + c) for s, c in zip(starts, ctxs)]).long()
    chk = torch.cat([torch.arange(s + c, s + c + n) for s, c, n in zip(starts, ctxs, lens)]).long()
    pcu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    ctx = torch.tensor(ctxs, dtype=torch.int32)
    pool = oracle.kv_write_fp8(w.k[pre], w.v[pre], pcu, _fp8_pool(w), w.block_table, bs, ks, vs)
    return w, w.q[chk].contiguous(), w.k[chk].contiguous(), w.v[chk].contiguous(), cu, ctx, pool, ks, vs


def _run_chunked_fp8(q, k, v, cu, ctx, pool_d, bt_d, ks, vs, scale, max_q, max_ctx):
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn_chunked_fp8(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), ctx.cuda(), max_q, max_ctx, scale, ks.cuda(),
                                  vs.cuda(), out, pool_d, bt_d, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu()


@pytest.mark.parametrize("lens,ctxs,H,G,d,bs", [
    ([37, 130, 1], [40, 0, 300], 8, 2, 64, 16),
    ([512], [1536], 8, 2, 128, 16),           # one long chunk: split-KV
    ([100, 1], [50, 300], 8, 8, 128, 32),
    ([129, 64], [0, 17], 4, 4, 64, 64),
    ([300], [1000], 16, 2, 128, 128),
])
def test_chunked_fp8_matches_oracle(lens, ctxs, H, G, d, bs):
    w, q, k, v, cu, ctx, pool, ks, vs = _chunk_case(lens, ctxs, H, G, d, bs, seed=700 + sum(lens) + sum(ctxs))
    ref_out = oracle.chunked_fp8(q, k, v, cu, ctx, H, G, d, w.scale, ks, vs, pool, w.block_table, bs)
    ref_pool = oracle.kv_write_fp8(k, v, cu, pool, w.block_table, bs, ks, vs, context_lens=ctx)
    pool_d = pool.cuda()
    out = _run_chunked_fp8(q, k, v, cu, ctx, pool_d, w.block_table.cuda(), ks, vs, w.scale, max(lens), max(ctxs))
    _assert_bytes_equal(pool_d.cpu(), ref_pool, "fp8 pool after the chunk")
    _compare(out, ref_out, vs, f"chunked fp8 {lens} {ctxs}")


def test_chunked_fp8_whole_sequence_in_chunks():
    """A 2048-token sequence in four 512-row chunks from an empty FP8 cache:
    every chunk's output against the oracle's single chunk over the whole
    sequence (a chunk's own keys are quantized as stored, so chunking does not
    change the definition), and the final pool byte-exact."""
    H, G, d, bs = 8, 2, 128, 16
    w = W.make_workload([2048], H, G, d, block_size=bs, seed=720, extra_pages=2)
    ks, vs = _scales(w.k), _scales(w.v)
    ref = oracle.chunked_fp8(w.q, w.k, w.v, w.cu_seqlens, torch.zeros(1, dtype=torch.int32), H, G, d, w.scale, ks, vs,
                             _fp8_pool(w), w.block_table, bs)
    pool_d, bt_d = _fp8_pool(w).cuda(), w.block_table.cuda()
    outs = []
    for q, k, v, cu, ctx, _ in W.chunk_views(w, 512):
        outs.append(_run_chunked_fp8(q, k, v, cu, ctx, pool_d, bt_d, ks, vs, w.scale, int(cu[-1]), int(ctx[0])))
    _compare(torch.cat(outs, 0), ref, vs, "chunks of 512")
    ref_pool = oracle.kv_write_fp8(w.k, w.v, w.cu_seqlens, _fp8_pool(w), w.block_table, bs, ks, vs)
    _assert_bytes_equal(pool_d.cpu(), ref_pool, "fp8 pool after all chunks")


def test_chunked_fp8_full_size_sampled():
    """The 8k GQA prompt in 16 chunks of 512 over the FP8 cache; the first and
    last row of every 128-row block of every chunk, for every head, and random
    rows against the oracle; the final pool byte-exact."""
    w = W.named_workload("chunked512_gqa_s8192_h32g8_d128")
    ks, vs = _scales(w.k), _scales(w.v)
    pool_d, bt_d = _fp8_pool(w).cuda(), w.block_table.cuda()
    outs = []
    for q, k, v, cu, ctx, _ in W.chunk_views(w, w.chunk):
        outs.append(_run_chunked_fp8(q, k, v, cu, ctx, pool_d, bt_d, ks, vs, w.scale, int(cu[-1]), int(ctx[0])))
    out = torch.cat(outs, 0)
    ref_pool = oracle.kv_write_fp8(w.k, w.v, w.cu_seqlens, _fp8_pool(w), w.block_table, w.block_size, ks, vs)
    _assert_bytes_equal(pool_d.cpu(), ref_pool, "fp8 pool, 16 chunks")
    rows, heads = U.sample_rows(w, 42, seed=8)  # every (128-row block, head): first and last row
    rows += [511, 512, 4095, 4096]
    heads += [3, 30, 0, 17]
    ref = oracle.chunked_fp8(w.q, w.k, w.v, w.cu_seqlens, torch.zeros(1, dtype=torch.int32), w.n_head, w.n_kv_head,
                             w.head_dim, w.scale, ks, vs, _fp8_pool(w), w.block_table, w.block_size, rows=rows,
                             heads=heads)
    _compare(out[rows, heads], ref, vs, "chunked fp8 full size")

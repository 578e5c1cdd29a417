"""Failure path on the GPU without a fault or a hang: a test hook makes the
pipelined kernel's producer withhold one Q tile, so a consumer's bounded wait
(about one second) expires.  The call must report PREFILL_ERR_TIMEOUT, every
role must stop and release its resources, and the same CUDA context must then
run a normal call correctly."""
import time

import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def test_stalled_pipeline_reports_timeout_and_context_survives():
    w = W.make_workload([600, 300], 8, 2, 128, seed=61)
    t = U.to_dev(w)
    cache = w.empty_cache().cuda()
    out = torch.zeros_like(t["q"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.inject_stall(True)
    t0 = time.time()
    rc = _lib.prefill_attn(t["q"], t["k"], t["v"], t["cu"], w.max_seqlen, w.scale, out, cache, t["bt"], status=status)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert rc == 0  # the launch itself succeeded
    assert int(status.item()) == 6, _lib.status_string(int(status.item()))
    assert elapsed < 30.0
    # the context is intact: a normal call on fresh buffers gives correct results
    out2, cache2, st2 = U.run_prefill(w)
    assert st2 == 0
    ref_out, ref_cache = oracle.prefill(w)
    U.assert_cache_bits_equal(cache2, ref_cache, "after timeout")
    U.compare_out(out2, ref_out, "after timeout")


def test_hook_resets_after_one_launch():
    w = W.make_workload([256], 4, 2, 128, seed=62)
    _lib.inject_stall(True)
    _, _, st1 = U.run_prefill(w)
    _, _, st2 = U.run_prefill(w)
    assert st1 == 6 and st2 == 0


def test_stalled_split_call_leaves_no_stale_merge_state():
    """A chunked call whose kv ranges are split is stalled: some of its CTAs
    give up before writing their split partials, so the workspace is left
    holding a mix of this call's partials and stale ones.  The next identical
    call must not read any of them as its own: its combine kernel may only
    merge partials that its own attention kernel wrote, which every split of
    every row does before the combine runs.  (The fixed array of the
    no-allocation entry point relies on the same property: it keeps whatever
    the last call left in it.)"""
    ctx, L, H, G, d, bs = 3000, 300, 8, 2, 128, 16
    full = W.make_workload([ctx + L], H, G, d, block_size=bs, seed=63, extra_pages=2)
    cache = oracle.kv_write(full.k[:ctx], full.v[:ctx], torch.tensor([0, ctx], dtype=torch.int32),
                            full.empty_cache(), full.block_table, bs)
    q, k, v = (x[ctx:].contiguous() for x in (full.q, full.k, full.v))
    cu = torch.tensor([0, L], dtype=torch.int32)
    ctxs = torch.tensor([ctx], dtype=torch.int32)
    ref_out = oracle.attention(q, k, v, cu, H, G, d, full.scale, context_lens=ctxs, kv_cache=cache,
                               block_table=full.block_table, block_size=bs)
    dev = [x.cuda() for x in (q, k, v, cu, ctxs, full.block_table)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for stall in (True, False):
        cache_d = cache.cuda()
        out = torch.full(dev[0].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        status.zero_()
        _lib.inject_stall(stall)
        _lib.prefill_attn_chunked(dev[0], dev[1], dev[2], dev[3], dev[4], L, ctx, full.scale, out, cache_d, dev[5],
                                  status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == (6 if stall else 0)
    U.compare_out(out.cpu(), ref_out, "split call after a stalled split call")

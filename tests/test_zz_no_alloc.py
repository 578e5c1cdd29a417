"""prefill_attn_chunked_noalloc: the chunked call for callers that cannot let
the library allocate device memory (engines that own all device memory
through their own pool, processes with a device-memory budget fixed at
start-up).  Its split-KV partials live in a fixed 32 MiB device array in the
library instead of a cudaMalloc'd workspace.

Checked through the C ABI against the allocating entry point,
prefill_attn_chunked, on the same inputs: two calls in a row must each match
it (output within the suite's tolerance, KV cache bit-exact), and a call whose
chosen split count would not fit the array must run with fewer splits and
still match.

This file is collected after the other parity files, so that a run stopping at
the first failure has already run them; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _chunk_inputs(ctxs, lens, H, G, d, bs, seed):
    """A chunked call: each sequence's chunk attends to its cached prefix."""
    full = W.make_workload([c + L for c, L in zip(ctxs, lens)], H, G, d, block_size=bs, seed=seed, extra_pages=2)
    starts = full.cu_seqlens.tolist()
    pre_k = torch.cat([full.k[s:s + c] for s, c in zip(starts, ctxs)])
    pre_v = torch.cat([full.v[s:s + c] for s, c in zip(starts, ctxs)])
    pre_cu = torch.tensor(np.concatenate([[0], np.cumsum(ctxs)]), dtype=torch.int32)
    cache = oracle.kv_write(pre_k, pre_v, pre_cu, full.empty_cache(), full.block_table, bs)
    sel = torch.cat([torch.arange(s + c, s + c + L) for s, c, L in zip(starts, ctxs, lens)])
    dev = torch.device("cuda")
    return dict(q=full.q[sel].contiguous().to(dev), k=full.k[sel].contiguous().to(dev),
                v=full.v[sel].contiguous().to(dev),
                cu=torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev),
                ctx=torch.tensor(ctxs, dtype=torch.int32, device=dev), bt=full.block_table.to(dev),
                cache=cache, max_q=max(lens), max_ctx=max(ctxs), scale=full.scale)


def _call(fn, a):
    cache = a["cache"].to("cuda")
    out = torch.full(a["q"].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = fn(a["q"], a["k"], a["v"], a["cu"], a["ctx"], a["max_q"], a["max_ctx"], a["scale"], out, cache, a["bt"],
            status=status, raise_on_error=False)
    torch.cuda.synchronize()
    return rc, int(status.item()), out.cpu(), cache.cpu()


@pytest.mark.parametrize("ctxs,lens,H,G,d", [
    ([3000], [300], 8, 2, 128),                 # four work items against a long prefix: split
    ([2000, 50, 1500, 0], [200, 30, 129, 5], 4, 1, 128),  # split and unsplit pairs in one call
    ([2500], [256], 8, 8, 64),                  # head_dim 64
])
def test_noalloc_matches_allocating_entry_point_twice(ctxs, lens, H, G, d):
    a = _chunk_inputs(ctxs, lens, H, G, d, 16, seed=81)
    rc, st, ref_out, ref_cache = _call(_lib.prefill_attn_chunked, a)
    assert rc == 0 and st == 0
    for _ in range(2):  # two calls in a row share the static array
        rc, st, out, cache = _call(_lib.prefill_attn_chunked_noalloc, a)
        assert rc == 0 and st == 0, (rc, st)
        U.compare_out(out, ref_out.to(torch.float64).numpy(), "noalloc vs allocating entry point")
        U.assert_cache_bits_equal(cache, ref_cache, "noalloc cache")


def test_noalloc_runs_with_fewer_splits_when_its_array_is_too_small():
    # 60 work items against 4000-token prefixes: the allocating call takes seven
    # splits, whose partials (7 x 3840 rows x 4 heads x 130 floats = 55.9 MB)
    # exceed the 32 MiB array; the no-allocation call runs with the largest
    # split count that fits (four: 31.9 MB) and must give the same result
    a = _chunk_inputs([4000] * 15, [256] * 15, 4, 1, 128, 16, seed=82)
    assert _lib.load().prefill_noalloc_scratch_bytes() == 32 << 20
    rc, st, ref_out, ref_cache = _call(_lib.prefill_attn_chunked, a)
    assert rc == 0 and st == 0
    for _ in range(2):
        rc, st, out, cache = _call(_lib.prefill_attn_chunked_noalloc, a)
        assert rc == 0 and st == 0, (rc, st)
        U.compare_out(out, ref_out.to(torch.float64).numpy(), "noalloc with fewer splits vs allocating entry point")
        U.assert_cache_bits_equal(cache, ref_cache, "noalloc cache, fewer splits")

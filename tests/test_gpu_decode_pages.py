"""GPU parity of the whole-page decode kernel (the decode path for kv-head
counts that are a multiple of 8, and head_dim 128 for the FP8 cache): the
same oracle checks as the per-warp kernel's tests, on shapes that select it --
one and several slabs of 8 kv heads, 1 to 16 query heads per kv head, head_dim
64 and 128, every page size, contexts that end anywhere inside a 16-token step
(so the new token's row and the zeroed rows past it fall everywhere), long
contexts with many key splits.  Output within the suite's tolerance, the whole
pool bit-exact (byte-exact for the FP8 codes).  The per-warp kernel is re-run
on the same cases in a child process with LIBPREFILL_DECODE=warp."""
import os
import subprocess
import sys

import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U
from tests.test_gpu_decode import _case, _check
from tests.test_gpu_fp8 import _decode_case

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n", [1, 2, 15, 16, 17, 31, 33, 255, 256, 257, 513, 1000, 4097])
def test_pages_context_lengths(n):
    _check(_case([n], 32, 8, 128, seed=700 + n), f"G=8 len={n}")


@pytest.mark.parametrize("H,G", [(8, 8), (16, 8), (32, 8), (64, 8), (128, 8), (16, 16), (64, 16), (96, 24)])
def test_pages_head_groupings(H, G):
    _check(_case([700, 37, 1], H, G, 128, seed=720 + H + G), f"H={H} G={G}")


@pytest.mark.parametrize("n", [1, 65, 600, 2100])
def test_pages_head_dim_64(n):
    _check(_case([n, 19], 32, 8, 64, seed=740 + n), f"d=64 len={n}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
def test_pages_block_sizes(bs):
    _check(_case([1, 300, 129, 1000, 47], 32, 8, 128, bs=bs, seed=760 + bs), f"bs={bs}")


def test_pages_long_context():
    """40001 keys: units of 1024 keys (at most 64 units per sequence)."""
    _check(_case([40001, 3], 16, 8, 128, seed=780), "long context")


def test_pages_empty_context_returns_own_value_bit_exact():
    c = _case([1, 1, 1], 32, 8, 128, seed=781)
    assert c["status"] == 0
    v_rep = c["v"].repeat_interleave(4, dim=1)
    assert torch.equal(c["out"].view(torch.int16), v_rep.view(torch.int16))
    U.assert_cache_bits_equal(c["cache"], c["ref_cache"], "ctx 0 cache")


def test_pages_equal_one_row_chunked_prefill():
    c = _case([900, 5, 260, 16], 32, 8, 128, seed=782)
    w, q, k, v, ctx = c["w"], c["q"], c["k"], c["v"], c["ctx"]
    B = len(w.seqlens)
    cache_d = c["prompt_cache"].cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    _lib.prefill_attn_chunked(q.cuda(), k.cuda(), v.cuda(), torch.arange(B + 1, dtype=torch.int32).cuda(), ctx.cuda(),
                              1, int(ctx.max()), w.scale, out, cache_d, w.block_table.cuda())
    torch.cuda.synchronize()
    U.assert_cache_bits_equal(cache_d.cpu(), c["cache"], "same cache")
    U.compare_out(out.cpu(), c["out"].to(torch.float64).numpy(), "decode vs one-row chunks")


def test_pages_nan_in_unused_slots_does_not_leak():
    """Slots past each context hold NaN bit patterns (another sequence's stale
    data could be anything): the rows past the new token are zeroed before P V."""
    w = W.make_workload([37, 300, 16], 32, 8, 128, seed=783, extra_pages=2)
    pq, pk, pv, pcu, q, k, v, ctx = W.decode_views(w)
    cu1 = torch.arange(len(w.seqlens) + 1, dtype=torch.int32)
    pool = w.empty_cache()
    pool.view(torch.int16).fill_(0x7FC1)  # NaN everywhere the prompts do not write
    cache = oracle.kv_write(pk, pv, pcu, pool, w.block_table, w.block_size)
    ref_out = oracle.attention(q, k, v, cu1, 32, 8, 128, w.scale, context_lens=ctx, kv_cache=cache,
                               block_table=w.block_table, block_size=w.block_size)
    cache_d = cache.cuda()
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.paged_decode_attn(q.cuda(), k.cuda(), v.cuda(), ctx.cuda(), int(ctx.max()), w.scale, out, cache_d,
                           w.block_table.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    U.compare_out(out.cpu(), ref_out, "NaN-filled pool")


def test_pages_bad_block_table_entry_is_reported():
    w = W.make_workload([300], 16, 8, 128, seed=784, extra_pages=1)
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


def test_pages_context_above_bound_is_reported():
    c = _case([200, 50], 32, 8, 128, seed=785, max_ctx=100)
    assert c["status"] == 2
    U.compare_out(c["out"][1:], c["ref_out"][1:], "the sequence within the bound")


@pytest.mark.parametrize("n", [1, 16, 17, 300, 1025, 4097])
def test_pages_fp8_context_lengths(n):
    _decode_case([n, 33], 32, 8, 128, seed=790 + n)


@pytest.mark.parametrize("H,G", [(8, 8), (128, 8), (32, 16)])
def test_pages_fp8_head_groupings(H, G):
    _decode_case([700, 37], H, G, 128, seed=800 + H + G)


@pytest.mark.parametrize("bs", [16, 32, 128])
def test_pages_fp8_block_sizes(bs):
    _decode_case([1, 300, 129, 1000], 32, 8, 128, bs=bs, seed=810 + bs)


def test_pages_fp8_after_fp8_prefill():
    _decode_case([1, 300, 129, 1000, 2], 32, 8, 128, seed=820, fill_by_prefill=True)


WARP_SELECTION = [
    "tests/test_gpu_decode_pages.py::test_pages_context_lengths",
    "tests/test_gpu_decode_pages.py::test_pages_head_groupings",
    "tests/test_gpu_decode_pages.py::test_pages_block_sizes",
    "tests/test_gpu_decode_pages.py::test_pages_fp8_context_lengths",
    "tests/test_gpu_decode.py::test_decode_full_size_varlen64_after_prefill",
]


def test_per_warp_kernel_on_the_same_cases():
    """LIBPREFILL_DECODE=warp: the per-warp kernel on the shapes above."""
    if os.environ.get("LIBPREFILL_DECODE") == "warp":
        pytest.skip("already the per-warp kernel")
    env = dict(os.environ, LIBPREFILL_DECODE="warp")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        *WARP_SELECTION], cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]

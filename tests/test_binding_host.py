"""CPU tests of the Python binding's argument checks: each wrapper rejects a
wrong dtype, rank or layout with ValueError before anything reaches the C
library (so these calls never launch)."""
import pytest
import torch

from causal_prefill_attention_b200 import _lib

bf = torch.bfloat16


def _t(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def _i32(*shape):
    return torch.zeros(*shape, dtype=torch.int32)


def test_prefill_attn_checks():
    q, k, v, out = _t(8, 4, 64), _t(8, 2, 64), _t(8, 2, 64), _t(8, 4, 64)
    cache, cu, bt = _t(2, 2, 16, 2, 64), _i32(2), _i32(1, 2)
    with pytest.raises(ValueError):
        _lib.prefill_attn(q.float(), k, v, cu, 8, 0.125, out, cache, bt)
    with pytest.raises(ValueError):
        _lib.prefill_attn(q, k, v, cu.long(), 8, 0.125, out, cache, bt)
    with pytest.raises(ValueError):
        _lib.prefill_attn(q, k, v, cu, 8, 0.125, out, cache[:, 0], bt)          # cache rank
    with pytest.raises(ValueError):
        _lib.prefill_attn(q.transpose(0, 1), k, v, cu, 8, 0.125, out, cache, bt)  # not contiguous


def test_fp8_wrapper_checks():
    q, k, v, out = _t(8, 4, 64), _t(8, 2, 64), _t(8, 2, 64), _t(8, 4, 64)
    pool, cu, ctx, bt = _t(2, 2, 16, 2, 64, dtype=torch.uint8), _i32(2), _i32(1), _i32(1, 2)
    ks = torch.ones(2)
    with pytest.raises(ValueError):   # a bf16 pool where codes are expected
        _lib.prefill_attn_fp8_cache(q, k, v, cu, 8, 0.125, ks, ks, out, pool.to(bf), bt)
    with pytest.raises(ValueError):   # fp64 scales
        _lib.prefill_attn_fp8_cache(q, k, v, cu, 8, 0.125, ks.double(), ks, out, pool, bt)
    with pytest.raises(ValueError):
        _lib.prefill_attn_chunked_fp8(q, k, v, cu, ctx.long(), 8, 0, 0.125, ks, ks, out, pool, bt)
    with pytest.raises(ValueError):
        _lib.kv_cache_store_fp8(k, v, cu, None, ks, ks, pool[:, 0], bt)
    with pytest.raises(ValueError):
        _lib.paged_decode_attn_fp8(q[:2], k[:2], v[:2], ctx.repeat(2), 8, 0.125, ks, ks, out[:2].float(), pool, bt)


def test_projection_wrapper_checks():
    with pytest.raises(ValueError):
        _lib.qkv_projection(_t(8, 64).float(), _t(256, 64), 2, 1, 64, _t(8, 2, 64), _t(8, 1, 64), _t(8, 1, 64))
    with pytest.raises(ValueError):
        _lib.attn_out_projection(_t(8, 256), _t(256, 256), _t(8, 256))           # o must be [T, H, d]
    with pytest.raises(ValueError):
        _lib.attn_out_projection(_t(8, 4, 64), _t(256, 256), _t(8, 256).float())

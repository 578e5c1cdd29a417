"""libprefill: causal prefill attention (MHA/GQA, varlen, chunked, sliding
window) fused with the paged KV-cache write, paged decode, an FP8 (e4m3) KV
cache, and the QKV / W_o projections, as hand-written CUDA for B200 (sm_100a)
behind a C ABI (include/prefill.h).  This package is the thin Python binding."""
from ._lib import (PrefillError, load, status_string, num_kv_blocks, kv_block_rule,  # noqa: F401
                   first_kv_block, kv_block_rule_window,
                   prefill_attn, prefill_attn_chunked, prefill_attn_chunked_noalloc, prefill_attn_sliding_window,
                   prefill_attn_fp8_cache, prefill_attn_chunked_fp8, paged_decode_attn, paged_decode_attn_fp8,
                   kv_cache_store_fp8, qkv_projection, attn_out_projection)
from . import workloads  # noqa: F401

"""libprefill: causal prefill attention (MHA/GQA, varlen, chunked) fused with
the paged KV-cache write, as hand-written CUDA for B200 (sm_100a) behind a C
ABI (include/prefill.h).  This package is the thin Python binding."""
from ._lib import (PrefillError, load, prefill_attn, prefill_attn_chunked, status_string,  # noqa: F401
                   num_kv_blocks, kv_block_rule)
from . import workloads  # noqa: F401

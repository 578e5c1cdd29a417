"""ctypes binding of libprefill's C ABI (include/prefill.h).

Argument marshalling only: tensors are turned into device pointers and sizes,
and every step of the computation runs in the CUDA kernels behind the ABI.
There is no fallback: if the shared library is missing, loading fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libprefill.so")

STATUS_NAMES = {
    0: "PREFILL_OK", 1: "PREFILL_ERR_NULL", 2: "PREFILL_ERR_SHAPE", 3: "PREFILL_ERR_UNSUPPORTED",
    4: "PREFILL_ERR_BLOCK_TABLE", 5: "PREFILL_ERR_CUDA", 6: "PREFILL_ERR_TIMEOUT", 7: "PREFILL_ERR_ALIGNMENT",
    8: "PREFILL_ERR_SCRATCH_LIMIT",
}
EXPORTED = ("prefill_attn", "prefill_attn_chunked", "prefill_status_string",
            "prefill_num_kv_blocks", "prefill_kv_block_rule", "prefill_test_inject_stall",
            "prefill_attn_chunked_noalloc", "prefill_noalloc_scratch_bytes",
            "prefill_attn_sliding_window", "prefill_first_kv_block", "prefill_kv_block_rule_window",
            "paged_decode_attn", "qkv_projection", "kv_cache_store_fp8", "paged_decode_attn_fp8",
            "attn_out_projection", "prefill_attn_fp8_cache", "prefill_attn_chunked_fp8", "prefill_test_exp2_fma2")

_lib = None


class PrefillError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def load() -> ctypes.CDLL:
    """Load libprefill.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libprefill.so not built at {LIB_PATH}; run causal_prefill_attention_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.prefill_attn.argtypes = [P, P, P, I, P, I, I, I, I, I, F, P, P, I, P, I, I, P, P]
        lib.prefill_attn.restype = I
        lib.prefill_attn_chunked.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, F, P, P, I, P, I, I, P, P]
        lib.prefill_attn_chunked.restype = I
        lib.prefill_status_string.argtypes = [I]
        lib.prefill_status_string.restype = ctypes.c_char_p
        lib.prefill_num_kv_blocks.argtypes = [I, I, I, I, I]
        lib.prefill_num_kv_blocks.restype = I
        lib.prefill_kv_block_rule.argtypes = [I, I, I, I, I, I, P, P]
        lib.prefill_kv_block_rule.restype = I
        lib.prefill_test_inject_stall.argtypes = [I]
        lib.prefill_test_inject_stall.restype = None
        lib.prefill_attn_chunked_noalloc.argtypes = lib.prefill_attn_chunked.argtypes
        lib.prefill_attn_chunked_noalloc.restype = I
        lib.prefill_noalloc_scratch_bytes.argtypes = []
        lib.prefill_noalloc_scratch_bytes.restype = ctypes.c_size_t
        lib.prefill_attn_sliding_window.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, F, I, P, P, I, P, I, I, P, P]
        lib.prefill_attn_sliding_window.restype = I
        lib.prefill_first_kv_block.argtypes = [I, I, I, I, I, I]
        lib.prefill_first_kv_block.restype = I
        lib.prefill_kv_block_rule_window.argtypes = [I, I, I, I, I, I, I, P, P, P]
        lib.prefill_kv_block_rule_window.restype = I
        lib.paged_decode_attn.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, I, P, I, I, P, P]
        lib.paged_decode_attn.restype = I
        lib.qkv_projection.argtypes = [P, P, I, I, I, I, I, P, P, P, P, P]
        lib.qkv_projection.restype = I
        lib.attn_out_projection.argtypes = [P, P, I, I, I, I, P, P, P]
        lib.attn_out_projection.restype = I
        lib.prefill_attn_fp8_cache.argtypes = [P, P, P, I, P, I, I, I, I, I, F, P, P, P, P, I, P, I, I, P, P]
        lib.prefill_attn_fp8_cache.restype = I
        lib.prefill_attn_chunked_fp8.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, F, P, P, P, P, I, P, I, I, P, P]
        lib.prefill_attn_chunked_fp8.restype = I
        lib.kv_cache_store_fp8.argtypes = [P, P, I, P, P, I, I, I, P, P, P, I, P, I, I, P, P]
        lib.kv_cache_store_fp8.restype = I
        lib.paged_decode_attn_fp8.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, P, P, I, P, I, I, P, P]
        lib.paged_decode_attn_fp8.restype = I
        lib.prefill_test_exp2_fma2.argtypes = [P, P, I, P]
        lib.prefill_test_exp2_fma2.restype = I
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().prefill_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check_bf16(name, t, ndim):
    if t.dtype != torch.bfloat16 or t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {ndim}-d bfloat16 tensor")


def _check_i32(name, t):
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous int32 tensor")


def prefill_attn(q, k, v, cu_seqlens, max_seqlen: int, scale: float, out, kv_cache, block_table,
                 status: Optional[torch.Tensor] = None, stream=None, raise_on_error: bool = True) -> int:
    """Causal prefill attention + paged KV write (C ABI ``prefill_attn``).

    q/out [T, n_head, head_dim], k/v [T, n_kv_head, head_dim], kv_cache
    [num_blocks, 2, block_size, n_kv_head, head_dim] (bf16, CUDA);
    cu_seqlens int32 [B+1], block_table int32 [B, max_blocks_per_seq].
    """
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    _check_bf16("out", out, 3), _check_bf16("kv_cache", kv_cache, 5)
    _check_i32("cu_seqlens", cu_seqlens), _check_i32("block_table", block_table)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1, int(max_seqlen),
        H, G, D, float(scale), _ptr(out), _ptr(kv_cache), kv_cache.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn")
    return rc


def prefill_attn_chunked(q, k, v, cu_seqlens_q, context_lens, max_q_len: int, max_context_len: int,
                         scale: float, out, kv_cache, block_table, status: Optional[torch.Tensor] = None,
                         stream=None, raise_on_error: bool = True) -> int:
    """Chunked prefill (C ABI ``prefill_attn_chunked``): each chunk attends to
    ``context_lens[i]`` cached tokens plus itself, then appends its K/V."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    _check_bf16("out", out, 3), _check_bf16("kv_cache", kv_cache, 5)
    _check_i32("cu_seqlens_q", cu_seqlens_q), _check_i32("context_lens", context_lens)
    _check_i32("block_table", block_table)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn_chunked(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens_q), _ptr(context_lens), cu_seqlens_q.numel() - 1,
        int(max_q_len), int(max_context_len), H, G, D, float(scale), _ptr(out), _ptr(kv_cache),
        kv_cache.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn_chunked")
    return rc


def prefill_attn_chunked_noalloc(q, k, v, cu_seqlens_q, context_lens, max_q_len: int, max_context_len: int,
                                 scale: float, out, kv_cache, block_table, status: Optional[torch.Tensor] = None,
                                 stream=None, raise_on_error: bool = True) -> int:
    """``prefill_attn_chunked`` for callers that cannot allocate device memory
    (C ABI ``prefill_attn_chunked_noalloc``): split-KV partials go to a fixed
    32 MiB device array inside the library instead of a cudaMalloc'd workspace."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    _check_bf16("out", out, 3), _check_bf16("kv_cache", kv_cache, 5)
    _check_i32("cu_seqlens_q", cu_seqlens_q), _check_i32("context_lens", context_lens)
    _check_i32("block_table", block_table)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn_chunked_noalloc(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens_q), _ptr(context_lens), cu_seqlens_q.numel() - 1,
        int(max_q_len), int(max_context_len), H, G, D, float(scale), _ptr(out), _ptr(kv_cache),
        kv_cache.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn_chunked_noalloc")
    return rc


def prefill_attn_sliding_window(q, k, v, cu_seqlens_q, context_lens, max_q_len: int, max_context_len: int,
                                scale: float, window: int, out, kv_cache, block_table,
                                status: Optional[torch.Tensor] = None, stream=None,
                                raise_on_error: bool = True) -> int:
    """Causal prefill with a sliding window of ``window`` keys (C ABI
    ``prefill_attn_sliding_window``): row P sees keys P-window+1 .. P.
    ``context_lens`` None means plain prefill (``max_context_len`` 0)."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    _check_bf16("out", out, 3), _check_bf16("kv_cache", kv_cache, 5)
    _check_i32("cu_seqlens_q", cu_seqlens_q), _check_i32("block_table", block_table)
    if context_lens is not None:
        _check_i32("context_lens", context_lens)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn_sliding_window(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens_q), _ptr(context_lens), cu_seqlens_q.numel() - 1,
        int(max_q_len), int(max_context_len), H, G, D, float(scale), int(window), _ptr(out), _ptr(kv_cache),
        kv_cache.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn_sliding_window")
    return rc


def paged_decode_attn(q, k, v, context_lens, max_context_len: int, scale: float, out, kv_cache, block_table,
                      status: Optional[torch.Tensor] = None, stream=None, raise_on_error: bool = True) -> int:
    """Decode step over the paged cache (C ABI ``paged_decode_attn``): the new
    token of each sequence (q [B, n_head, d], k/v [B, n_kv_head, d]) attends to
    its ``context_lens[i]`` cached tokens and itself; its K/V are appended."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    _check_bf16("out", out, 3), _check_bf16("kv_cache", kv_cache, 5)
    _check_i32("context_lens", context_lens), _check_i32("block_table", block_table)
    B, H, D = q.shape
    G = k.shape[1]
    rc = load().paged_decode_attn(
        _ptr(q), _ptr(k), _ptr(v), _ptr(context_lens), B, int(max_context_len), H, G, D, float(scale), _ptr(out),
        _ptr(kv_cache), kv_cache.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "paged_decode_attn")
    return rc


def qkv_projection(x, w, n_head: int, n_kv_head: int, head_dim: int, q, k, v,
                   status: Optional[torch.Tensor] = None, stream=None, raise_on_error: bool = True) -> int:
    """Fused QKV projection (C ABI ``qkv_projection``): y = x w^T on the tensor
    cores, cut by columns into q [T, n_head, d], k and v [T, n_kv_head, d].
    x [T, hidden] and w [(n_head + 2 n_kv_head) d, hidden] are bf16."""
    _check_bf16("x", x, 2), _check_bf16("w", w, 2)
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3)
    T, hid = x.shape
    rc = load().qkv_projection(_ptr(x), _ptr(w), T, hid, int(n_head), int(n_kv_head), int(head_dim), _ptr(q),
                               _ptr(k), _ptr(v), _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "qkv_projection")
    return rc


def attn_out_projection(o, w_o, y, status: Optional[torch.Tensor] = None, stream=None,
                        raise_on_error: bool = True) -> int:
    """Output projection W_o after the attention (C ABI ``attn_out_projection``):
    o [T, n_head, d] read as [T, n_head d] (heads merged, head after head),
    w_o [hidden, n_head d], y [T, hidden] = o w_o^T; bf16, on the tensor cores."""
    _check_bf16("o", o, 3), _check_bf16("w_o", w_o, 2), _check_bf16("y", y, 2)
    T, H, D = o.shape
    rc = load().attn_out_projection(_ptr(o), _ptr(w_o), T, H, D, w_o.shape[0], _ptr(y), _ptr(status),
                                    _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "attn_out_projection")
    return rc


def _check_f32(name, t):
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous float32 tensor")


def _check_u8_cache(t):
    if t.dtype != torch.uint8 or t.dim() != 5 or not t.is_contiguous():
        raise ValueError("kv_cache_fp8: expected a contiguous 5-d uint8 tensor")


def kv_cache_store_fp8(k, v, cu_seqlens, context_lens, k_scale, v_scale, kv_cache_fp8, block_table,
                       status: Optional[torch.Tensor] = None, stream=None, raise_on_error: bool = True) -> int:
    """Quantize a call's K/V rows into their FP8 (e4m3) cache slots (C ABI
    ``kv_cache_store_fp8``); ``context_lens`` None means every context is 0."""
    _check_bf16("k", k, 3), _check_bf16("v", v, 3), _check_u8_cache(kv_cache_fp8)
    _check_i32("cu_seqlens", cu_seqlens), _check_i32("block_table", block_table)
    _check_f32("k_scale", k_scale), _check_f32("v_scale", v_scale)
    if context_lens is not None:
        _check_i32("context_lens", context_lens)
    T, G, D = k.shape
    rc = load().kv_cache_store_fp8(
        _ptr(k), _ptr(v), T, _ptr(cu_seqlens), _ptr(context_lens), cu_seqlens.numel() - 1, G, D, _ptr(k_scale),
        _ptr(v_scale), _ptr(kv_cache_fp8), kv_cache_fp8.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache_fp8.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "kv_cache_store_fp8")
    return rc


def prefill_attn_fp8_cache(q, k, v, cu_seqlens, max_seqlen: int, scale: float, k_scale, v_scale, out,
                           kv_cache_fp8, block_table, status: Optional[torch.Tensor] = None, stream=None,
                           raise_on_error: bool = True) -> int:
    """prefill_attn writing an FP8 (e4m3) cache (C ABI ``prefill_attn_fp8_cache``):
    the same attention output, the K/V rows stored as per-kv-head scaled codes."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3), _check_bf16("out", out, 3)
    _check_u8_cache(kv_cache_fp8), _check_i32("cu_seqlens", cu_seqlens), _check_i32("block_table", block_table)
    _check_f32("k_scale", k_scale), _check_f32("v_scale", v_scale)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn_fp8_cache(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1, int(max_seqlen), H, G, D,
        float(scale), _ptr(k_scale), _ptr(v_scale), _ptr(out), _ptr(kv_cache_fp8), kv_cache_fp8.shape[0],
        _ptr(block_table), block_table.shape[1] if block_table.dim() == 2 else block_table.numel(),
        kv_cache_fp8.shape[2], _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn_fp8_cache")
    return rc


def prefill_attn_chunked_fp8(q, k, v, cu_seqlens_q, context_lens, max_q_len: int, max_context_len: int,
                             scale: float, k_scale, v_scale, out, kv_cache_fp8, block_table,
                             status: Optional[torch.Tensor] = None, stream=None, raise_on_error: bool = True) -> int:
    """Chunked prefill over an FP8 (e4m3) cache (C ABI ``prefill_attn_chunked_fp8``):
    each chunk attends to its dequantized cached prefix and to its own rows
    quantized the same way, then its codes are appended."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3), _check_bf16("out", out, 3)
    _check_u8_cache(kv_cache_fp8), _check_i32("cu_seqlens_q", cu_seqlens_q), _check_i32("context_lens", context_lens)
    _check_i32("block_table", block_table), _check_f32("k_scale", k_scale), _check_f32("v_scale", v_scale)
    T, H, D = q.shape
    G = k.shape[1]
    rc = load().prefill_attn_chunked_fp8(
        _ptr(q), _ptr(k), _ptr(v), T, _ptr(cu_seqlens_q), _ptr(context_lens), cu_seqlens_q.numel() - 1,
        int(max_q_len), int(max_context_len), H, G, D, float(scale), _ptr(k_scale), _ptr(v_scale), _ptr(out),
        _ptr(kv_cache_fp8), kv_cache_fp8.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache_fp8.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "prefill_attn_chunked_fp8")
    return rc


def paged_decode_attn_fp8(q, k, v, context_lens, max_context_len: int, scale: float, k_scale, v_scale, out,
                          kv_cache_fp8, block_table, status: Optional[torch.Tensor] = None, stream=None,
                          raise_on_error: bool = True) -> int:
    """Decode step over an FP8 (e4m3) cache (C ABI ``paged_decode_attn_fp8``)."""
    _check_bf16("q", q, 3), _check_bf16("k", k, 3), _check_bf16("v", v, 3), _check_bf16("out", out, 3)
    _check_u8_cache(kv_cache_fp8), _check_i32("context_lens", context_lens), _check_i32("block_table", block_table)
    _check_f32("k_scale", k_scale), _check_f32("v_scale", v_scale)
    B, H, D = q.shape
    G = k.shape[1]
    rc = load().paged_decode_attn_fp8(
        _ptr(q), _ptr(k), _ptr(v), _ptr(context_lens), B, int(max_context_len), H, G, D, float(scale),
        _ptr(k_scale), _ptr(v_scale), _ptr(out), _ptr(kv_cache_fp8), kv_cache_fp8.shape[0], _ptr(block_table),
        block_table.shape[1] if block_table.dim() == 2 else block_table.numel(), kv_cache_fp8.shape[2],
        _ptr(status), _stream_ptr(stream))
    if rc != 0 and raise_on_error:
        raise PrefillError(rc, "paged_decode_attn_fp8")
    return rc


def inject_stall(enable: bool = True) -> None:
    """Test hook: the next pipelined launch withholds one Q tile so that a
    bounded device wait expires and the call reports PREFILL_ERR_TIMEOUT."""
    load().prefill_test_inject_stall(1 if enable else 0)


def exp2_fma2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """Test hook: the kernel's FMA-pipe exponential applied to a CUDA float32
    tensor (C ABI ``prefill_test_exp2_fma2``)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x: expected a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    rc = load().prefill_test_exp2_fma2(_ptr(x), _ptr(y), x.numel(), _stream_ptr(stream))
    if rc != 0:
        raise PrefillError(rc, "prefill_test_exp2_fma2")
    return y


def num_kv_blocks(qb: int, ctx: int, n: int, bm: int = 128, bn: int = 128) -> int:
    return load().prefill_num_kv_blocks(qb, ctx, n, bm, bn)


def kv_block_rule(qb: int, j: int, ctx: int, n: int, bm: int = 128, bn: int = 128):
    """(kind, col_limit[bm], key_begin): kind 0 = unmasked, 1 = masked, -1 = out of range."""
    lim = (ctypes.c_int32 * bm)()
    kb = ctypes.c_int32(0)
    kind = load().prefill_kv_block_rule(qb, j, ctx, n, bm, bn, lim, ctypes.byref(kb))
    return kind, list(lim), kb.value


def first_kv_block(qb: int, ctx: int, n: int, window: int, bm: int = 128, bn: int = 128) -> int:
    return load().prefill_first_kv_block(qb, ctx, n, bm, bn, window)


def kv_block_rule_window(qb: int, j: int, ctx: int, n: int, window: int, bm: int = 128, bn: int = 128):
    """(kind, col_lo[bm], col_limit[bm], key_begin) under a sliding window."""
    lo = (ctypes.c_int32 * bm)()
    lim = (ctypes.c_int32 * bm)()
    kb = ctypes.c_int32(0)
    kind = load().prefill_kv_block_rule_window(qb, j, ctx, n, bm, bn, window, lo, lim, ctypes.byref(kb))
    return kind, list(lo), list(lim), kb.value

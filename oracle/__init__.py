"""Oracle: TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU statement of the prefill attention path (see ``oracle.c``
for the definition and its sources).  Only ``tests/``, the smoke check and
the bench's CPU-baseline / reference legs may import this package; the
product library never does and shares no code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

# x86-64-v3 (AVX2/FMA) rather than -march=native: the shared object is built
# on one host and may run on another.
CFLAGS = ["-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB_PATH))
    return _lib


def _configure(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    prob = [P, P, P, P, P, I, I, I, I, D, P, I, P, I, I, I]
    lib.oracle_attention_rows.argtypes = prob + [P, P, I, P]
    lib.oracle_attention_all.argtypes = prob + [P]
    lib.oracle_softmax_weights.argtypes = prob + [I, I, P, P]
    lib.oracle_kv_write.argtypes = [P, P, P, P, I, I, I, P, I, P, I, I]
    for f in (lib.oracle_attention_rows, lib.oracle_attention_all,
              lib.oracle_softmax_weights, lib.oracle_kv_write):
        f.restype = I
    lib.oracle_num_threads.restype = I
    lib.oracle_set_num_threads.argtypes = [I]
    lib.oracle_set_num_threads.restype = None
    F = ctypes.c_float
    lib.oracle_e4m3_encode.argtypes = [F]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = D
    lib.oracle_kv_write_fp8.argtypes = [P, P, P, P, I, I, I, P, P, P, I, P, I, I]
    lib.oracle_kv_write_fp8.restype = I
    lib.oracle_decode_fp8.argtypes = [P, P, P, P, I, I, I, I, D, P, P, P, I, P, I, I, P]
    lib.oracle_decode_fp8.restype = I
    lib.oracle_chunked_fp8.argtypes = [P, P, P, P, P, I, I, I, I, D, P, P, P, I, P, I, I, P, P, I, P]
    lib.oracle_chunked_fp8.restype = I
    return lib


def _swap_library(path: str):
    """Use another build of ``oracle.c`` (the mutation tests load deliberately
    broken copies).  Returns the previous handle for ``_restore_library``."""
    global _lib
    old = _lib
    _lib = _configure(ctypes.CDLL(path))
    return old


def _restore_library(handle):
    global _lib
    _lib = handle


def _bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 numpy array of its bits."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.int32))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class _Problem:
    def __init__(self, q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale,
                 context_lens=None, kv_cache=None, block_table=None, block_size=16, window=0):
        if window < 0:
            raise ValueError("window must be >= 0 (0: no window)")
        self.q, self.k, self.v = _bits(q), _bits(k), _bits(v)
        self.cu = _i32(cu_seqlens)
        self.ctx = None if context_lens is None else _i32(context_lens)
        self.cache = None if kv_cache is None else _bits(kv_cache)
        self.bt = None if block_table is None else _i32(block_table)
        self.num_blocks = 0 if kv_cache is None else int(kv_cache.shape[0])
        self.mbps = 0 if block_table is None else int(self.bt.shape[1]) if self.bt.ndim == 2 else int(self.bt.shape[0])
        self.args = (_ptr(self.q), _ptr(self.k), _ptr(self.v), _ptr(self.cu), _ptr(self.ctx),
                     len(self.cu) - 1, n_head, n_kv_head, head_dim, float(scale),
                     _ptr(self.cache), self.num_blocks, _ptr(self.bt), self.mbps, block_size, int(window))
        self.n_head, self.head_dim = n_head, head_dim


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with oracle status {rc}")


def attention(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale, *,
              context_lens=None, kv_cache=None, block_table=None, block_size=16, window=0) -> np.ndarray:
    """Full output [T, n_head, head_dim] in fp64.  With ``context_lens`` the
    prefix keys come from ``kv_cache`` (as it stands) through ``block_table``.
    ``window`` W >= 1 limits row P to keys P-W+1 .. P (0: plain causal)."""
    p = _Problem(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale,
                 context_lens, kv_cache, block_table, block_size, window)
    T = int(p.cu[-1]) if len(p.cu) else 0
    out = np.zeros((T, n_head, head_dim), dtype=np.float64)
    _check(_load().oracle_attention_all(*p.args, _ptr(out)), "oracle_attention_all")
    return out


def attention_rows(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale, rows: Sequence[int],
                   heads: Sequence[int], *, context_lens=None, kv_cache=None, block_table=None,
                   block_size=16, window=0) -> np.ndarray:
    """Output rows for selected (packed row, head) pairs: [n_sel, head_dim] fp64."""
    p = _Problem(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale,
                 context_lens, kv_cache, block_table, block_size, window)
    r = _i32(rows)
    h = _i32(heads)
    assert r.shape == h.shape
    out = np.zeros((len(r), head_dim), dtype=np.float64)
    _check(_load().oracle_attention_rows(*p.args, _ptr(r), _ptr(h), len(r), _ptr(out)),
           "oracle_attention_rows")
    return out


def softmax_weights(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale, row: int, head: int, *,
                    context_lens=None, kv_cache=None, block_table=None, block_size=16,
                    window=0) -> np.ndarray:
    """Softmax weights of one (row, head) over keys 0 .. P (0 outside the window)."""
    p = _Problem(q, k, v, cu_seqlens, n_head, n_kv_head, head_dim, scale,
                 context_lens, kv_cache, block_table, block_size, window)
    mk = int(max((p.ctx[i] if p.ctx is not None else 0) + p.cu[i + 1] - p.cu[i]
                 for i in range(len(p.cu) - 1)))
    w = np.zeros(max(mk, 1), dtype=np.float64)
    n = ctypes.c_int(0)
    _check(_load().oracle_softmax_weights(*p.args, row, head, _ptr(w), ctypes.byref(n)),
           "oracle_softmax_weights")
    return w[: n.value]


def kv_write(k, v, cu_seqlens, kv_cache: torch.Tensor, block_table, block_size, *,
             context_lens=None) -> torch.Tensor:
    """Return a copy of ``kv_cache`` with every token's K/V written to its slot."""
    kb, vb = _bits(k), _bits(v)
    cu = _i32(cu_seqlens)
    ctx = None if context_lens is None else _i32(context_lens)
    bt = _i32(block_table)
    cache = _bits(kv_cache).copy()
    G, d = int(k.shape[1]), int(k.shape[2])
    rc = _load().oracle_kv_write(_ptr(kb), _ptr(vb), _ptr(cu), _ptr(ctx), len(cu) - 1, G, d,
                                 _ptr(cache), int(kv_cache.shape[0]), _ptr(bt), int(bt.shape[1]),
                                 block_size)
    _check(rc, "oracle_kv_write")
    return torch.from_numpy(cache.view(np.int16)).view(torch.bfloat16).reshape(kv_cache.shape)


def prefill(w, *, kv_cache=None, context_lens=None, rows=None, heads=None, window=0):
    """Oracle for one call on a ``workloads.Workload``-shaped problem:
    attention first (prefix read from the cache as it stood), then the KV
    write.  Returns (out fp64, new cache)."""
    cache = w.empty_cache() if kv_cache is None else kv_cache
    kw = dict(context_lens=context_lens, kv_cache=cache if context_lens is not None else None,
              block_table=w.block_table if context_lens is not None else None,
              block_size=w.block_size, window=window)
    if rows is None:
        out = attention(w.q, w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim, w.scale, **kw)
    else:
        out = attention_rows(w.q, w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim, w.scale,
                             rows, heads, **kw)
    new_cache = kv_write(w.k, w.v, w.cu_seqlens, cache, w.block_table, w.block_size,
                         context_lens=context_lens)
    return out, new_cache


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> int:
    """Run the parallel loops on n threads; returns the count now in effect."""
    _load().oracle_set_num_threads(int(n))
    return num_threads()


def qkv_projection(x, w, n_head: int, n_kv_head: int, head_dim: int):
    """The fused QKV projection (hncyxsy.com/news/270449 §4.1: one GEMM with the
    W_q, W_k, W_v blocks concatenated, its (s, (H + 2G) d) output cut by
    columns into Q, K, V; §2.2: each reshaped to (s, heads, head_dim)).

    x: [T, hidden] bf16; w: [(n_head + 2 n_kv_head) head_dim, hidden] bf16, one
    row per output feature (the Q block's rows first, then K's, then V's).
    Returns (q [T, H, d], k [T, G, d], v [T, G, d]) in fp64: the plain product
    y = x w^T in fp64 from the bf16 values, then the column split."""
    xs = x.detach().cpu().to(torch.float64).numpy()
    ws = w.detach().cpu().to(torch.float64).numpy()
    y = xs @ ws.T
    T = y.shape[0]
    hq, hk = n_head * head_dim, n_kv_head * head_dim
    assert y.shape[1] == hq + 2 * hk
    return (y[:, :hq].reshape(T, n_head, head_dim), y[:, hq:hq + hk].reshape(T, n_kv_head, head_dim),
            y[:, hq + hk:].reshape(T, n_kv_head, head_dim))


def out_projection(o, w_o):
    """The output projection after the attention (hncyxsy.com/news/270449 §3.3:
    the heads' outputs (s, n_head, head_dim) flattened back to (s, h), head
    after head, then one GEMM with W_o).

    o: [T, H, d] (any float dtype); w_o: [hidden, H d] bf16, one row per output
    feature.  Returns y [T, hidden] in fp64: the merge, then the plain product
    y = o_merged w_o^T in fp64."""
    os_ = o.detach().cpu().to(torch.float64).numpy() if isinstance(o, torch.Tensor) else np.asarray(o, np.float64)
    T = os_.shape[0]
    merged = os_.reshape(T, -1)
    ws = w_o.detach().cpu().to(torch.float64).numpy()
    assert ws.shape[1] == merged.shape[1]
    return merged @ ws.T


# ---------------------------------------------------------------- FP8 (e4m3) KV cache
def e4m3_encode(x: float) -> int:
    """e4m3 code of a float32 value: round to nearest (ties to even), magnitudes
    beyond 448 saturate to 448."""
    return int(_load().oracle_e4m3_encode(float(x)))


def e4m3_decode(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def _f32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def kv_write_fp8(k, v, cu_seqlens, kv_cache: torch.Tensor, block_table, block_size, k_scale, v_scale, *,
                 context_lens=None) -> torch.Tensor:
    """Copy of the FP8 cache (uint8 codes [NB, 2, bs, G, d]) with every token's K
    and V quantized into its slot: code = e4m3(fp32(x) / scale[g])."""
    kb, vb = _bits(k), _bits(v)
    cu = _i32(cu_seqlens)
    ctx = None if context_lens is None else _i32(context_lens)
    bt = _i32(block_table)
    ks, vs = _f32(k_scale), _f32(v_scale)
    cache = kv_cache.detach().cpu().contiguous().numpy().copy()
    assert cache.dtype == np.uint8
    G, d = int(k.shape[1]), int(k.shape[2])
    rc = _load().oracle_kv_write_fp8(_ptr(kb), _ptr(vb), _ptr(cu), _ptr(ctx), len(cu) - 1, G, d, _ptr(ks), _ptr(vs),
                                     _ptr(cache), int(kv_cache.shape[0]), _ptr(bt), int(bt.shape[1]), block_size)
    _check(rc, "oracle_kv_write_fp8")
    return torch.from_numpy(cache).reshape(kv_cache.shape)


def decode_fp8(q, k, v, context_lens, n_head, n_kv_head, head_dim, scale, k_scale, v_scale, kv_cache, block_table,
               block_size) -> np.ndarray:
    """Decode over an FP8 cache: the new token of sequence i (q [B, H, d],
    k/v [B, G, d]) attends to the dequantized cache entries 0 .. ctx_i - 1 and
    to its own K/V quantized the same way.  Returns [B, H, d] fp64."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    ctx = _i32(context_lens)
    bt = _i32(block_table)
    ks, vs = _f32(k_scale), _f32(v_scale)
    cache = kv_cache.detach().cpu().contiguous().numpy()
    B = len(ctx)
    out = np.zeros((B, n_head, head_dim), dtype=np.float64)
    rc = _load().oracle_decode_fp8(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(ctx), B, n_head, n_kv_head, head_dim,
                                   float(scale), _ptr(ks), _ptr(vs), _ptr(cache), int(kv_cache.shape[0]), _ptr(bt),
                                   int(bt.shape[1]), block_size, _ptr(out))
    _check(rc, "oracle_decode_fp8")
    return out


def chunked_fp8(q, k, v, cu_seqlens, context_lens, n_head, n_kv_head, head_dim, scale, k_scale, v_scale, kv_cache,
                block_table, block_size, *, rows=None, heads=None) -> np.ndarray:
    """Chunked prefill over an FP8 cache (hncyxsy.com/news/227904 §2.1 chunked
    prefill, §2.3 an FP8 KV cache with the softmax in higher precision): chunk
    row a of sequence i at position ctx_i + a attends to the dequantized cache
    entries 0 .. ctx_i - 1 and to the chunk's rows 0 .. a quantized with the
    same per-kv-head scales.  q [T, H, d], k/v [T, G, d] bf16; kv_cache uint8
    [NB, 2, bs, G, d] as it stood before the call.  Returns [T, H, d] fp64, or
    [n, d] for the selected (packed row, head) pairs."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cu, ctx, bt = _i32(cu_seqlens), _i32(context_lens), _i32(block_table)
    ks, vs = _f32(k_scale), _f32(v_scale)
    cache = kv_cache.detach().cpu().contiguous().numpy()
    T = int(cu[-1])
    if rows is None:
        sr = sh = None
        n_sel = -1
        out = np.zeros((T, n_head, head_dim), dtype=np.float64)
    else:
        sr, sh = _i32(rows), _i32(heads)
        n_sel = len(sr)
        out = np.zeros((n_sel, head_dim), dtype=np.float64)
    rc = _load().oracle_chunked_fp8(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(cu), _ptr(ctx), len(cu) - 1, n_head,
                                    n_kv_head, head_dim, float(scale), _ptr(ks), _ptr(vs), _ptr(cache),
                                    int(kv_cache.shape[0]), _ptr(bt), int(bt.shape[1]), block_size, _ptr(sr),
                                    _ptr(sh), n_sel, _ptr(out))
    _check(rc, "oracle_chunked_fp8")
    return out

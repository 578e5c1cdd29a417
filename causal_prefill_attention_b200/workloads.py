"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module draws random inputs and lays them out; it holds none of the
attention arithmetic.  Every workload is a prefill of one decoder layer's
attention: packed bf16 Q/K/V rows, ``cu_seqlens`` offsets, a paged KV pool
pre-filled with a sentinel bit pattern, and a per-sequence block table.

Shapes follow the workloads the source pages talk about: 8k-token prompts
(hncyxsy.com/news/270449, introduction), h=4096 with 32 heads of 128 and GQA
with 8 KV heads (same page, §3.4 "MHA 和 GQA 对 KV cache 数据量的影响"),
64 concurrent ~2k-token sequences (hncyxsy.com/news/227904, §4.1), and a
block size of 16 with 512-token prefill chunks (lnwmold.com/news/496245,
§3.3 "框架级优化技巧").

Draw order (fixed, so a seed names one input exactly): lengths -> Q -> K -> V
-> block-table permutation.  Values are ``randn`` fp32 rounded to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

# bf16 bit pattern written into every cache slot before a call, so that any
# slot the call must not touch can be checked bit for bit afterwards.
SENTINEL_BITS = 0xDEAD


def sentinel_value_int16() -> int:
    return SENTINEL_BITS - 0x10000 if SENTINEL_BITS >= 0x8000 else SENTINEL_BITS


@dataclass
class Workload:
    """One prefill call's inputs (host tensors)."""
    name: str
    seqlens: List[int]
    n_head: int
    n_kv_head: int
    head_dim: int
    scale: float
    block_size: int
    q: torch.Tensor            # [T, n_head, head_dim] bf16
    k: torch.Tensor            # [T, n_kv_head, head_dim] bf16
    v: torch.Tensor            # [T, n_kv_head, head_dim] bf16
    cu_seqlens: torch.Tensor   # [B+1] int32
    block_table: torch.Tensor  # [B, max_blocks_per_seq] int32, -1 = unused
    num_blocks: int
    chunk: Optional[int] = None  # query-chunk length for chunked prefill
    meta: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)

    @property
    def max_seqlen(self) -> int:
        return max(self.seqlens) if self.seqlens else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    def empty_cache(self) -> torch.Tensor:
        """Paged pool [num_blocks, 2, block_size, n_kv_head, head_dim] filled with the sentinel."""
        c = torch.full((self.num_blocks, 2, self.block_size, self.n_kv_head, self.head_dim),
                       sentinel_value_int16(), dtype=torch.int16)
        return c.view(torch.bfloat16)

    def causal_flops(self) -> float:
        """2*s^2*head_dim*n_head per sequence: the causal half of 4*s^2*d*H."""
        return float(sum(2.0 * s * s * self.head_dim * self.n_head for s in self.seqlens))

    def window_flops(self, window: int) -> float:
        """4*head_dim*n_head per visible (query, key) pair under a sliding window
        of ``window`` keys: row a of a sequence sees min(a + 1, window) keys."""
        pairs = 0
        for s in self.seqlens:
            w = min(s, window)
            pairs += w * (w + 1) // 2 + (s - w) * window
        return 4.0 * self.head_dim * self.n_head * pairs


def _bf16_randn(gen: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_workload(seqlens: List[int], n_head: int, n_kv_head: int, head_dim: int, *,
                  block_size: int = 16, seed: int = 0, name: str = "custom",
                  shuffle_pages: bool = True, extra_pages: int = 0,
                  max_blocks_per_seq: Optional[int] = None,
                  chunk: Optional[int] = None, scale: Optional[float] = None) -> Workload:
    """Build a packed varlen workload.

    Pages are dealt from one permutation of the pool in sequence order, so
    sequence i takes the next ceil(len_i / block_size) pages.  ``extra_pages``
    adds unused pages to the pool (they must keep the sentinel after a call).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return _build(gen, list(seqlens), n_head, n_kv_head, head_dim, block_size, name,
                  shuffle_pages, extra_pages, max_blocks_per_seq, chunk, scale)


def _build(gen, seqlens, n_head, n_kv_head, head_dim, block_size, name, shuffle_pages,
           extra_pages, max_blocks_per_seq, chunk, scale) -> Workload:
    T = sum(seqlens)
    q = _bf16_randn(gen, (T, n_head, head_dim))
    k = _bf16_randn(gen, (T, n_kv_head, head_dim))
    v = _bf16_randn(gen, (T, n_kv_head, head_dim))
    pages_per_seq = [-(-s // block_size) for s in seqlens]
    used = sum(pages_per_seq)
    num_blocks = max(1, used + extra_pages)
    if shuffle_pages:
        perm = torch.randperm(num_blocks, generator=gen).to(torch.int32)
    else:
        perm = torch.arange(num_blocks, dtype=torch.int32)
    mbps = max_blocks_per_seq if max_blocks_per_seq is not None else max(1, max(pages_per_seq, default=1))
    bt = torch.full((len(seqlens), mbps), -1, dtype=torch.int32)
    pos = 0
    for i, np_ in enumerate(pages_per_seq):
        bt[i, :np_] = perm[pos:pos + np_]
        pos += np_
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    if seqlens:
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    return Workload(name=name, seqlens=seqlens, n_head=n_head, n_kv_head=n_kv_head,
                    head_dim=head_dim, scale=scale if scale is not None else 1.0 / math.sqrt(head_dim),
                    block_size=block_size, q=q, k=k, v=v, cu_seqlens=cu, block_table=bt,
                    num_blocks=num_blocks, chunk=chunk)


# The five workloads the measurements and parity tests are quoted on.  Seed =
# 1000 + position in this list (1-based).
NAMED = (
    "mha_s128_h4_d64",
    "mha_s2048_h32_d128",
    "gqa_s8192_h32g8_d128",
    "varlen64_gqa_h32g8_d128",
    "chunked512_gqa_s8192_h32g8_d128",
)


def named_workload(name: str, seed: Optional[int] = None) -> Workload:
    idx = NAMED.index(name) + 1
    gen = torch.Generator(device="cpu")
    gen.manual_seed(1000 + idx if seed is None else seed)
    if name == "mha_s128_h4_d64":
        # identity block table over 8 pages
        return _build(gen, [128], 4, 4, 64, 16, name, False, 0, None, None, None)
    if name == "mha_s2048_h32_d128":
        return _build(gen, [2048], 32, 32, 128, 16, name, True, 0, None, None, None)
    if name == "gqa_s8192_h32g8_d128":
        return _build(gen, [8192], 32, 8, 128, 16, name, True, 0, None, None, None)
    if name == "varlen64_gqa_h32g8_d128":
        lens = torch.randint(256, 4097, (64,), generator=gen).tolist()
        return _build(gen, lens, 32, 8, 128, 16, name, True, 0, 4096 // 16, None, None)
    if name == "chunked512_gqa_s8192_h32g8_d128":
        return _build(gen, [8192], 32, 8, 128, 16, name, True, 0, None, 512, None)
    raise KeyError(name)


def chunk_views(w: Workload, chunk: int, seq: int = 0):
    """Split sequence ``seq`` of ``w`` into query chunks.

    Yields (q, k, v, cu_seqlens_q, context_lens, block_table_row) for each
    chunk: the chunk's own rows plus the number of earlier tokens it attends
    to (already in the cache when the chunk runs).
    """
    start = int(w.cu_seqlens[seq])
    n = w.seqlens[seq]
    bt = w.block_table[seq:seq + 1].contiguous()
    for c0 in range(0, n, chunk):
        L = min(chunk, n - c0)
        sl = slice(start + c0, start + c0 + L)
        yield (w.q[sl].contiguous(), w.k[sl].contiguous(), w.v[sl].contiguous(),
               torch.tensor([0, L], dtype=torch.int32), torch.tensor([c0], dtype=torch.int32), bt)


def decode_views(w: Workload):
    """Split every sequence of ``w`` into its prompt (all tokens but the last)
    and one decode token (the last).

    Returns (prompt_q, prompt_k, prompt_v, prompt_cu_seqlens, new_q, new_k,
    new_v, context_lens): the packed prompts, whose K/V a prefill call writes
    into the cache, and for each sequence the last token's q [B, H, d] and
    k, v [B, G, d] with its position (= its prompt length).  Every sequence
    needs at least one token; ``w``'s block table then has a page for the
    decode token's slot.
    """
    lens = [int(s) for s in w.seqlens]
    assert all(n >= 1 for n in lens), "every sequence needs its decode token"
    starts = w.cu_seqlens[:-1].tolist()
    keep = torch.cat([torch.arange(s, s + n - 1) for s, n in zip(starts, lens)]) if lens else torch.zeros(0, dtype=torch.long)
    last = torch.tensor([s + n - 1 for s, n in zip(starts, lens)], dtype=torch.long)
    ctx = torch.tensor([n - 1 for n in lens], dtype=torch.int32)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(ctx.to(torch.int64), 0).to(torch.int32)
    return (w.q[keep].contiguous(), w.k[keep].contiguous(), w.v[keep].contiguous(), cu,
            w.q[last].contiguous(), w.k[last].contiguous(), w.v[last].contiguous(), ctx)


def make_projection(tokens: int, hidden: int, n_head: int, n_kv_head: int, head_dim: int, seed: int):
    """Inputs of the fused QKV projection: activations x [tokens, hidden] and the
    concatenated weight w [(n_head + 2 n_kv_head) head_dim, hidden], bf16, drawn
    x ~ N(0, 1) then w ~ N(0, 1 / hidden) so that outputs are O(1)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    x = _bf16_randn(gen, (tokens, hidden))
    w = (torch.randn((n_head + 2 * n_kv_head) * head_dim, hidden, generator=gen, dtype=torch.float32)
         / math.sqrt(hidden)).to(torch.bfloat16)
    return x, w

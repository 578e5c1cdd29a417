"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on a
workload and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W

# Output tolerance for bf16 inputs with fp32 accumulation (the stated target).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev(w: W.Workload):
    d = torch.device("cuda:0")
    return dict(q=w.q.to(d), k=w.k.to(d), v=w.v.to(d), cu=w.cu_seqlens.to(d), bt=w.block_table.to(d))


def run_prefill(w: W.Workload, cache: torch.Tensor | None = None):
    """One prefill_attn call; returns (out bf16 cpu, cache bf16 cpu, status)."""
    t = to_dev(w)
    cache_d = (w.empty_cache() if cache is None else cache).cuda()
    out = torch.full_like(t["q"], float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.prefill_attn(t["q"], t["k"], t["v"], t["cu"], w.max_seqlen, w.scale, out, cache_d, t["bt"], status=status)
    torch.cuda.synchronize()
    return out.cpu(), cache_d.cpu(), int(status.item())


def run_chunked(w: W.Workload, chunk: int):
    """Prefill sequence 0 of ``w`` chunk by chunk; returns (out, cache, statuses)."""
    cache_d = w.empty_cache().cuda()
    outs, statuses = [], []
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for q, k, v, cu, ctx, bt in W.chunk_views(w, chunk):
        out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        status.zero_()
        _lib.prefill_attn_chunked(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), ctx.cuda(), int(cu[-1]), int(ctx[0]),
                                  w.scale, out, cache_d, bt.cuda(), status=status)
        torch.cuda.synchronize()
        statuses.append(int(status.item()))
        outs.append(out.cpu())
    return torch.cat(outs, 0), cache_d.cpu(), statuses


def compare_out(gpu_out: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = gpu_out.to(torch.float64).numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def assert_cache_bits_equal(a: torch.Tensor, b: torch.Tensor, what: str = ""):
    ai, bi = a.view(torch.int16), b.view(torch.int16)
    if not torch.equal(ai, bi):
        bad = (ai != bi).nonzero()
        raise AssertionError(f"{what}: {bad.shape[0]} cache elements differ, first at {bad[0].tolist()}")


def sample_rows(w: W.Workload, n_random: int, seed: int = 0, block: int = 128):
    """(row, head) pairs that reach every work item of the kernels.

    A work item is (sequence, head, pair of 128-row query blocks, split of the
    kv range), and every split of an item contributes to every row of its two
    blocks.  So for every sequence, every 128-row query block and EVERY head,
    the block's first and last valid rows are checked (on the 8k prompt:
    64 blocks x 2 rows x 32 heads = 4096 pairs), plus each sequence's edge
    rows and ``n_random`` random pairs."""
    rng = np.random.default_rng(seed)
    rows, heads = [], []
    for i, n in enumerate(w.seqlens):
        if n == 0:
            continue
        base = int(w.cu_seqlens[i])
        for b0 in range(0, n, block):
            for a in sorted({b0, min(b0 + block, n) - 1}):
                rows += [base + a] * w.n_head
                heads += list(range(w.n_head))
        for a in {1, n // 2}:
            rows.append(base + min(a, n - 1))
            heads.append(int(rng.integers(0, w.n_head)))
    T = w.total_tokens
    rows += rng.integers(0, T, n_random).tolist()
    heads += rng.integers(0, w.n_head, n_random).tolist()
    return rows, heads


def block_edge_rows(T: int, block: int = 128):
    """First and last row of every ``block``-row tile of a T-row GEMM output
    (every output tile of the projection kernels holds two of them)."""
    rows = set()
    for b0 in range(0, T, block):
        rows.add(b0)
        rows.add(min(b0 + block, T) - 1)
    return sorted(rows)

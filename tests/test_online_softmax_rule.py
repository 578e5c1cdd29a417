"""The blocked online-softmax rule, stated in fp64 and checked against the
oracle's two-pass softmax.

hncyxsy.com/news/270449 §3.2: S is produced block by block, so each block
keeps its own max and exp-sum, and when a new block raises the running max the
old partial results are rescaled before the new block is added; the weighted
sum is divided by the exp-sum once at the end.  The kernels use that rule with
three refinements, each stated here exactly as the kernels apply it:

* log2 units: scores are scaled by scale * log2(e) and exponentials are 2^x;
* lazy rescale: the running max moves only when a block's max exceeds it by
  more than TAU (8 in log2 units), so between moves P may reach 2^TAU; a row
  whose first block holds no visible key (a sliding window's lower edge) keeps
  a finite floor (-1e30) as its max until a visible key arrives;
* split-KV: a key range cut into parts gives per part an unnormalised O, its
  max and its exp-sum; the parts are merged by rescaling each to the largest
  max.

These are rules of arithmetic, not of the kernels' code: the tests show that,
in fp64, every variant equals the two-pass definition (1e-12), and that a rule
with a planted mistake does not.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import workloads as W

LOG2E = 1.0 / math.log(2.0)
NO_KEY_MAX = -1e30


def _visible(P, window):
    lo = max(0, P - window + 1) if window > 0 else 0
    return lo, P  # keys lo .. P


def _blocked_row(qrow, K, V, P, scale, bn, tau, window, j_range=None, mistake=None):
    """One query row at position P over key blocks of bn, as (O unnormalised,
    m in log2 units, l).  j_range restricts to kv blocks [a, b) (one split)."""
    lo, hi = _visible(P, window)
    nblk = hi // bn + 1
    # like the kernels, a row's visit starts at the block holding the lowest key
    # of its 128-row query block's first row, so under a window the leading
    # blocks can hold no key this row sees
    first = max(0, (P // 128) * 128 - window + 1) // bn if window > 0 else 0
    a, b = (first, nblk) if j_range is None else j_range
    m, l = NO_KEY_MAX, 0.0
    O = np.zeros(V.shape[1])
    for j in range(a, b):
        keys = [c for c in range(j * bn, min((j + 1) * bn, hi + 1)) if c >= lo]
        s = np.array([scale * LOG2E * float(qrow @ K[c]) for c in keys])
        m_blk = s.max() if keys else -math.inf  # a block with no visible key leaves the floor alone
        if m_blk > m + tau:  # move the max (always on the first visible block: m is the floor)
            alpha = 2.0 ** (m - m_blk)
            O *= alpha
            if mistake != "l_not_rescaled":
                l *= alpha
            m = m_blk
        if keys:
            p = 2.0 ** (s - m)
            l += p.sum()
            O += p @ V[keys]
    return O, m, l


def _combine(parts, mistake=None):
    M = max(m for _, m, _ in parts)
    O = sum((2.0 ** (m - M) if mistake != "no_split_rescale" else 1.0) * o for o, m, _ in parts)
    l = sum((2.0 ** (m - M) if mistake != "no_split_rescale" else 1.0) * ll for _, m, ll in parts)
    return O / l


def _inputs(n, H, G, d, seed, boost):
    w = W.make_workload([n], H, G, d, block_size=16, seed=seed)
    q = w.q.to(torch.float64).numpy() * boost  # larger scores: more moves of the running max
    return w, q, w.k.to(torch.float64).numpy(), w.v.to(torch.float64).numpy()


def _run(w, q, K, V, bn, tau, window, splits=1, mistake=None, rows=None):
    H, G, d = w.n_head, w.n_kv_head, w.head_dim
    r = H // G
    n = w.total_tokens
    out = np.zeros((n, H, d))
    for P in (range(n) if rows is None else rows):
        for h in range(H):
            g = h // r
            Kg, Vg = K[:, g, :], V[:, g, :]
            if splits == 1:
                O, m, l = _blocked_row(q[P, h], Kg, Vg, P, w.scale, bn, tau, window, mistake=mistake)
                out[P, h] = O / l
            else:
                nblk = P // bn + 1
                cuts = [nblk * s // splits for s in range(splits + 1)]
                parts = [_blocked_row(q[P, h], Kg, Vg, P, w.scale, bn, tau, window, (cuts[s], cuts[s + 1]),
                                      mistake=mistake)
                         for s in range(splits) if cuts[s + 1] > cuts[s]]
                parts = [p for p in parts if p[2] > 0.0]  # a part with no visible key contributes nothing
                out[P, h] = _combine(parts, mistake=mistake)
    return out


def _reference(w, q, window):
    qb = torch.from_numpy(q).to(torch.float64)
    # the oracle takes bf16 inputs: q scaled by a power of two stays exact in bf16
    return oracle.attention(qb.to(torch.bfloat16), w.k, w.v, w.cu_seqlens, w.n_head, w.n_kv_head, w.head_dim,
                            w.scale, window=window)


@pytest.mark.parametrize("bn,tau,boost", [(16, 8.0, 1.0), (16, 8.0, 8.0), (64, 8.0, 8.0), (128, 0.0, 8.0),
                                          (64, 0.0, 1.0)])
def test_blocked_lazy_rule_equals_two_pass(bn, tau, boost):
    w, q, K, V = _inputs(300, 4, 2, 16, seed=80, boost=boost)
    got = _run(w, q, K, V, bn, tau, 0)
    ref = _reference(w, q, 0)
    assert np.max(np.abs(got - ref)) < 1e-12


@pytest.mark.parametrize("window,bn", [(1, 16), (7, 16), (50, 16), (100, 64), (130, 128)])
def test_window_edge_floor_rule_equals_two_pass(window, bn):
    """Rows whose first blocks hold no visible key keep the floor max."""
    w, q, K, V = _inputs(300, 4, 2, 16, seed=81, boost=8.0)
    got = _run(w, q, K, V, bn, 8.0, window)
    ref = _reference(w, q, window)
    assert np.max(np.abs(got - ref)) < 1e-12


@pytest.mark.parametrize("splits", [2, 3, 5])
def test_split_combine_equals_two_pass(splits):
    w, q, K, V = _inputs(400, 4, 2, 16, seed=82, boost=8.0)
    got = _run(w, q, K, V, 16, 8.0, 0, splits=splits)
    ref = _reference(w, q, 0)
    assert np.max(np.abs(got - ref)) < 1e-12


@pytest.mark.parametrize("mistake,splits", [("l_not_rescaled", 1), ("no_split_rescale", 3)])
def test_planted_rule_mistakes_are_detected(mistake, splits):
    w, q, K, V = _inputs(300, 4, 2, 16, seed=83, boost=8.0)
    got = _run(w, q, K, V, 16, 0.0, 0, splits=splits, mistake=mistake)
    ref = _reference(w, q, 0)
    assert np.max(np.abs(got - ref)) > 1e-3

"""GPU parity of the fused QKV projection (qkv_projection) against the oracle:
y = x W^T (fp64 from the bf16 values) cut into Q | K | V; every output element
within the suite's tolerance (bf16 inputs, fp32 accumulation, one rounding to
bf16), and an identity weight reproduces x bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _run(x, w, H, G, d):
    T = x.shape[0]
    dev = torch.device("cuda")
    q = torch.full((T, H, d), float("nan"), dtype=torch.bfloat16, device=dev)
    k = torch.full((T, G, d), float("nan"), dtype=torch.bfloat16, device=dev)
    v = torch.full((T, G, d), float("nan"), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    _lib.qkv_projection(x.to(dev), w.to(dev), H, G, d, q, k, v, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return q.cpu(), k.cpu(), v.cpu()


@pytest.mark.parametrize("T,hid,H,G,d", [
    (1, 64, 2, 1, 64), (127, 128, 4, 2, 32), (128, 256, 2, 1, 64), (300, 512, 4, 2, 64),
    (129, 256, 8, 2, 128), (500, 1024, 16, 4, 64), (777, 192, 4, 4, 64),
])
def test_qkv_projection_matches_oracle(T, hid, H, G, d):
    x, w = W.make_projection(T, hid, H, G, d, seed=500 + T)
    q, k, v = _run(x, w, H, G, d)
    rq, rk, rv = oracle.qkv_projection(x, w, H, G, d)
    U.compare_out(q, rq, f"q T={T}")
    U.compare_out(k, rk, f"k T={T}")
    U.compare_out(v, rv, f"v T={T}")


def test_identity_weight_copies_activations_bit_exact():
    T, H, G, d = 333, 4, 2, 64
    N = (H + 2 * G) * d
    x, _ = W.make_projection(T, N, H, G, d, seed=510)
    w = torch.eye(N, dtype=torch.bfloat16)
    q, k, v = _run(x, w, H, G, d)
    y = torch.cat([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], dim=1)
    assert torch.equal(y.view(torch.int16), x.view(torch.int16))


def test_full_size_sampled_rows():
    """8192 tokens x hidden 4096 -> 32 q heads + 2 x 8 kv heads of 128 (the
    headline attention's inputs); both edge rows of every 128-row output tile
    and random rows, every column, against the oracle."""
    T, hid, H, G, d = 8192, 4096, 32, 8, 128
    x, w = W.make_projection(T, hid, H, G, d, seed=511)
    q, k, v = _run(x, w, H, G, d)
    # both edge rows of every 128-row output tile (every tile of the kernel), plus random rows
    rows = U.block_edge_rows(T) + np.random.default_rng(5).integers(0, T, 56).tolist()
    rq, rk, rv = oracle.qkv_projection(x[rows], w, H, G, d)
    U.compare_out(q[rows], rq, "q full")
    U.compare_out(k[rows], rk, "k full")
    U.compare_out(v[rows], rv, "v full")
    assert torch.isfinite(q.float()).all() and torch.isfinite(v.float()).all()


# ---------------------------------------------------------------- output projection W_o
def _run_out(o, w_o):
    T = o.shape[0]
    y = torch.full((T, w_o.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.attn_out_projection(o.cuda(), w_o.cuda(), y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return y.cpu()


def _out_inputs(T, H, d, hid, seed):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    w_o = (torch.randn(hid, H * d, generator=g) / np.sqrt(H * d)).to(torch.bfloat16)
    return o, w_o


@pytest.mark.parametrize("T,H,d,hid", [
    (1, 1, 64, 256), (127, 2, 64, 256), (300, 4, 32, 512), (129, 8, 128, 768), (500, 16, 64, 1024),
])
def test_out_projection_matches_oracle(T, H, d, hid):
    o, w_o = _out_inputs(T, H, d, hid, seed=520 + T)
    U.compare_out(_run_out(o, w_o), oracle.out_projection(o, w_o), f"y T={T}")


def test_out_projection_identity_weight_bit_exact():
    T, H, d = 333, 4, 64
    o, _ = _out_inputs(T, H, d, H * d, seed=530)
    y = _run_out(o, torch.eye(H * d, dtype=torch.bfloat16))
    assert torch.equal(y.view(torch.int16), o.reshape(T, -1).view(torch.int16))


def test_out_projection_full_size_sampled_rows():
    """8192 tokens: 32 heads x 128 merged -> hidden 4096; both edge rows of
    every 128-row output tile and random rows, every column."""
    T, H, d, hid = 8192, 32, 128, 4096
    o, w_o = _out_inputs(T, H, d, hid, seed=531)
    y = _run_out(o, w_o)
    rows = U.block_edge_rows(T) + np.random.default_rng(6).integers(0, T, 56).tolist()
    U.compare_out(y[rows], oracle.out_projection(o[rows], w_o), "y full")
    assert torch.isfinite(y.float()).all()


def test_projection_attention_projection_chain():
    """x -> qkv_projection -> prefill_attn -> attn_out_projection on the GPU,
    against the oracle's chain in fp64 (projections, attention, projection)."""
    lens, H, G, d, hid = [700, 300], 8, 2, 128, 1024
    T = sum(lens)
    x, w = W.make_projection(T, hid, H, G, d, seed=532)
    _, w_o = _out_inputs(1, H, d, hid, seed=533)
    q, k, v = _run(x, w, H, G, d)
    cu = torch.tensor([0, lens[0], T], dtype=torch.int32)
    bs, mbps = 16, (max(lens) + 15) // 16
    nb = sum((n + bs - 1) // bs for n in lens)
    bt = torch.full((2, mbps), -1, dtype=torch.int32)
    bt[0, :(lens[0] + bs - 1) // bs] = torch.arange((lens[0] + bs - 1) // bs, dtype=torch.int32)
    bt[1, :(lens[1] + bs - 1) // bs] = torch.arange((lens[0] + bs - 1) // bs, nb, dtype=torch.int32)
    cache = torch.zeros(nb, 2, bs, G, d, dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / np.sqrt(d)
    _lib.prefill_attn(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lens), scale, out, cache, bt.cuda())
    y = _run_out(out.cpu(), w_o)
    # oracle chain: the attention takes bf16 inputs, so it is fed the oracle's
    # projections rounded to bf16 (round to nearest even, as the GPU stores them)
    rq, rk, rv = (torch.from_numpy(a).to(torch.bfloat16) for a in oracle.qkv_projection(x, w, H, G, d))
    ro = oracle.attention(rq, rk, rv, cu, H, G, d, scale)
    U.compare_out(y, oracle.out_projection(ro, w_o), "chain")

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
    headline attention's inputs); sampled rows against the oracle."""
    T, hid, H, G, d = 8192, 4096, 32, 8, 128
    x, w = W.make_projection(T, hid, H, G, d, seed=511)
    q, k, v = _run(x, w, H, G, d)
    rows = [0, 1, 127, 128, 4095, 4096, 8190, 8191] + np.random.default_rng(5).integers(0, T, 56).tolist()
    rq, rk, rv = oracle.qkv_projection(x[rows], w, H, G, d)
    U.compare_out(q[rows], rq, "q full")
    U.compare_out(k[rows], rk, "k full")
    U.compare_out(v[rows], rv, "v full")
    assert torch.isfinite(q.float()).all() and torch.isfinite(v.float()).all()

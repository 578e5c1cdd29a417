"""Failure path on the GPU without a fault or a hang: a test hook makes the
pipelined kernel's producer withhold one Q tile, so a consumer's bounded wait
(about one second) expires.  The call must report PREFILL_ERR_TIMEOUT, every
role must stop and release its resources, and the same CUDA context must then
run a normal call correctly."""
import time

import numpy as np
import pytest
import torch

import oracle
from causal_prefill_attention_b200 import _lib
from causal_prefill_attention_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def test_stalled_pipeline_reports_timeout_and_context_survives():
    w = W.make_workload([600, 300], 8, 2, 128, seed=61)
    t = U.to_dev(w)
    cache = w.empty_cache().cuda()
    out = torch.zeros_like(t["q"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.inject_stall(True)
    t0 = time.time()
    rc = _lib.prefill_attn(t["q"], t["k"], t["v"], t["cu"], w.max_seqlen, w.scale, out, cache, t["bt"], status=status)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert rc == 0  # the launch itself succeeded
    assert int(status.item()) == 6, _lib.status_string(int(status.item()))
    assert elapsed < 30.0
    # the context is intact: a normal call on fresh buffers gives correct results
    out2, cache2, st2 = U.run_prefill(w)
    assert st2 == 0
    ref_out, ref_cache = oracle.prefill(w)
    U.assert_cache_bits_equal(cache2, ref_cache, "after timeout")
    U.compare_out(out2, ref_out, "after timeout")


def test_hook_resets_after_one_launch():
    w = W.make_workload([256], 4, 2, 128, seed=62)
    _lib.inject_stall(True)
    _, _, st1 = U.run_prefill(w)
    _, _, st2 = U.run_prefill(w)
    assert st1 == 6 and st2 == 0

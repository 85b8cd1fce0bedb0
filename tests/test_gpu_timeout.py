"""Failure detection without a GPU fault: every wait in the attention kernel is bounded. Setting
the bound to zero makes the waits run out; the kernel must record it, drain its own copies and
tensor-core work, free its tensor memory and return, leaving the context usable."""
import numpy as np
import pytest
import torch

import gen
import long_context_sparse_stripe_b200 as s2o

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    w = gen.Workload("timeout", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=2048, head_dim=128,
                     segment_len=512, block_size=128, tau=0.02, seed=21)
    q, k, v = (t.cuda() for t in gen.make_inputs(w))
    cfg = s2o.Config.of(w)
    idx = s2o.build_indices(cfg, q, k)
    ref = s2o.attention_prefill_with_indices(cfg, q, k, v, idx)
    assert s2o.check_device_status() == 0
    s2o.set_wait_limit_ns(0)
    try:
        s2o.attention_prefill_with_indices(cfg, q, k, v, idx)
        status = s2o.check_device_status()
    finally:
        s2o.set_wait_limit_ns(2_000_000_000)
    assert status == 6  # S2O_ERR_DEVICE_TIMEOUT
    assert s2o.check_device_status() == 0  # the record was cleared
    again = s2o.attention_prefill_with_indices(cfg, q, k, v, idx)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    assert torch.equal(again, ref)

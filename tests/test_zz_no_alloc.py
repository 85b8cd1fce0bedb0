"""s2o_build_indices_static: the index build for callers that cannot allocate device memory.

Some callers only get their inputs and outputs handed to them (an operator embedded in another
framework, a serving loop that must not call cudaMalloc once running), so they cannot provide the
scratch workspace that s2o_build_indices takes. The static entry point uses a fixed scratch array
inside the library instead. These tests call it through the C ABI and check it against the
existing entry point on consecutive calls; the file is named to run last.
"""
import numpy as np
import pytest
import torch

import gen
import long_context_sparse_stripe_b200 as s2o

SMALL = gen.Workload("no-alloc-small", batch=1, n_q_heads=4, n_kv_heads=2, seq_len=4096,
                     head_dim=128, segment_len=1024, block_size=128, tau=0.01, seed=31)
MEDIUM = gen.Workload("no-alloc-medium", batch=2, n_q_heads=8, n_kv_heads=2, seq_len=12288,
                      head_dim=64, segment_len=1536, block_size=64, tau=0.005, seed=32)


def assert_same_indices(a: s2o.Indices, b: s2o.Indices):
    for name in ("perm_q", "perm_k", "sel_cnt", "local_tiles"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    cnt = a.sel_cnt.cpu().numpy()
    sa, sb = a.sel_blk.cpu().numpy(), b.sel_blk.cpu().numpy()
    nB = sa.shape[-1]
    listed = np.arange(nB)[None, None, None, :] < cnt[..., None]
    np.testing.assert_array_equal(np.where(listed, sa, -1), np.where(listed, sb, -1))


# The size the array is advertised for: a 32-query-head, 8-KV-head, 32K-token layer with d = 128
# (its scratch reaches close to the end of the array).
LLAMA_32K = gen.workload("llama-32k")


def test_static_scratch_covers_the_advertised_layer():
    assert s2o.workspace_size(s2o.Config.of(LLAMA_32K)) <= s2o.STATIC_WORKSPACE_BYTES


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    # Different layers back to back (each call finds the previous call's leftovers in the shared
    # array), the largest one the array is sized for among them, then the first layer again.
    for w in (SMALL, MEDIUM, LLAMA_32K, SMALL):
        cfg = s2o.Config.of(w)
        assert s2o.workspace_size(cfg) <= s2o.STATIC_WORKSPACE_BYTES
        q, k, _ = (t.cuda() for t in gen.make_inputs(w))
        want = s2o.build_indices(cfg, q, k)
        got = s2o.build_indices_static(cfg, q, k, out=s2o.alloc_indices(cfg))
        torch.cuda.synchronize()
        assert_same_indices(got, want)


def test_static_scratch_rejects_layers_beyond_its_size():
    cfg = s2o.Config.of(gen.workload("llama-128k"))
    assert s2o.workspace_size(cfg) > s2o.STATIC_WORKSPACE_BYTES
    fake = s2o._Indices(0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    status = s2o._load().s2o_build_indices_static(
        __import__("ctypes").byref(cfg._c()), 0x1000, 0x1000,
        __import__("ctypes").byref(fake), None)
    assert status == 3  # S2O_ERR_WORKSPACE_TOO_SMALL, returned before any device work

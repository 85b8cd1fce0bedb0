"""Parity at the benchmark configurations' full sizes, in the launch configuration bench.py times.

The GPU runs the whole layer (all 32 query heads, every kernel as the bench launches it); the CPU
oracle recomputes every KV group (4 query heads each) of the same inputs — each head's indices
depend only on its own queries and its group's keys — and a sample of output rows of each group:
every segment's first and last row of its heads, rows of query blocks that selected permuted
blocks, and random rows. Index arrays must be bit-exact for all heads, outputs within max-abs 2e-2
and mean-abs 1e-3 of the oracle's binary64 result. The 32-layer stack checks every layer, one KV
group per layer (group l mod 8 for layer l, so the eight groups are all covered).

Inputs of one workload are generated once (about half a minute on the host for a 128K layer) and
reused for its variants (τ, segment length, query permutation off), which is how the ablation
configurations differ.
"""
import numpy as np
import pytest
import torch

import gen
import long_context_sparse_stripe_b200 as s2o
import oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 1e-3
_inputs = {}


def inputs(w):
    key = (w.name, w.seed, w.seq_len, w.stripe_frac)
    if key not in _inputs:
        _inputs.clear()
        _inputs[key] = gen.make_inputs(w)
    return _inputs[key]


def group_slice(w, q, k, v, g):
    G = w.n_q_heads // w.n_kv_heads
    sub = w.replace(n_q_heads=G, n_kv_heads=1)
    return (sub, q[:, g * G:(g + 1) * G].contiguous(), k[:, g:g + 1].contiguous(),
            v[:, g:g + 1].contiguous())


def check_layer(w, groups=None, n_random=384, seed=0):
    q, k, v = inputs(w)
    cfg = s2o.Config.of(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, idx = s2o.attention_prefill(cfg, qd, kd, vd)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    G = w.n_q_heads // w.n_kv_heads
    nB = w.seq_len // w.block_size
    rng = np.random.default_rng(seed)
    selected = 0
    if groups is None:
        groups = range(w.n_kv_heads)
    for g in groups:
        sub, qs, ks, vs = group_slice(w, q, k, v, g)
        ocfg = oracle.config(sub)
        ref = oracle.build_indices(ocfg, qs, ks)
        heads = slice(g * G, (g + 1) * G)
        for name in ("perm_q", "perm_k", "sel_cnt", "local_tiles"):
            got = getattr(idx, name)[:, heads].cpu().numpy()
            np.testing.assert_array_equal(got, ref[name], err_msg=f"{w.name} group {g}: {name}")
        cnt = ref["sel_cnt"]
        sel = idx.sel_blk[:, heads].cpu().numpy()
        mask = np.arange(nB)[None, None, None, :] < cnt[..., None]
        np.testing.assert_array_equal(np.where(mask, sel, -1), ref["sel_blk"],
                                      err_msg=f"{w.name} group {g}: sel_blk")
        selected += int(cnt.sum())
        total = G * w.seq_len
        edge = [h * w.seq_len + s0 + e for h in range(G)
                for s0 in range(0, w.seq_len, w.segment_len) for e in (0, w.segment_len - 1)]
        # Rows of query blocks with selected blocks (the permuted pass) are sampled on purpose.
        perm_q = ref["perm_q"].reshape(G, w.seq_len)
        busy = np.argwhere(cnt.reshape(G, nB) > 0)
        busy_rows = [h * w.seq_len + perm_q[h, b * w.block_size + e]
                     for h, b in busy[rng.permutation(len(busy))[:16]] for e in (0, 63, 127)]
        rows = np.unique(np.concatenate([rng.choice(total, n_random, replace=False), edge,
                                         np.array(busy_rows, dtype=np.int64)]))
        want, _ = oracle.attention(ocfg, qs, ks, vs, ref, rows=rows)
        got = o[:, heads].reshape(-1, w.head_dim)[torch.from_numpy(rows).cuda()]
        err = np.abs(got.float().cpu().numpy().astype(np.float64) - want)
        assert err.max() <= MAX_ABS, f"{w.name} group {g}: max abs error {err.max():.3g}"
        assert err.mean() <= MEAN_ABS, f"{w.name} group {g}: mean abs error {err.mean():.3g}"
    return selected


def test_llama_32k():
    check_layer(gen.workload("llama-32k"))


@pytest.mark.parametrize("tau", [0.005, 0.01, 0.02])
def test_llama_128k_tau_sweep(tau):
    check_layer(gen.workload("llama-128k", tau=tau))


def test_llama_128k_strong_stripes():
    """The labelled strong-stripe workload: dozens of selected blocks per query block, so the
    permuted pass (and the permuted copy of K and V it takes at this density) does most of the
    work."""
    selected = check_layer(gen.workload("llama-128k-strong"), n_random=256)
    assert selected > 100000


def test_dense_kernel_full_size_sampled_rows():
    """The in-repo dense baseline (the bench's MSE reference and speed baseline) at 128K against
    Eq. 1 on sampled rows: the first and last row of every head and random rows."""
    w = gen.workload("llama-128k")
    q, k, v = inputs(w)
    cfg = s2o.Config.of(w)
    o = s2o.dense_causal_prefill(cfg, *(t.cuda() for t in (q, k, v)))
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    rng = np.random.default_rng(3)
    total = w.n_q_heads * w.seq_len
    heads = np.arange(w.n_q_heads) * w.seq_len
    rows = np.unique(np.concatenate([heads, heads + w.seq_len - 1,
                                     rng.choice(total, 192, replace=False)]))
    want = oracle.dense_causal(oracle.config(w), q, k, v, rows=rows)
    got = o.reshape(-1, w.head_dim)[torch.from_numpy(rows).cuda()]
    err = np.abs(got.float().cpu().numpy().astype(np.float64) - want)
    assert err.max() <= MAX_ABS, f"max abs error {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"mean abs error {err.mean():.3g}"


@pytest.mark.parametrize("variant", ["tau0.001", "S1024", "S4096", "qperm-off", "shared-keys",
                                     "int4-centroids"])
def test_qwen_128k_ablation(variant):
    w = gen.workload("qwen-128k")
    w = {"tau0.001": w.replace(tau=0.001), "S1024": w.replace(segment_len=1024),
         "S4096": w.replace(segment_len=4096), "qperm-off": w.replace(query_perm=0),
         "shared-keys": w.replace(shared_key_order=1),
         "int4-centroids": w.replace(int4_centroids=1)}[variant]
    selected = check_layer(w, n_random=256 if variant == "tau0.001" else 384)
    if variant == "tau0.001":
        assert selected > 0  # the permuted pass does real work at this threshold


@pytest.mark.parametrize("layer", range(32))
def test_stack_layer(layer):
    check_layer(gen.layer_workload(layer), groups=(layer % 8,), n_random=128, seed=layer)

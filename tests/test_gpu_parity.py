"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on the same seeded inputs.

Index arrays and every intermediate value of the index build must be bit-exact; attention
outputs must be within max-abs 2e-2 and mean-abs 1e-3 of the oracle's binary64 result when run
on the oracle's own indices (bf16 tensor-core products with fp32 accumulation against binary64).
"""
import numpy as np
import pytest
import torch

import gen
import long_context_sparse_stripe_b200 as s2o
import oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 1e-3

W_A = gen.Workload("a-d128-b128", batch=1, n_q_heads=4, n_kv_heads=2, seq_len=4096, head_dim=128,
                   segment_len=1024, block_size=128, tau=0.01, seed=5)
# Ragged: N is not a power of two (the key sort's last merge pairs 8192 with 4096 words) and S is
# not a multiple of the 2048-word segment sort tile; two batch elements.
W_B = gen.Workload("b-ragged", batch=2, n_q_heads=4, n_kv_heads=2, seq_len=12288, head_dim=128,
                   segment_len=1536, block_size=128, tau=0.01, seed=6)
W_C = gen.Workload("c-d64-b128", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=2048, head_dim=64,
                   segment_len=512, block_size=128, tau=0.02, seed=8)
W_D = gen.Workload("d-d128-b64", batch=1, n_q_heads=2, n_kv_heads=2, seq_len=2048, head_dim=128,
                   segment_len=512, block_size=64, tau=0.02, seed=9)
# Segments longer than one CTA's sort (S > 4096): the query ordering takes the multi-CTA radix
# sort, and the key ordering then runs before the query-side kernels instead of next to them.
W_E = gen.Workload("e-long-segments", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=16384,
                   head_dim=64, segment_len=8192, block_size=128, tau=0.01, seed=10)
# Ragged everywhere: a key run of 1.5 radix tiles, 96 blocks (not a multiple of the 32-block
# chunks of the schedule or of the 128-block score tiles), 3072-query segments.
W_F = gen.Workload("f-ragged-tiles", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=6144,
                   head_dim=64, segment_len=3072, block_size=64, tau=0.01, seed=11)
# One segment spanning the whole sequence (the local window is the causal triangle of all keys).
W_G = gen.Workload("g-one-segment", batch=1, n_q_heads=2, n_kv_heads=2, seq_len=4096,
                   head_dim=128, segment_len=4096, block_size=128, tau=0.01, seed=12)
# A segment that is not a whole number of 128-row chunks (320 = 2·128 + 64): the fused
# ρ/order/Q̄ kernel stages a partial last chunk.
W_H = gen.Workload("h-partial-chunk", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=1920,
                   head_dim=64, segment_len=320, block_size=64, tau=0.01, seed=15)
W_TINY = gen.workload("tiny")

INDEX_NAMES = ("perm_q", "perm_k", "sel_cnt", "local_tiles")
VIEW_NAMES = ("qbar", "kbar_all", "kbar_top", "u", "kappa", "rho", "Qbar", "Kbar", "r", "n")

_inputs_cache = {}


def inputs(w):
    key = (w.name, w.seed, w.seq_len, w.batch)
    if key not in _inputs_cache:
        _inputs_cache.clear()
        _inputs_cache[key] = gen.make_inputs(w)
    return _inputs_cache[key]


def to_dev(*ts):
    return [t.cuda() for t in ts]


def gpu_indices(w, q, k):
    cfg = s2o.Config.of(w)
    ws = s2o.alloc_workspace(cfg)
    idx = s2o.build_indices(cfg, q, k, ws=ws)
    torch.cuda.synchronize()
    return cfg, idx, ws


def assert_indices_equal(idx, ref, nB):
    for name in INDEX_NAMES:
        got = getattr(idx, name).cpu().numpy()
        np.testing.assert_array_equal(got, ref[name], err_msg=name)
    cnt = ref["sel_cnt"]
    sel = idx.sel_blk.cpu().numpy()
    mask = np.arange(nB)[None, None, None, :] < cnt[..., None]
    np.testing.assert_array_equal(np.where(mask, sel, -1), ref["sel_blk"], err_msg="sel_blk")


def oracle_indices_on_device(ref):
    return s2o.Indices(*(torch.from_numpy(np.ascontiguousarray(ref[n])).cuda()
                         for n in ("perm_q", "perm_k", "sel_cnt", "sel_blk", "local_tiles")))


def assert_close(got_bf16, want_f64):
    got = got_bf16.float().cpu().numpy().astype(np.float64).reshape(want_f64.shape)
    err = np.abs(got - want_f64)
    assert err.max() <= MAX_ABS, f"max abs error {err.max():.3g}"
    assert err.mean() <= MEAN_ABS, f"mean abs error {err.mean():.3g}"


# ----------------------------------------------------------------------------- exp64

def test_exp64_bit_exact_with_oracle():
    xs = np.concatenate([-np.linspace(0, 720, 40001), -np.geomspace(1e-300, 50, 4001),
                         [0.0, -0.0, -699.9999, -700.0, -700.0000001]])
    got = s2o.exp64_eval(torch.from_numpy(xs).cuda()).cpu().numpy()
    want = np.array([oracle.exp64(x) for x in xs])
    np.testing.assert_array_equal(got.view(np.uint64), want.view(np.uint64))


# ----------------------------------------------------------------------------- index build

@pytest.mark.parametrize("w", [
    W_TINY, W_TINY.replace(tau=0.0), W_TINY.replace(tau=0.07), W_TINY.replace(tau=0.2),
    W_TINY.replace(tau=1.5), W_A, W_A.replace(query_perm=0), W_B, W_C, W_D, W_E, W_F, W_G, W_H,
    W_A.replace(shared_key_order=1), W_B.replace(shared_key_order=1),
    W_E.replace(shared_key_order=1),
    W_TINY.replace(int4_centroids=1), W_A.replace(int4_centroids=1), W_C.replace(int4_centroids=1),
    W_F.replace(int4_centroids=1), W_B.replace(shared_key_order=1, int4_centroids=1),
], ids=lambda w: f"{w.name}-tau{w.tau}-qp{w.query_perm}-sk{w.shared_key_order}"
                 f"-i4{w.int4_centroids}")
def test_indices_and_intermediates_bit_exact(w):
    q, k, _ = inputs(w)
    ref = oracle.build_indices(oracle.config(w), q, k, debug=True)
    cfg, idx, ws = gpu_indices(w, *to_dev(q, k))
    assert_indices_equal(idx, ref, cfg.n_blocks)
    views = s2o.workspace_views(cfg, ws)
    for name in VIEW_NAMES:
        got = views[name].cpu().numpy()
        want = ref[name]
        np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32), err_msg=name)


def test_index_build_is_deterministic():
    q, k, _ = inputs(W_B)
    qd, kd = to_dev(q, k)
    _, a, _ = gpu_indices(W_B, qd, kd)
    _, b, _ = gpu_indices(W_B, qd, kd)
    for name in ("perm_q", "perm_k", "sel_cnt", "local_tiles"):
        assert torch.equal(getattr(a, name), getattr(b, name))


@pytest.mark.parametrize("tau", [0.25, 0.125, float(np.nextafter(np.float32(0.25), np.float32(1)))],
                         ids=["quarter", "eighth", "above-quarter"])
def test_scores_equal_to_tau_bit_exact(tau):
    """Block scores that equal τ exactly (the stop keeps a block with p = τ). Every key is the
    same vector, so the key scores tie (identity key ordering) and the candidate blocks of
    segment s (the 4s key blocks before it, 64 visible keys each) share one weight: p = 1/(4s)
    exactly, 1/4 in segment 1 and 1/8 in segment 2. Indices bit-exact with the oracle and the
    list lengths of the closed form."""
    w = W_TINY.replace(tau=tau)
    N, d = w.seq_len, w.head_dim
    rng = np.random.default_rng(3)
    q = torch.from_numpy(rng.standard_normal((1, 1, N, d), dtype=np.float32)).to(torch.bfloat16)
    k = torch.tensor([1.0, -0.5, 0.25, 2.0] * (d // 4)).repeat(1, 1, N, 1).to(torch.bfloat16)
    ref = oracle.build_indices(oracle.config(w), q, k)
    cfg, idx, _ = gpu_indices(w, *to_dev(q, k))
    assert_indices_equal(idx, ref, cfg.n_blocks)
    per_segment = {0.25: [0, 4, 0, 0], 0.125: [0, 4, 8, 0]}.get(tau, [0, 0, 0, 0])
    np.testing.assert_array_equal(ref["sel_cnt"][0, 0], np.repeat(per_segment, 4))


@pytest.mark.parametrize("case", ["keys", "query-row"])
def test_non_finite_inputs_keep_valid_orderings(case):
    """Non-finite inputs (outside the definition's domain, but the index arrays must stay valid):
    a NaN score has the smallest sort key, so it goes after every number, ties by lower index.
    "keys": three NaN key rows and one key with an infinite element; the mean key is NaN, so
    every query score is NaN and the query ordering is the identity. "query-row": one NaN query
    row; the pooled query is NaN, so every key score is NaN (identity key ordering) and the row
    goes last in its segment. The orderings and local tiles are bit-exact with the oracle; the
    lists (unspecified when a score is not finite) only have to be valid."""
    w = W_TINY
    q, k, _ = inputs(w)
    q, k = q.clone(), k.clone()
    N, S = w.seq_len, w.segment_len
    if case == "keys":
        k[0, 0, [5, 300, 777]] = float("nan")
        k[0, 0, 901, 3] = float("inf")
    else:
        q[0, 0, 700] = float("nan")
    ref = oracle.build_indices(oracle.config(w), q, k)
    cfg, idx, ws = gpu_indices(w, *to_dev(q, k))
    for name in ("perm_q", "perm_k", "local_tiles"):
        np.testing.assert_array_equal(getattr(idx, name).cpu().numpy(), ref[name], err_msg=name)
    assert s2o.validate_indices(cfg, idx, ws)
    if case == "keys":
        np.testing.assert_array_equal(ref["perm_k"][0, 0, -3:], [5, 300, 777])
        np.testing.assert_array_equal(ref["perm_q"][0, 0], np.arange(N))
    else:
        np.testing.assert_array_equal(ref["perm_k"][0, 0], np.arange(N))
        assert ref["perm_q"][0, 0, (700 // S + 1) * S - 1] == 700


# ----------------------------------------------------------------------------- attention

@pytest.mark.parametrize("w", [W_TINY, W_TINY.replace(tau=0.07), W_TINY.replace(tau=1.5), W_A,
                               W_A.replace(query_perm=0), W_C, W_D, W_F, W_G, W_H],
                         ids=lambda w: f"{w.name}-tau{w.tau}-qp{w.query_perm}")
def test_attention_on_oracle_indices(w):
    q, k, v = inputs(w)
    cfg = oracle.config(w)
    ref = oracle.build_indices(cfg, q, k)
    want, _ = oracle.attention(cfg, q, k, v, ref)
    qd, kd, vd = to_dev(q, k, v)
    o = s2o.attention_prefill_with_indices(s2o.Config.of(w), qd, kd, vd,
                                           oracle_indices_on_device(ref))
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    assert_close(o, want)


def test_full_path_ragged_sampled_rows():
    w = W_B
    q, k, v = inputs(w)
    cfg = oracle.config(w)
    ref = oracle.build_indices(cfg, q, k)
    qd, kd, vd = to_dev(q, k, v)
    o, idx = s2o.attention_prefill(s2o.Config.of(w), qd, kd, vd)
    torch.cuda.synchronize()
    assert_indices_equal(idx, ref, w.seq_len // w.block_size)
    rng = np.random.default_rng(0)
    total = w.batch * w.n_q_heads * w.seq_len
    # every segment's first and last rows plus a random sample
    edge = [(bh * w.seq_len + s0 + e) for bh in range(w.batch * w.n_q_heads)
            for s0 in range(0, w.seq_len, w.segment_len) for e in (0, w.segment_len - 1)]
    rows = np.unique(np.concatenate([rng.choice(total, 3000, replace=False), edge]))
    want, _ = oracle.attention(cfg, q, k, v, ref, rows=rows)
    got = o.reshape(-1, w.head_dim)[torch.from_numpy(rows).cuda()]
    assert_close(got, want)


@pytest.mark.parametrize("w", [W_TINY, W_A, W_C, W_D], ids=lambda w: w.name)
def test_dense_causal_kernel(w):
    q, k, v = inputs(w)
    want = oracle.dense_causal(oracle.config(w), q, k, v)
    qd, kd, vd = to_dev(q, k, v)
    o = s2o.dense_causal_prefill(s2o.Config.of(w), qd, kd, vd)
    torch.cuda.synchronize()
    assert_close(o, want)


@pytest.mark.parametrize("w", [W_TINY.replace(tau=0.0), W_A.replace(tau=0.0)],
                         ids=["tiny", "a-d128-b128"])
def test_tau_zero_matches_dense_causal(w):
    """τ = 0 keeps every candidate block, so the whole path (index build, then both attention
    passes) is dense causal attention, Eq. 1, on the same bf16 inputs (the tiny configuration's
    exact dense check; its fp32 inputs are rounded to bf16 before both sides run)."""
    q, k, v = inputs(w)
    want = oracle.dense_causal(oracle.config(w), q, k, v)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    o, idx = s2o.attention_prefill(cfg, qd, kd, vd)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    assert s2o.index_stats(cfg, idx).pair_sparsity == 0.0
    assert_close(o, want)


def test_permutation_invariance_full_selection():
    """Arbitrary orderings with every block listed: the output is dense causal attention."""
    w = W_A
    q, k, v = inputs(w)
    B, H, N = w.batch, w.n_q_heads, w.seq_len
    nB, S = N // w.block_size, w.segment_len
    rng = np.random.default_rng(3)
    perm_k = np.stack([np.stack([rng.permutation(N) for _ in range(H)]) for _ in range(B)])
    perm_q = np.empty_like(perm_k)
    for b in range(B):
        for h in range(H):
            for s0 in range(0, N, S):
                perm_q[b, h, s0:s0 + S] = s0 + rng.permutation(S)
    blk = perm_q.reshape(B, H, nB, w.block_size)
    lt = (blk.max(-1) - (np.arange(nB) * w.block_size // S * S)) // w.block_size + 1
    ref = dict(perm_q=perm_q.astype(np.int32), perm_k=perm_k.astype(np.int32),
               sel_cnt=np.full((B, H, nB), nB, np.int32),
               sel_blk=np.broadcast_to(rng.permutation(nB).astype(np.int32), (B, H, nB, nB)),
               local_tiles=lt.astype(np.int32))
    want = oracle.dense_causal(oracle.config(w), q, k, v)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    idx = oracle_indices_on_device(ref)
    assert s2o.validate_indices(cfg, idx)
    o = s2o.attention_prefill_with_indices(cfg, qd, kd, vd, idx)
    torch.cuda.synchronize()
    assert_close(o, want)


# ----------------------------------------------------------------------------- validation/stats

def test_validate_indices_accepts_and_rejects():
    w = W_A
    q, k, _ = inputs(w)
    cfg, idx, ws = gpu_indices(w, *to_dev(q, k))
    assert s2o.validate_indices(cfg, idx, ws)
    nB = cfg.n_blocks

    def corrupted(fn):
        c = s2o.Indices(*(t.clone() for t in (idx.perm_q, idx.perm_k, idx.sel_cnt, idx.sel_blk,
                                              idx.local_tiles)))
        fn(c)
        return c

    bad = [
        corrupted(lambda c: c.perm_k[0, 1, :2].copy_(torch.tensor([5, 5]))),      # duplicate
        corrupted(lambda c: c.perm_k[0, 0, 7].fill_(w.seq_len)),                   # range
        corrupted(lambda c: c.perm_q[0, 2, 3].fill_(w.segment_len + 3)),           # other segment
        corrupted(lambda c: c.sel_cnt[0, 0, nB - 1].fill_(nB + 1)),                # count
        corrupted(lambda c: (c.sel_cnt[0, 3, nB - 2].fill_(2),
                             c.sel_blk[0, 3, nB - 2, :2].copy_(torch.tensor([4, 4])))),
        corrupted(lambda c: (c.sel_cnt[0, 3, nB - 2].fill_(1),
                             c.sel_blk[0, 3, nB - 2, :1].fill_(-1))),
        corrupted(lambda c: c.local_tiles[0, 1, 9].fill_(0)),
        corrupted(lambda c: c.local_tiles[0, 1, 9].fill_(w.segment_len // w.block_size + 1)),
    ]
    for i, c in enumerate(bad):
        assert not s2o.validate_indices(cfg, c, ws), i


@pytest.mark.parametrize("w", [W_TINY.replace(tau=0.07), W_A, W_B], ids=lambda w: w.name)
def test_index_stats_match_oracle(w):
    q, k, _ = inputs(w)
    ref = oracle.build_indices(oracle.config(w), q, k)
    cfg, idx, ws = gpu_indices(w, *to_dev(q, k))
    st = s2o.index_stats(cfg, idx, ws)
    assert st.pairs == oracle.pair_count(oracle.config(w), ref)
    assert st.local_tiles == int(ref["local_tiles"].sum())
    assert st.selected_tiles == int(ref["sel_cnt"].sum())
    N = w.seq_len
    assert st.causal_pairs == w.batch * w.n_q_heads * N * (N + 1) // 2


def test_sparsity_monotone_in_tau_on_gpu():
    w = W_B
    q, k, _ = inputs(w)
    qd, kd = to_dev(q, k)
    prev = None
    for tau in (0.0, 0.002, 0.005, 0.01, 0.02, 0.05, 2.0):
        cfg, idx, ws = gpu_indices(w.replace(tau=tau), qd, kd)
        pairs = s2o.index_stats(cfg, idx, ws).pairs
        if prev is not None:
            assert pairs <= prev
        prev = pairs


def test_attention_independent_of_grid_and_windows():
    """A grid of one, two or five CTAs makes every CTA walk several work-list windows (the work
    list holds 128 work items): the local, permuted and dense passes give the same bits as the
    full grid, and the selected blocks of the ragged case reach the permuted pass."""
    w = W_B
    q, k, v = inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    idx = s2o.build_indices(cfg, qd, kd)
    assert int(idx.sel_cnt.sum()) > 0
    base = s2o.attention_prefill_with_indices(cfg, qd, kd, vd, idx)
    dense = s2o.dense_causal_prefill(cfg, qd, kd, vd)
    try:
        for n in (1, 2, 5):
            s2o.set_attention_max_ctas(n)
            o = s2o.attention_prefill_with_indices(cfg, qd, kd, vd, idx)
            d = s2o.dense_causal_prefill(cfg, qd, kd, vd)
            torch.cuda.synchronize()
            assert s2o.check_device_status() == 0
            assert torch.equal(o, base), f"grid of {n}: S2O output differs"
            assert torch.equal(d, dense), f"grid of {n}: dense output differs"
    finally:
        s2o.set_attention_max_ctas(0)


# ----------------------------------------------------------------------------- merge path, packed streams

# Strong stripes (dozens of selected blocks per query block) on shapes the oracle finishes in
# seconds: d = 128 with B = 128, and d = 64 with B = 64 and 32 blocks per segment.
W_S1 = gen.Workload("s1-strong-d128", batch=1, n_q_heads=4, n_kv_heads=1, seq_len=8192,
                    head_dim=128, segment_len=1024, block_size=128, tau=0.01, seed=21, amp=16.0,
                    stripe_frac=0.05, q_shift=4.0)
W_S2 = gen.Workload("s2-strong-d64-b64", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=8192,
                    head_dim=64, segment_len=2048, block_size=64, tau=0.01, seed=22, amp=12.0,
                    stripe_frac=0.05, q_shift=4.0)
# Ragged: two batch elements, 96 blocks, 1536-query segments (12 blocks), 3 query heads per KV head
# (pairs of heads straddle KV heads under one key ordering per KV head).
W_S3 = gen.Workload("s3-strong-ragged", batch=2, n_q_heads=6, n_kv_heads=2, seq_len=12288,
                    head_dim=128, segment_len=1536, block_size=128, tau=0.005, seed=23, amp=16.0,
                    stripe_frac=0.05, q_shift=4.0)


def _copy_flag(cfg, ws):
    at = s2o.workspace_size(cfg)
    return int(ws[at:at + 4].cpu().numpy().view(np.uint32)[0])


def _with_mode(mode, fn):
    try:
        s2o.set_permuted_copy(mode)
        out = fn()
        torch.cuda.synchronize()
        return out
    finally:
        s2o.set_permuted_copy(1)


@pytest.mark.parametrize("w", [W_A.replace(tau=0.0), W_C.replace(tau=0.0), W_D.replace(tau=0.0),
                               W_F.replace(tau=0.0), W_H.replace(tau=0.0), W_A.replace(tau=0.01),
                               W_S1, W_S2, W_S3, W_S3.replace(query_perm=0)],
                         ids=lambda w: f"{w.name}-tau{w.tau}-qp{w.query_perm}")
def test_merge_and_packed_paths_match_oracle(w):
    """On the oracle's indices, every form of steps 3-4 gives the oracle's output: the merge path
    with gathered selected blocks (mode 0), the merge path with packed streams from the permuted
    copy (mode 2: only the visible keys of each block, in 16-row chunks, blocks two paired query
    blocks both selected loaded once), and the path without a workspace (mode 3: the permuted pass
    reruns the local tiles)."""
    q, k, v = inputs(w)
    ocfg = oracle.config(w)
    ref = oracle.build_indices(ocfg, q, k)
    want, _ = oracle.attention(ocfg, q, k, v, ref)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    idx = oracle_indices_on_device(ref)
    ws = s2o.alloc_prefill_workspace(cfg)
    for mode, flag in ((0, 2), (2, 3), (3, None)):
        o = _with_mode(mode, lambda: s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx,
                                                                           ws))
        assert s2o.check_device_status() == 0, mode
        if flag is not None:
            assert _copy_flag(cfg, ws) == flag
        assert_close(o, want)


def test_permuted_copy_decision():
    """Mode 1 merges and packs when the selected blocks outnumber twice the copied blocks: with
    every block selected (τ = 0) it does both; with none (τ > 1) neither, and the call then runs
    the kernels of the path without a workspace (same bits)."""
    for w, expect in ((W_A.replace(tau=0.0), 3), (W_A.replace(tau=1.5), 0)):
        q, k, v = to_dev(*inputs(w))
        cfg = s2o.Config.of(w)
        idx = s2o.build_indices(cfg, q, k)
        ws = s2o.alloc_prefill_workspace(cfg)
        ws[s2o.workspace_size(cfg):s2o.workspace_size(cfg) + 4].fill_(7)
        o = s2o.attention_prefill_with_indices_ws(cfg, q, k, v, idx, ws)
        torch.cuda.synchronize()
        assert _copy_flag(cfg, ws) == expect, w.name
        if expect == 0:
            small = s2o.alloc_workspace(cfg)
            o_small = s2o.attention_prefill_with_indices_ws(cfg, q, k, v, idx, small)
            torch.cuda.synchronize()
            assert torch.equal(o, o_small)


@pytest.mark.parametrize("w", [W_B.replace(tau=0.001), W_S3], ids=["b-ragged", "s3-strong"])
def test_permuted_copy_per_kv_head_under_shared_key_order(w):
    """The whole path with one key ordering per KV head copies K and V once per KV head and pairs
    two query heads of a KV head at one block, so a block both selected is loaded once for both:
    every mode agrees with the oracle on sampled rows, and the indices stay the oracle's."""
    w = w.replace(shared_key_order=1)
    q, k, v = inputs(w)
    ocfg = oracle.config(w)
    ref = oracle.build_indices(ocfg, q, k)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    ws = s2o.alloc_prefill_workspace(cfg)
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(w.batch * w.n_q_heads * w.seq_len, 1500, replace=False))
    want, _ = oracle.attention(ocfg, q, k, v, ref, rows=rows)
    for mode in (0, 2, 3):
        o, idx = _with_mode(mode, lambda: s2o.attention_prefill(cfg, qd, kd, vd, ws=ws))
        assert s2o.check_device_status() == 0
        assert int(idx.sel_cnt.sum()) > 0
        assert_indices_equal(idx, ref, cfg.n_blocks)
        got = o.reshape(-1, w.head_dim)[torch.from_numpy(rows).cuda()]
        assert_close(got, want)


def test_packed_path_independent_of_grid_and_windows():
    """Packed streams and the merge with a grid of one, two or five CTAs (several work-list windows
    each) give the same bits as the full grid."""
    w = W_S3
    q, k, v = inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w)
    idx = s2o.build_indices(cfg, qd, kd)
    ws = s2o.alloc_prefill_workspace(cfg)
    base = _with_mode(2, lambda: s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx, ws))
    try:
        for n in (1, 2, 5):
            s2o.set_attention_max_ctas(n)
            o = _with_mode(2, lambda: s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx,
                                                                            ws))
            assert s2o.check_device_status() == 0
            assert torch.equal(o, base), f"grid of {n}"
    finally:
        s2o.set_attention_max_ctas(0)


def test_attention_work_counts():
    """The work report: gathered selected blocks run once per unit (mode 0); packed streams run
    about the attended pairs, and load each tile once even when both units of a pair use it."""
    w = W_S1
    q, k, v = to_dev(*inputs(w))
    cfg = s2o.Config.of(w)
    idx = s2o.build_indices(cfg, q, k)
    ws = s2o.alloc_prefill_workspace(cfg)
    st = s2o.index_stats(cfg, idx)
    per_seg = w.segment_len // w.block_size
    local = w.n_q_heads * (w.seq_len // w.segment_len) * per_seg * (per_seg + 1) // 2
    _with_mode(0, lambda: s2o.attention_prefill_with_indices_ws(cfg, q, k, v, idx, ws))
    gathered = s2o.attention_work(cfg, idx, ws)
    assert gathered.merged and not gathered.packed
    assert gathered.local_pass_tiles == local
    assert gathered.permuted_unit_tiles == gathered.permuted_loaded_tiles == st.selected_tiles
    _with_mode(2, lambda: s2o.attention_prefill_with_indices_ws(cfg, q, k, v, idx, ws))
    packed = s2o.attention_work(cfg, idx, ws)
    assert packed.packed and packed.merged and packed.local_pass_tiles == local
    attended = st.pairs / w.block_size ** 2
    assert packed.unit_tiles < 1.3 * attended
    assert packed.permuted_unit_tiles < gathered.permuted_unit_tiles
    assert packed.permuted_loaded_tiles < packed.permuted_unit_tiles


# ----------------------------------------------------------------------------- online early stop

# Full candidate lists (built at τ = 0) on GPU-supported shapes, so that later blocks carry little
# mass and the measured-share stop cuts them: d = 64 with B = 64, and d = 128 with B = 128 and GQA.
W_OS1 = gen.Workload("os1-d64-b64", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=2048, head_dim=64,
                     segment_len=256, block_size=64, tau=0.0, seed=13, amp=4.0, stripe_count=60,
                     diag=0.5)
W_OS2 = gen.Workload("os2-d128-b128", batch=1, n_q_heads=4, n_kv_heads=2, seq_len=8192,
                     head_dim=128, segment_len=1024, block_size=128, tau=0.0, seed=14, amp=4.0,
                     stripe_frac=0.02, diag=0.5)
STOP_TOL = 0.05  # relative band around τ inside which the GPU and the oracle may decide apart


@pytest.mark.parametrize("w,tau", [(W_OS1, 0.03), (W_OS1, 0.08), (W_OS2, 0.02), (W_OS2, 0.03)],
                         ids=["os1-0.03", "os1-0.08", "os2-0.02", "os2-0.03"])
def test_online_stop_matches_oracle(w, tau):
    """The measured-share stop (the definition's online-stop section) on the oracle's full
    candidate lists: every GPU stop position agrees with the oracle's shares (blocks the GPU went
    past have an oracle share of at least τ·(1 − 5 %), the block it stopped after one below
    τ·(1 + 5 %)), the stops actually cut lists, and the output equals the oracle's attention over
    the GPU's kept blocks."""
    q, k, v = inputs(w)
    ref = oracle.build_indices(oracle.config(w), q, k)
    ocfg = oracle.config(w, tau=tau)
    stop_o, share = oracle.online_stop(ocfg, q, k, ref)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w, tau=tau)
    o, stop = s2o.attention_prefill_online_stop(cfg, qd, kd, vd, oracle_indices_on_device(ref))
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    stop_g = stop.cpu().numpy()
    cnt = ref["sel_cnt"]
    assert (stop_g <= cnt).all() and ((stop_g > 0) == (cnt > 0)).all()
    assert (stop_g < cnt).sum() > 0, "no list was cut"
    for idx in np.argwhere(stop_g != stop_o):
        g, c = int(stop_g[tuple(idx)]), int(cnt[tuple(idx)])
        sh = share[tuple(idx)]
        assert (sh[:g - 1] >= tau * (1 - STOP_TOL)).all(), (idx, g, sh[:g])
        if g < c:
            assert sh[g - 1] < tau * (1 + STOP_TOL), (idx, g, sh[g - 1])
    agree = (stop_g == stop_o).mean()
    assert agree > 0.95, f"only {agree:.3f} of the stop positions agree"
    want, _ = oracle.attention(oracle.config(w), q, k, v, oracle.with_counts(ref, stop_g))
    assert_close(o, want)


def test_online_stop_tau_zero_keeps_lists_and_output():
    """τ = 0 never stops: the kept counts are the list lengths and the output is the path
    without a workspace, bit for bit (the same products in the same order)."""
    w = W_A
    q, k, v = to_dev(*inputs(w))
    cfg = s2o.Config.of(w, tau=0.0)
    idx = s2o.build_indices(cfg, q, k)
    o, stop = s2o.attention_prefill_online_stop(cfg, q, k, v, idx)
    base = s2o.attention_prefill_with_indices(cfg, q, k, v, idx)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    assert torch.equal(stop, idx.sel_cnt)
    assert torch.equal(o, base)


def test_online_stop_independent_of_grid():
    w = W_OS1
    q, k, v = inputs(w)
    ref = oracle.build_indices(oracle.config(w), q, k)
    qd, kd, vd = to_dev(q, k, v)
    cfg = s2o.Config.of(w, tau=0.05)
    idx = oracle_indices_on_device(ref)
    o0, s0 = s2o.attention_prefill_online_stop(cfg, qd, kd, vd, idx)
    try:
        for n in (1, 3):
            s2o.set_attention_max_ctas(n)
            o, st = s2o.attention_prefill_online_stop(cfg, qd, kd, vd, idx)
            torch.cuda.synchronize()
            assert s2o.check_device_status() == 0
            assert torch.equal(st, s0) and torch.equal(o, o0), f"grid of {n}"
    finally:
        s2o.set_attention_max_ctas(0)

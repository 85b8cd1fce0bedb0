"""Pins for the CPU oracle: what the pages and the mathematics fix, checked on the CPU.

Each test ties the oracle to something other than itself: a hand-worked case, a library routine
that the method reduces to in a special case (torch's causal scaled-dot-product attention at
τ = 0, per-segment causal attention at τ > 1), invariants the pages state (tensors are never moved,
so permutations leave the output unchanged; blocks are visited in importance order and the loop
stops at τ, so the selected sets are nested), libm for exp64, and float64 re-derivations of every
pooled quantity. A dropped term, a wrong sign or index, or a transposed operand anywhere in the
oracle fails at least one of them.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_case.json")

SMALL_GQA = gen.Workload("small-gqa", batch=2, n_q_heads=4, n_kv_heads=2, seq_len=512,
                         head_dim=64, segment_len=128, block_size=64, tau=0.05, seed=7,
                         amp=4.0, stripe_count=12, diag=0.5)


def _hand():
    with open(GOLDEN) as f:
        g = json.load(f)
    c = g["config"]
    q = torch.tensor(g["q"], dtype=torch.bfloat16).reshape(1, 1, 8, 4)
    k = torch.tensor(g["k"], dtype=torch.bfloat16).reshape(1, 1, 8, 4)
    v = torch.arange(32, dtype=torch.float32).reshape(1, 1, 8, 4).to(torch.bfloat16)
    return g, c, q, k, v


def _cfg(c, tau, query_perm=1):
    return oracle.Config(c["batch"], c["n_q_heads"], c["n_kv_heads"], c["seq_len"],
                         c["head_dim"], c["segment_len"], c["block_size"], tau, query_perm)


def _sdpa_causal(q, k, v, G):
    """torch's causal SDPA in float64 (K/V heads shared by G query heads)."""
    q64, k64, v64 = (x.to(torch.float64) for x in (q, k, v))
    k64 = k64.repeat_interleave(G, dim=1)
    v64 = v64.repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, is_causal=True)


def _sdpa_segment_local(q, k, v, G, S):
    outs = []
    for s0 in range(0, q.shape[2], S):
        sl = slice(s0, s0 + S)
        outs.append(_sdpa_causal(q[:, :, sl], k[:, :, sl], v[:, :, sl], G))
    return torch.cat(outs, dim=2)


# ----------------------------------------------------------------------------- hand case

def test_hand_case_intermediates():
    g, c, q, k, _ = _hand()
    idx = oracle.build_indices(_cfg(c, 0.3), q, k, debug=True)
    for name in ("qbar", "kbar_all", "kappa", "kbar_top", "u", "rho", "Qbar", "Kbar", "r"):
        np.testing.assert_array_equal(idx[name].reshape(-1), np.asarray(g[name], np.float32)
                                      .reshape(-1), err_msg=name)
    np.testing.assert_array_equal(idx["perm_k"][0, 0], g["perm_k"])
    np.testing.assert_array_equal(idx["perm_q"][0, 0], g["perm_q"])
    np.testing.assert_array_equal(idx["n"][0, 0], g["n"])
    np.testing.assert_array_equal(idx["local_tiles"][0, 0], g["local_tiles"])


def test_hand_case_probabilities_closed_form():
    g, c, q, k, _ = _hand()
    p = oracle.build_indices(_cfg(c, 0.3), q, k, debug=True)["p"][0, 0]
    z2 = 1 + math.exp(-0.25) + 2 * math.exp(-0.625)
    z3 = 2 + 2 * math.exp(-0.25)
    want = np.array([[0, 0, 0, 0], [0, 0, 0, 0],
                     [1 / z2, math.exp(-0.25) / z2, 2 * math.exp(-0.625) / z2, 0],
                     [1 / z3, 1 / z3, 2 * math.exp(-0.25) / z3, 0]])
    np.testing.assert_allclose(p, want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("tau", ["0.0", "0.28", "0.3", "0.4", "0.5"])
def test_hand_case_selection_and_pairs(tau):
    g, c, q, k, v = _hand()
    cfg = _cfg(c, float(tau))
    idx = oracle.build_indices(cfg, q, k)
    want = g["selection"][tau]
    for b, sel in enumerate(want["sel"]):
        assert idx["sel_cnt"][0, 0, b] == len(sel)
        np.testing.assert_array_equal(idx["sel_blk"][0, 0, b, :len(sel)], sel)
        assert (idx["sel_blk"][0, 0, b, len(sel):] == -1).all()
    assert oracle.pair_count(cfg, idx) == want["pairs"]
    _, pairs = oracle.attention(cfg, q, k, v, idx)
    assert pairs == want["pairs"]


def test_hand_case_key_sets():
    """At τ = 0.3 row i attends exactly to the hand-derived key set: compare with SDPA over it."""
    g, c, q, k, v = _hand()
    cfg = _cfg(c, 0.3)
    idx = oracle.build_indices(cfg, q, k)
    rows = np.array([4, 5, 6, 7])
    out, _ = oracle.attention(cfg, q, k, v, idx, rows=rows)
    for x, i in enumerate(rows):
        keys = g["key_sets_tau_0.3"][str(i)]
        mask = torch.zeros(1, 8, dtype=torch.bool)
        mask[0, keys] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[0, 0, i:i + 1].double(), k[0, 0].double(), v[0, 0].double(), attn_mask=mask)
        np.testing.assert_allclose(out[x], ref[0].numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- exp64 / constants

def test_exp64_constants_from_high_precision():
    getcontext().prec = 60
    ln2 = Decimal(2).ln()
    inv = 1 / ln2

    def nearest(x):
        return float(x)  # Decimal -> float is correctly rounded

    assert nearest(inv).hex() == "0x1.71547652b82fep+0"
    hi = nearest(ln2)
    assert hi.hex() == "0x1.62e42fefa39efp-1"
    assert nearest(ln2 - Decimal(hi)).hex() == "0x1.abc9e3b39803fp-56"


def test_score_scale_constants():
    getcontext().prec = 60
    for d, want in ((64, "0x1.0000000000000p-3"), (128, "0x1.6a09e60000000p-4")):
        exact = 1 / Decimal(d).sqrt()
        f32 = np.float32(float(exact))  # float(Decimal) then float32: double rounding is safe here
        assert float(f32).hex() == want
        assert float(np.float32(oracle.score_scale(d))).hex() == want
        # nearest-to-exact check without double rounding: neighbours are farther away
        lo, hi = np.nextafter(f32, np.float32(0)), np.nextafter(f32, np.float32(1))
        err = abs(Decimal(float(f32)) - exact)
        assert err <= abs(Decimal(float(lo)) - exact) and err <= abs(Decimal(float(hi)) - exact)


def test_exp64_within_two_ulp_of_libm():
    xs = np.concatenate([-np.linspace(0, 700, 20001), -np.geomspace(1e-300, 1, 2001),
                         [-0.0, -0.5 * math.log(2), -math.log(2), -699.999]])
    worst = 0.0
    for x in xs:
        got, ref = oracle.exp64(float(x)), math.exp(float(x))
        worst = max(worst, abs(got - ref) / math.ulp(ref))
    assert worst <= 2.0, worst
    assert oracle.exp64(-700.5) == 0.0
    assert oracle.exp64(0.0) == 1.0


# ----------------------------------------------------------------------------- special cases

@pytest.mark.parametrize("w", [gen.workload("tiny"), SMALL_GQA], ids=["tiny", "small-gqa"])
def test_tau_zero_is_dense_causal_attention(w):
    """τ = 0 keeps every candidate block, so the key set is [0, i]: Eq. 1 exactly."""
    q, k, v = gen.make_inputs(w)
    cfg = oracle.config(w, tau=0.0)
    idx = oracle.build_indices(cfg, q, k)
    out, pairs = oracle.attention(cfg, q, k, v, idx)
    ref = _sdpa_causal(q, k, v, w.n_q_heads // w.n_kv_heads).reshape(-1, w.head_dim)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-10)
    N = w.seq_len
    assert pairs == w.batch * w.n_q_heads * N * (N + 1) // 2
    np.testing.assert_allclose(oracle.dense_causal(cfg, q, k, v), ref.numpy(), rtol=0, atol=1e-10)


@pytest.mark.parametrize("w", [gen.workload("tiny"), SMALL_GQA], ids=["tiny", "small-gqa"])
def test_tau_above_one_is_local_window_only(w):
    """τ > 1 selects nothing: each query sees only its own segment causally."""
    q, k, v = gen.make_inputs(w)
    cfg = oracle.config(w, tau=1.5)
    idx = oracle.build_indices(cfg, q, k)
    assert (idx["sel_cnt"] == 0).all()
    out, _ = oracle.attention(cfg, q, k, v, idx)
    ref = _sdpa_segment_local(q, k, v, w.n_q_heads // w.n_kv_heads, w.segment_len)
    np.testing.assert_allclose(out, ref.reshape(-1, w.head_dim).numpy(), rtol=0, atol=1e-10)


def test_permutation_invariance_with_full_selection():
    """Arbitrary key and segment-local query orderings with every block selected give Eq. 1:
    the orderings only relabel addresses, the tensors are never moved."""
    w = SMALL_GQA
    q, k, v = gen.make_inputs(w)
    cfg = oracle.config(w)
    rng = np.random.default_rng(11)
    B, Hq, N = w.batch, w.n_q_heads, w.seq_len
    nB, S = N // w.block_size, w.segment_len
    perm_k = np.stack([np.stack([rng.permutation(N) for _ in range(Hq)]) for _ in range(B)])
    perm_q = np.empty_like(perm_k)
    for b in range(B):
        for h in range(Hq):
            for s0 in range(0, N, S):
                perm_q[b, h, s0:s0 + S] = s0 + rng.permutation(S)
    sel_blk = np.broadcast_to(rng.permutation(nB).astype(np.int32), (B, Hq, nB, nB)).copy()
    idx = dict(perm_q=perm_q.astype(np.int32), perm_k=perm_k.astype(np.int32),
               sel_cnt=np.full((B, Hq, nB), nB, np.int32), sel_blk=sel_blk)
    out, _ = oracle.attention(cfg, q, k, v, idx)
    ref = _sdpa_causal(q, k, v, w.n_q_heads // w.n_kv_heads).reshape(-1, w.head_dim)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-10)


def test_segment_zero_is_dense_for_any_tau():
    w = SMALL_GQA
    q, k, v = gen.make_inputs(w)
    ref = _sdpa_causal(q, k, v, w.n_q_heads // w.n_kv_heads)
    S = w.segment_len
    for tau in (0.0, 0.05, 0.5, 2.0):
        cfg = oracle.config(w, tau=tau)
        idx = oracle.build_indices(cfg, q, k)
        rows = np.array([(bh * w.seq_len + i) for bh in range(w.batch * w.n_q_heads)
                         for i in range(S)])
        out, _ = oracle.attention(cfg, q, k, v, idx, rows=rows)
        np.testing.assert_allclose(out, ref[:, :, :S].reshape(-1, w.head_dim).numpy(), rtol=0,
                                   atol=1e-10)


def test_threshold_is_inclusive():
    """The stop keeps a block whose normalised score equals τ (p ≥ τ; "stops once a block's score
    falls under τ", S2O card, Summary ¶2). Closed form: with every key the same vector, the key
    scores tie and the stable ordering is the identity, so with S = 2B the first segment's keys
    fill key blocks 0 and 1. A query block of the second segment then has exactly two candidate
    blocks, each with B visible keys and the same centroid, so each has p = 1/2 exactly, whatever
    the queries. At τ = 1/2 both are selected (ties by lower block id); at the next float above
    1/2, none; query blocks of the first segment have no candidates."""
    Bk, S, N, d = 4, 8, 16, 4
    rng = np.random.default_rng(5)
    q = torch.from_numpy(rng.standard_normal((1, 1, N, d), dtype=np.float32)).to(torch.bfloat16)
    k = torch.tensor([1.0, -0.5, 0.25, 2.0]).repeat(1, 1, N, 1).to(torch.bfloat16)
    c = dict(batch=1, n_q_heads=1, n_kv_heads=1, seq_len=N, head_dim=d, segment_len=S,
             block_size=Bk)
    idx = oracle.build_indices(_cfg(c, 0.5), q, k, debug=True)
    np.testing.assert_array_equal(idx["perm_k"][0, 0], np.arange(N))
    np.testing.assert_array_equal(idx["p"][0, 0, 2:], [[0.5, 0.5, 0.0, 0.0]] * 2)
    np.testing.assert_array_equal(idx["sel_cnt"][0, 0], [0, 0, 2, 2])
    np.testing.assert_array_equal(idx["sel_blk"][0, 0, 2:, :2], [[0, 1], [0, 1]])
    above = float(np.nextafter(np.float32(0.5), np.float32(1.0)))
    idx = oracle.build_indices(_cfg(c, above), q, k)
    np.testing.assert_array_equal(idx["sel_cnt"][0, 0], [0, 0, 0, 0])


# ----------------------------------------------------------------------------- invariants

def test_selection_nested_in_tau_and_sparsity_monotone():
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    taus = [0.0, 0.001, 0.01, 0.02, 0.05, 0.1, 0.3, 1.0, 1.5]
    prev_sets, prev_pairs = None, None
    for tau in taus:
        cfg = oracle.config(w, tau=tau)
        idx = oracle.build_indices(cfg, q, k)
        sets = [set(idx["sel_blk"][b, h, x, :idx["sel_cnt"][b, h, x]].tolist())
                for b in range(w.batch) for h in range(w.n_q_heads)
                for x in range(w.seq_len // w.block_size)]
        pairs = oracle.pair_count(cfg, idx)
        if prev_sets is not None:
            assert all(s <= p for s, p in zip(sets, prev_sets))
            assert pairs <= prev_pairs
        prev_sets, prev_pairs = sets, pairs


def test_probabilities_and_selection_rule():
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    cfg = oracle.config(w)
    idx = oracle.build_indices(cfg, q, k, debug=True)
    S, Bk, nB = w.segment_len, w.block_size, w.seq_len // w.block_size
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            for x in range(nB):
                s = x * Bk // S
                cand = idx["n"][b, h, s] > 0
                p = idx["p"][b, h, x]
                cnt = idx["sel_cnt"][b, h, x]
                if s == 0:
                    assert not cand.any() and cnt == 0
                    continue
                assert abs(p[cand].sum() - 1.0) < 1e-12
                assert (p[~cand] == 0).all()
                chosen = np.nonzero(cand & (p >= np.float64(np.float32(w.tau))))[0]
                order = sorted(chosen, key=lambda c: (-p[c], c))
                np.testing.assert_array_equal(idx["sel_blk"][b, h, x, :cnt], order)


def test_index_arrays_are_sorted_permutations():
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(oracle.config(w), q, k, debug=True)
    N, S, Bk = w.seq_len, w.segment_len, w.block_size
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            pk, pq = idx["perm_k"][b, h], idx["perm_q"][b, h]
            assert sorted(pk.tolist()) == list(range(N))
            ks = idx["kappa"][b, h][pk]
            assert (np.diff(ks) <= 0).all()
            ties = np.nonzero(np.diff(ks) == 0)[0]
            assert (pk[ties] < pk[ties + 1]).all()
            for s0 in range(0, N, S):
                seg = pq[s0:s0 + S]
                assert sorted(seg.tolist()) == list(range(s0, s0 + S))
                rs = idx["rho"][b, h][seg]
                assert (np.diff(rs) <= 0).all()
                t = np.nonzero(np.diff(rs) == 0)[0]
                assert (seg[t] < seg[t + 1]).all()
            for x in range(N // Bk):
                s0 = (x * Bk // S) * S
                assert idx["local_tiles"][b, h, x] == (pq[x * Bk:(x + 1) * Bk].max() - s0) // Bk + 1


def test_query_perm_off_is_identity_and_triangle():
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(oracle.config(w, query_perm=0), q, k)
    N, S, Bk = w.seq_len, w.segment_len, w.block_size
    np.testing.assert_array_equal(idx["perm_q"], np.broadcast_to(np.arange(N), idx["perm_q"].shape))
    x = np.arange(N // Bk)
    np.testing.assert_array_equal(idx["local_tiles"][0, 0], x - (x * Bk // S) * (S // Bk) + 1)


def test_float64_rederivation_of_pooled_quantities():
    """Every pooled quantity against an independent float64 numpy computation (GQA mapping,
    operand order, signs and the 1/sqrt(d) scale); n and local tiles exactly."""
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(oracle.config(w), q, k, debug=True)
    Q, K = q.double().numpy(), k.double().numpy()
    G, N, S, Bk, d = w.n_q_heads // w.n_kv_heads, w.seq_len, w.segment_len, w.block_size, w.head_dim
    nB = N // Bk
    tol = dict(rtol=1e-5, atol=1e-5)
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            Kg = K[b, h // G]
            qbar = Q[b, h].mean(0)
            np.testing.assert_allclose(idx["qbar"][b, h], qbar, **tol)
            np.testing.assert_allclose(idx["kbar_all"][b, h // G], Kg.mean(0), **tol)
            np.testing.assert_allclose(idx["kappa"][b, h], Kg @ qbar, **tol)
            pk, pq = idx["perm_k"][b, h], idx["perm_q"][b, h]
            u = Kg[pk[:Bk]].mean(0) - Kg.mean(0)
            np.testing.assert_allclose(idx["u"][b, h], u, **tol)
            np.testing.assert_allclose(idx["rho"][b, h], Q[b, h] @ u, **tol)
            Qbar = Q[b, h][pq].reshape(nB, Bk, d).mean(1)
            Kbar = Kg[pk].reshape(nB, Bk, d).mean(1)
            np.testing.assert_allclose(idx["Qbar"][b, h], Qbar, **tol)
            np.testing.assert_allclose(idx["Kbar"][b, h], Kbar, **tol)
            np.testing.assert_allclose(idx["r"][b, h], Qbar @ Kbar.T / math.sqrt(d), **tol)
            seg_of_key = pk.reshape(nB, Bk) // S
            n = np.stack([(seg_of_key < s).sum(1) for s in range(N // S)])
            np.testing.assert_array_equal(idx["n"][b, h], n)


def test_shared_key_order_variant():
    """The labelled variant with one key ordering per KV head: the group's kappa is the float64
    product of K_g with the mean of the group's mean queries; every query head of a group carries
    that ordering (a sorted permutation of kappa, ties to the lower index) and reads its k̄_top and
    K̄ from it; it differs from the per-head ordering when G > 1, and equals it when G = 1."""
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(oracle.config(w, shared_key_order=1), q, k, debug=True)
    base = oracle.build_indices(oracle.config(w), q, k)
    Q, K = q.double().numpy(), k.double().numpy()
    G, N, Bk, d = w.n_q_heads // w.n_kv_heads, w.seq_len, w.block_size, w.head_dim
    nB = N // Bk
    tol = dict(rtol=1e-5, atol=1e-5)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            heads = range(g * G, (g + 1) * G)
            qg = np.mean([Q[b, h].mean(0) for h in heads], axis=0)
            Kg = K[b, g]
            pk = idx["perm_k"][b, g * G]
            assert sorted(pk.tolist()) == list(range(N))
            for h in heads:
                np.testing.assert_allclose(idx["kappa"][b, h], Kg @ qg, **tol)
                np.testing.assert_array_equal(idx["perm_k"][b, h], pk)
                u = Kg[pk[:Bk]].mean(0) - Kg.mean(0)
                np.testing.assert_allclose(idx["u"][b, h], u, **tol)
                np.testing.assert_allclose(idx["Kbar"][b, h],
                                           Kg[pk].reshape(nB, Bk, d).mean(1), **tol)
            ks = idx["kappa"][b, g * G][pk]
            assert (np.diff(ks) <= 0).all()
            ties = np.nonzero(np.diff(ks) == 0)[0]
            assert (pk[ties] < pk[ties + 1]).all()
    assert not np.array_equal(idx["perm_k"], base["perm_k"])
    w1 = SMALL_GQA.replace(name="small-mha", n_q_heads=2, n_kv_heads=2)
    q1, k1, _ = gen.make_inputs(w1)
    a = oracle.build_indices(oracle.config(w1, shared_key_order=1), q1, k1)
    c = oracle.build_indices(oracle.config(w1), q1, k1)
    for name in ("perm_q", "perm_k", "sel_cnt", "sel_blk", "local_tiles"):
        np.testing.assert_array_equal(a[name], c[name], err_msg=name)


def test_int4_centroid_variant():
    """The labelled variant with 4-bit key centroids: its block scores against the exact float64
    centroid product without the per-block constant (σ·Q̄_b·(K̄_c − lo)), within the quantisation
    error bound (half a key step per channel, half a query step per code); everything before the
    scores is the default's, and at τ = 0 both select every candidate."""
    w = SMALL_GQA
    q, k, _ = gen.make_inputs(w)
    v = oracle.build_indices(oracle.config(w, int4_centroids=1), q, k, debug=True)
    base = oracle.build_indices(oracle.config(w), q, k, debug=True)
    for name in ("perm_q", "perm_k", "local_tiles"):
        np.testing.assert_array_equal(v[name], base[name], err_msg=name)
    np.testing.assert_array_equal(v["Qbar"], base["Qbar"])
    np.testing.assert_array_equal(v["Kbar"], base["Kbar"])
    d = w.head_dim
    sigma = 1.0 / math.sqrt(d)
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            Qb = v["Qbar"][b, h].astype(np.float64)
            Kb = v["Kbar"][b, h].astype(np.float64)
            lo = Kb.min(0)
            step = (Kb.max(0) - lo) / 15.0
            step[step == 0] = 1.0
            exact = sigma * (Qb @ (Kb - lo).T)
            sq = np.abs(Qb * step).max(1) / 127.0
            bound = sigma * (np.abs(Qb) @ (step / 2.0) + 15.0 * d * sq / 2.0)
            err = np.abs(v["r"][b, h].astype(np.float64) - exact)
            assert (err <= bound[:, None] * 1.01 + 1e-6).all(), float((err - bound[:, None]).max())
            # The bound is not vacuous: the scores carry the centroid signal.
            assert np.corrcoef(v["r"][b, h].ravel(), exact.ravel())[0, 1] > 0.9
    v0 = oracle.build_indices(oracle.config(w, tau=0.0, int4_centroids=1), q, k)
    b0 = oracle.build_indices(oracle.config(w, tau=0.0), q, k)
    np.testing.assert_array_equal(v0["sel_cnt"], b0["sel_cnt"])
    np.testing.assert_array_equal(np.sort(v0["sel_blk"], axis=-1), np.sort(b0["sel_blk"], axis=-1))


def test_int4_scores_exact_on_grid_aligned_centroids():
    """Closed form of the 4-bit centroid variant: when every key centroid already lies on the
    variant's 16-level grid and the scaled query maps to one code, the integer product gives the
    exact centroid score σ·Q̄·(K̄ − lo)ᵀ up to float32 rounding. Keys come in 16 groups of B equal
    rows (j/16)·e₀ and every query is e₀, so κ_j is the key's first element, each key block of the
    ordering is one group, the centroids' first channel takes the values j/16 (lo = 0, step
    (15/16)/15 = 1/16 exactly, codes j), the other channels are zero (code 0), and the query's one
    non-zero scaled value takes the code 127."""
    Bk, nB, d = 4, 16, 4
    N = Bk * nB
    k = np.zeros((N, d), np.float32)
    for j in range(nB):
        k[j * Bk:(j + 1) * Bk, 0] = j / 16
    q = np.zeros((N, d), np.float32)
    q[:, 0] = 1.0
    qt, kt = (torch.from_numpy(a).to(torch.bfloat16).reshape(1, 1, N, d) for a in (q, k))
    cfg = oracle.Config(1, 1, 1, N, d, 16, Bk, 0.01, 1, 0, 1)
    idx = oracle.build_indices(cfg, qt, kt, debug=True)
    Kbar, Qbar = idx["Kbar"][0, 0].astype(np.float64), idx["Qbar"][0, 0].astype(np.float64)
    np.testing.assert_array_equal(Kbar[:, 0], (15 - np.arange(nB)) / 16)
    np.testing.assert_array_equal(Kbar[:, 1:], 0.0)
    np.testing.assert_array_equal(Qbar, np.tile([1.0, 0, 0, 0], (nB, 1)))
    exact = 0.5 * Qbar[:, :1] @ Kbar[:, :1].T  # σ = 1/√4, lo = 0
    np.testing.assert_allclose(idx["r"][0, 0], exact, rtol=1e-6, atol=0)


# ----------------------------------------------------------------------------- summation orders

SUM_ORDER = os.path.join(os.path.dirname(__file__), "golden", "sum_order_case.json")


def _sum_order_case():
    """Inputs of the hand-derived summation-order case, built from the rules in its JSON."""
    with open(SUM_ORDER) as f:
        g = json.load(f)
    c, inp = g["config"], g["inputs"]
    N, d = c["seq_len"], c["head_dim"]
    q = np.zeros((N, d), np.float32)
    q[:N // 2] = inp["q_segment0_row"]
    q[N // 2:] = inp["q_segment1_row"]
    for i, val in inp["q_channel2_overrides"].items():
        q[int(i), 2] = val
    k = np.zeros((N, d), np.float32)
    half = N // 2
    for j in range(half):
        v0 = inp["k_channel0"]["key0_and_key64"] if j == 0 else inp["k_channel0"]["other_keys"]
        k[j, 0] = k[half + j, 0] = v0
        k[j, 1] = k[half + j, 1] = 63 - j
    for j, val in inp["k_channel3_overrides"].items():
        k[int(j), 3] = val
    to_bf16 = lambda a: torch.from_numpy(a).to(torch.bfloat16).reshape(1, 1, N, d)  # noqa: E731
    qt, kt = to_bf16(q), to_bf16(k)
    # Every input value is exact in bf16.
    assert torch.equal(qt.float().reshape(N, d), torch.from_numpy(q))
    assert torch.equal(kt.float().reshape(N, d), torch.from_numpy(k))
    cfg = oracle.Config(c["batch"], c["n_q_heads"], c["n_kv_heads"], N, d, c["segment_len"],
                        c["block_size"], c["tau"], 1)
    return g, cfg, qt, kt


def test_sum_order_case_chunked_means():
    """D1's SUM: chunks of B list entries, then the chunk sums in order (hand-derived bits)."""
    g, cfg, q, k = _sum_order_case()
    idx = oracle.build_indices(cfg, q, k, debug=True)
    e = g["expected"]
    np.testing.assert_array_equal(idx["qbar"][0, 0],
                                  np.array([float.fromhex(x) for x in e["qbar"]], np.float32))
    assert idx["kbar_all"][0, 0, 0] == np.float32(float.fromhex(e["kbar_all_channel0"]))
    assert idx["kbar_all"][0, 0, 3] == np.float32(float.fromhex(e["kbar_all_channel3"]))
    half = cfg.seq_len // 2
    want_perm = np.stack([np.arange(half), np.arange(half) + half], axis=1).reshape(-1)
    np.testing.assert_array_equal(idx["perm_k"][0, 0], want_perm)


def test_sum_order_case_normaliser_chunks():
    """D7's Z: chunks of 32 consecutive blocks, then the chunk sums in order (hand-derived bits
    of p for the one block that carries almost all the weight)."""
    g, cfg, q, k = _sum_order_case()
    idx = oracle.build_indices(cfg, q, k, debug=True)
    e = g["expected"]
    nB = cfg.seq_len // cfg.block_size
    first = (cfg.seq_len // cfg.segment_len - 1) * (cfg.segment_len // cfg.block_size)
    r = idx["r"][0, 0]
    assert (r[first:, 0] == np.float32(float.fromhex(e["r_block0"]))).all()
    assert (r[first:, 1:] == np.float32(float.fromhex(e["r_other_blocks"]))).all()
    p0 = idx["p"][0, 0, first:, 0]
    assert (p0 == float.fromhex(e["p_block0_for_segment1_query_blocks"])).all(), p0[:4]
    assert (idx["sel_cnt"][0, 0, first:] == e["sel_cnt_segment1"]).all()
    assert (idx["sel_blk"][0, 0, first:, 0] == e["sel_blk0_segment1"]).all()
    assert (idx["sel_cnt"][0, 0, :first] == 0).all()
    assert nB > 32  # the normaliser spans more than one 32-block chunk


# ----------------------------------------------------------------------------- online early stop

def test_online_stop_hand_case():
    """The measured-share stop on the hand case with τ = 0.4 and given lists (closed forms derived
    by hand in tests/golden/online_stop_case.md)."""
    g, c, q, k, _ = _hand()
    cfg = _cfg(c, 0.4)
    idx = oracle.build_indices(cfg, q, k)
    lists = {3: [1, 2, 0], 2: [2, 0, 1]}
    sel_cnt = np.zeros((1, 1, 4), np.int32)
    sel_blk = np.full((1, 1, 4, 4), -1, np.int32)
    for b, lst in lists.items():
        sel_cnt[0, 0, b] = len(lst)
        sel_blk[0, 0, b, :len(lst)] = lst
    idx = dict(idx, sel_cnt=sel_cnt, sel_blk=sel_blk)
    stop, share = oracle.online_stop(cfg, q, k, idx)
    e, r = math.e, math.exp(0.5)
    want3 = [0.5, 2 / (2 * r + 2), e / (2 * r + 2 + e)]
    want2 = [(r + 1) / (e + 4 + r), e * e / (e + 4 + e * e), e / (2 * e + 4 + e * e)]
    np.testing.assert_allclose(share[0, 0, 3, :3], want3, rtol=1e-14)
    np.testing.assert_allclose(share[0, 0, 2, :3], want2, rtol=1e-14)
    np.testing.assert_array_equal(stop[0, 0], [0, 0, 1, 2])


def test_online_stop_tau_zero_keeps_every_list():
    w = SMALL_GQA.replace(tau=0.0)
    cfg = oracle.config(w)
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(cfg, q, k)
    stop, _ = oracle.online_stop(cfg, q, k, idx)
    np.testing.assert_array_equal(stop, idx["sel_cnt"])


STOP_CASE = gen.Workload("online-stop", batch=1, n_q_heads=2, n_kv_heads=1, seq_len=2048,
                         head_dim=64, segment_len=256, block_size=64, tau=0.0, seed=13, amp=4.0,
                         stripe_count=60, diag=0.5)


@pytest.mark.parametrize("tau", [0.005, 0.03, 0.08])
def test_online_stop_against_softmax_probabilities(tau):
    """Brute force from another formulation: each row's softmax probabilities over its whole list
    key set (torch, float64); a block's share is its probability mass over the mass of the keys up
    to and including it. Lists: every candidate block (built at τ = 0), so that later blocks carry
    little mass and the stop at τ cuts them. The stop keeps lists as prefixes and never lengthens
    them."""
    w = STOP_CASE
    q, k, _ = gen.make_inputs(w)
    idx = oracle.build_indices(oracle.config(w), q, k)
    cfg = oracle.config(w, tau=tau)
    stop, share = oracle.online_stop(cfg, q, k, idx)
    assert (stop <= idx["sel_cnt"]).all() and ((stop > 0) == (idx["sel_cnt"] > 0)).all()
    N, B, S, d = w.seq_len, w.block_size, w.segment_len, w.head_dim
    G = w.n_q_heads // w.n_kv_heads
    nB = N // B
    qf, kf = q.double(), k.double()
    stopped_somewhere = False
    for beta in range(w.batch):
        for h in range(w.n_q_heads):
            g = h // G
            for b in range(nB):
                cnt = idx["sel_cnt"][beta, h, b]
                if cnt == 0:
                    continue
                s0 = (b * B // S) * S
                lst = idx["sel_blk"][beta, h, b, :cnt]
                pk = idx["perm_k"][beta, h]
                vis = [[j for j in pk[c * B:(c + 1) * B] if j < s0] for c in lst]
                best = np.zeros(cnt)
                for i in idx["perm_q"][beta, h, b * B:(b + 1) * B]:
                    keys = list(range(s0, i + 1)) + [j for v in vis for j in v]
                    z = (qf[beta, h, i] @ kf[beta, g, keys].T) / math.sqrt(d)
                    prob = torch.softmax(z, dim=0).numpy()
                    mass = dict(zip(keys, prob))
                    run = sum(mass[j] for j in range(s0, i + 1))
                    for x, v in enumerate(vis):
                        blk = sum(mass[j] for j in v)
                        run += blk
                        best[x] = max(best[x], blk / run)
                np.testing.assert_allclose(share[beta, h, b, :cnt], best, rtol=1e-9, atol=1e-15)
                below = np.nonzero(best < tau)[0]
                want = int(below[0]) + 1 if len(below) else int(cnt)
                assert stop[beta, h, b] == want
                stopped_somewhere |= want < cnt
    if tau >= 0.03:
        assert stopped_somewhere  # the case exercises an actual stop

"""The seeded input generator (`gen/`) follows its stated recipe (the definition's synthetic-input
section): N(0, 1) slabs from per-(tensor, batch, head) PCG64 streams, planted stripes of
amplitude A along a unit direction per KV head, the query shift along that direction, the literal
diagonal q_i += diag·k_i with the final K, and bf16 round-to-nearest-even. Each property is
re-derived here from numpy's streams and torch's own bf16 conversion, not from gen's helpers; the
bytes must not depend on the number of threads that draw them."""
import numpy as np
import torch

import gen

SMALL = gen.Workload("gen-small", batch=2, n_q_heads=4, n_kv_heads=2, seq_len=512, head_dim=64,
                     segment_len=128, block_size=64, tau=0.01, seed=21, amp=4.0,
                     stripe_frac=0.02, q_shift=1.5, diag=0.5)


def stream(seed, *key):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def bits(t):
    return t.contiguous().view(torch.int16).numpy()


def test_bytes_independent_of_thread_count():
    a = gen.make_inputs(SMALL, threads=1)
    b = gen.make_inputs(SMALL, threads=5)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_recipe_rederived_from_the_streams():
    w = SMALL
    q, k, v, (qf, kf, vf) = gen.make_inputs(w, keep_fp32=True)
    N, d, G = w.seq_len, w.head_dim, w.n_q_heads // w.n_kv_heads
    n_stripe = int(round(w.stripe_frac * N))
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            base = stream(w.seed, 1, b, g).standard_normal((N, d), dtype=np.float32)
            rng = stream(w.seed, 3, b, g)
            ug = rng.standard_normal(d)
            u = (ug / np.linalg.norm(ug)).astype(np.float32)
            pos = rng.choice(N, size=n_stripe, replace=False)
            assert abs(float(np.linalg.norm(u.astype(np.float64))) - 1.0) < 1e-6
            # Stripes: exactly the drawn positions moved, each by A·u (float32 addition).
            moved = np.nonzero((kf[b, g] != base).any(axis=1))[0]
            assert set(moved.tolist()) <= set(pos.tolist()) and len(pos) == n_stripe
            want_k = base.copy()
            want_k[pos] += np.float32(w.amp) * u
            np.testing.assert_array_equal(kf[b, g], want_k)
            np.testing.assert_array_equal(
                vf[b, g], stream(w.seed, 2, b, g).standard_normal((N, d), dtype=np.float32))
            for h in range(g * G, (g + 1) * G):
                qbase = stream(w.seed, 0, b, h).standard_normal((N, d), dtype=np.float32)
                want_q = qbase + np.float32(w.q_shift) * u
                want_q += np.float32(w.diag) * want_k  # the literal diagonal, final K
                np.testing.assert_array_equal(qf[b, h], want_q)
    # bf16 rounding: torch's float32 -> bf16 conversion (round to nearest even).
    for t, f in ((q, qf), (k, kf), (v, vf)):
        np.testing.assert_array_equal(bits(t), bits(torch.from_numpy(f).to(torch.bfloat16)))


def test_rounding_ties_go_to_even():
    """Values exactly halfway between two bf16 numbers round to the one with an even last bit."""
    lo = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    want = torch.from_numpy(lo).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(want, [1.0, 1.0 + 2.0 ** -6, -1.0])
    # gen's own conversion of the same values.
    got = torch.from_numpy(gen._to_bf16_bits(lo.copy()).view(np.int16)).view(torch.bfloat16)
    np.testing.assert_array_equal(got.float().numpy(), want)


def test_specified_workloads():
    """The stand-in shapes: 32 query / 8 KV heads, d = 128; 1 % stripe keys at amplitude 4; the
    tiny case with 8 stripe keys at amplitude 3 and no diagonal."""
    t = gen.workload("tiny")
    assert (t.seq_len, t.head_dim, t.segment_len, t.block_size) == (1024, 64, 256, 64)
    assert (t.stripe_count, t.amp, t.diag, t.seed) == (8, 3.0, 0.0, 0)
    for name, n in (("llama-32k", 32768), ("llama-128k", 131072), ("qwen-128k", 131072)):
        w = gen.workload(name)
        assert (w.n_q_heads, w.n_kv_heads, w.head_dim, w.seq_len) == (32, 8, 128, n)
        assert (w.segment_len, w.block_size, w.tau, w.amp, w.diag) == (2048, 128, 0.01, 4.0, 0.5)
        assert int(round(w.stripe_frac * w.seq_len)) == {32768: 328, 131072: 1311}[n]
    stack = [gen.layer_workload(l) for l in (0, 31)]
    assert stack[0].stripe_frac == 0.005 and abs(stack[1].stripe_frac - 0.03) < 1e-15
    assert [s.seed for s in stack] == [1000, 1031]

"""Seeded synthetic Q/K/V for the S2O prefill path.

This module is the only code shared by the CPU oracle's tests and the CUDA path's tests and
benchmark: it produces input bytes and nothing else (none of the method's arithmetic lives here).

The pages evaluate on Llama-3.1-8B / Qwen3-8B activations over long-context datasets that are not
available; these inputs stand in for them with the same attention shapes (32 query heads, 8 KV
heads, d = 128) and with the stripe patterns the S2O card's Summary says real attention maps are
made of (vertical stripes on a few key positions, a diagonal).

Recipe (each (tensor, batch, head) slab has its own numpy stream, so the bytes do not depend on
how many threads draw them):

1. Q, K, V ~ N(0, 1) float32; slab (t, beta, head) drawn from
   ``Generator(PCG64(SeedSequence(seed, spawn_key=(t, beta, head))))`` with t = 0, 1, 2 for Q, K, V.
2. For each (beta, g): from ``SeedSequence(seed, spawn_key=(3, beta, g))`` draw a direction
   u_g ~ N(0, I_d) (float64, then normalised) and ``round(stripe_frac * N)`` distinct key positions
   (or ``stripe_count`` when given); those keys get ``+ amp * u_g`` and every query of the heads of
   group g gets ``+ q_shift * u_g``.
3. If ``diag`` is non-zero: ``q[h, i] += diag * k[g(h), i]`` using the final K (the literal
   diagonal reading of "diagonal band for local window 512").
4. Round to bf16, nearest-even.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "workload", "LayerShape", "LAYER_8B", "make_layer"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    seq_len: int
    head_dim: int
    segment_len: int
    block_size: int
    tau: float
    seed: int
    amp: float = 4.0
    stripe_frac: float = 0.01
    stripe_count: int | None = None
    q_shift: float = 1.0
    diag: float = 0.5
    query_perm: int = 1
    shared_key_order: int = 0
    int4_centroids: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def dense_causal_flops(self) -> float:
        """4·d·N(N+1)/2 per query head: QKᵀ and PV over the causal triangle."""
        n = self.seq_len
        return 4.0 * self.head_dim * n * (n + 1) / 2 * self.n_q_heads * self.batch


WORKLOADS = {
    # 1 head, d = 64, N = 1024; 8 planted stripe keys at amplitude 3, all queries +1·u.
    "tiny": Workload("tiny", 1, 1, 1, 1024, 64, 256, 64, 0.01, 0, amp=3.0,
                     stripe_count=8, diag=0.0),
    "llama-32k": Workload("llama-32k", 1, 32, 8, 32768, 128, 2048, 128, 0.01, 1),
    "llama-128k": Workload("llama-128k", 1, 32, 8, 131072, 128, 2048, 128, 0.01, 2),
    "qwen-128k": Workload("qwen-128k", 1, 32, 8, 131072, 128, 2048, 128, 0.01, 3),
    # Labelled extra workload beside the specified ones: the llama-128k shape with strong stripes
    # (5 % of the keys, amplitude 16, queries shifted by 4·u), so that at τ = 0.01 the method
    # selects dozens of permuted blocks per query block and pair sparsity lands in the range the
    # S2O card reports for real 128K prefill (≈ 0.94 here; 0.933 on the card's Key points).
    "llama-128k-strong": Workload("llama-128k-strong", 1, 32, 8, 131072, 128, 2048, 128, 0.01,
                                  4, amp=16.0, stripe_frac=0.05, q_shift=4.0),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def layer_workload(layer: int) -> Workload:
    """Layer l of the 32-layer stack: stripe density 0.5 % + 2.5 %·l/31, seed 1000 + l."""
    frac = 0.005 + 0.025 * layer / 31.0
    return WORKLOADS["llama-128k"].replace(name=f"stack-layer{layer}", stripe_frac=frac,
                                           seed=1000 + layer)


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=key)))


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (inputs are finite)."""
    b = x.view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) \
        .astype(np.uint16)


def make_inputs(w: Workload, threads: int | None = None, keep_fp32: bool = False):
    """Return ``(q, k, v)`` as contiguous CPU bf16 tensors in BHND layout.

    With ``keep_fp32`` also returns the float32 arrays before rounding (used by the tiny case's
    own Eq. 1 check).
    """
    B, Hq, Hkv, N, d = w.batch, w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim
    G = Hq // Hkv
    threads = threads or min(32, os.cpu_count() or 1)
    n_stripe = w.stripe_count if w.stripe_count is not None else int(round(w.stripe_frac * N))
    kf = np.empty((B, Hkv, N, d), np.float32)
    qb = np.empty((B, Hq, N, d), np.uint16)
    kb = np.empty((B, Hkv, N, d), np.uint16)
    vb = np.empty((B, Hkv, N, d), np.uint16)
    qf = np.empty((B, Hq, N, d), np.float32) if keep_fp32 else None
    vf = np.empty((B, Hkv, N, d), np.float32) if keep_fp32 else None
    u = np.empty((B, Hkv, d), np.float32)

    def kv_job(job):
        b, g = job
        _stream(w.seed, 1, b, g).standard_normal(out=kf[b, g], dtype=np.float32)
        rng = _stream(w.seed, 3, b, g)
        ug = rng.standard_normal(d)
        u[b, g] = (ug / np.linalg.norm(ug)).astype(np.float32)
        pos = rng.choice(N, size=n_stripe, replace=False)
        kf[b, g, pos, :] += np.float32(w.amp) * u[b, g]
        kb[b, g] = _to_bf16_bits(kf[b, g])
        vslab = np.empty((N, d), np.float32) if vf is None else vf[b, g]
        _stream(w.seed, 2, b, g).standard_normal(out=vslab, dtype=np.float32)
        vb[b, g] = _to_bf16_bits(vslab)

    def q_job(job):
        b, h = job
        g = h // G
        slab = np.empty((N, d), np.float32) if qf is None else qf[b, h]
        _stream(w.seed, 0, b, h).standard_normal(out=slab, dtype=np.float32)
        slab += np.float32(w.q_shift) * u[b, g]
        if w.diag:
            slab += np.float32(w.diag) * kf[b, g]
        qb[b, h] = _to_bf16_bits(slab)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(kv_job, [(b, g) for b in range(B) for g in range(Hkv)]))
        list(ex.map(q_job, [(b, h) for b in range(B) for h in range(Hq)]))

    out = tuple(torch.from_numpy(x).view(torch.bfloat16) for x in (qb, kb, vb))
    if keep_fp32:
        return out + ((qf, kf, vf),)
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU bf16 tensor as a uint16 numpy array (no copy)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ decoder layer (random weights)

@dataclasses.dataclass(frozen=True)
class LayerShape:
    """The non-attention sizes of a Llama-3.1-8B-shaped decoder layer (the attention shape comes
    from the Workload: hidden = n_q_heads · head_dim)."""
    intermediate: int = 14336
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0
    rope_factor: float = 8.0
    rope_low_freq_factor: float = 1.0
    rope_high_freq_factor: float = 4.0
    rope_original_context: int = 8192

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


LAYER_8B = LayerShape()


def make_layer(w: Workload, shape: LayerShape = LAYER_8B, seed: int | None = None,
               threads: int | None = None) -> dict:
    """Random weights and input rows of one decoder layer, as CPU bf16 tensors.

    x [batch, N, H] ~ N(0, 1); each projection W [fan_in, fan_out] ~ N(0, 1/fan_in); norm gains
    ~ N(1, 0.1²). Every tensor is drawn in 1024-row chunks, chunk c of tensor t from
    ``SeedSequence(seed, spawn_key=(100 + t, c))`` (seed defaults to the workload's), then rounded
    to bf16 (nearest-even).
    """
    seed = w.seed if seed is None else seed
    threads = threads or min(32, os.cpu_count() or 1)
    H = w.n_q_heads * w.head_dim
    qkv = (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim
    I = shape.intermediate
    specs = [  # name, shape (rows, cols), mean, std
        ("x", (w.batch * w.seq_len, H), 0.0, 1.0),
        ("attn_norm", (1, H), 1.0, 0.1),
        ("w_qkv", (H, qkv), 0.0, H ** -0.5),
        ("w_o", (H, H), 0.0, H ** -0.5),
        ("mlp_norm", (1, H), 1.0, 0.1),
        ("w_gu", (H, 2 * I), 0.0, H ** -0.5),
        ("w_down", (I, H), 0.0, I ** -0.5),
    ]
    out = {}
    jobs = []
    for t, (name, (rows, cols), mean, std) in enumerate(specs):
        bits = np.empty((rows, cols), np.uint16)
        out[name] = bits
        for c, r0 in enumerate(range(0, rows, 1024)):
            jobs.append((t, c, bits, r0, min(rows, r0 + 1024), cols, mean, std))

    def job(j):
        t, c, bits, r0, r1, cols, mean, std = j
        x = _stream(seed, 100 + t, c).standard_normal((r1 - r0, cols), dtype=np.float32)
        x *= np.float32(std)
        x += np.float32(mean)
        bits[r0:r1] = _to_bf16_bits(x)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(job, jobs))
    res = {k: torch.from_numpy(v).view(torch.bfloat16) for k, v in out.items()}
    res["x"] = res["x"].reshape(w.batch, w.seq_len, H)
    res["attn_norm"] = res["attn_norm"].reshape(H)
    res["mlp_norm"] = res["mlp_norm"].reshape(H)
    return res

"""CPU oracle of the decoder layer around the S2O attention — TEST INFRASTRUCTURE, not part of
the product (only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import it).

Written from the project definition's decoder-layer section, itself the public Llama-3 decoder
layer (pre-norm residual blocks, grouped-query attention with rotary position embedding and the
Llama 3.1 frequency scaling, SwiGLU MLP); the pages only name the model ("S2O: Early Stopping
for Sparse Attention via Online Permutation", Key points: Llama-3.1-8B, end-to-end speedup at
128K). Everything is binary64 (numpy), rounded to bf16 at the points where the GPU stores bf16;
the attention is this package's oracle (``attention`` / ``dense_causal``) on the bf16 q, k, v.

Parity pins (``tests/test_layer_oracle_pins.py``): RMS norm of constant rows, the rotation's
norm preservation, identity at position 0 and relative-position property, the frequency table
against the scaling's three regimes and against transformers' "llama3" rotary table, silu at
known points, bf16 rounding against torch, the whole layer with zero projections (the residual
passes through unchanged), and the whole layer against transformers' Llama decoder layer in
float64 on the same weights (within a few bf16 ulps: the oracle rounds to bf16 where the GPU
stores bf16, the library does not). ``tests/test_layer_oracle_mutations.py`` checks that these
pins reject planted mistakes.
"""
from __future__ import annotations

import math

import numpy as np

from . import attention, build_indices, config, dense_causal


def bf16_round(x) -> np.ndarray:
    """Nearest bf16 value (ties to even) of binary64 values, as binary64; one rounding (no pass
    through float32). Finite normal-range inputs."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)  # x = m·2^e, 0.5 <= |m| < 1: a bf16 keeps 8 significant bits
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def bf16_value(t) -> np.ndarray:
    """A torch bf16 tensor (or uint16 bit patterns) as binary64 values."""
    if hasattr(t, "view") and not isinstance(t, np.ndarray):
        import torch
        t = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    b = np.ascontiguousarray(t, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 values (binary64 holding exact bf16 numbers) as uint16 bit patterns."""
    return (np.ascontiguousarray(x, np.float64).astype(np.float32).view(np.uint32)
            >> np.uint32(16)).astype(np.uint16)


def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """bf16(gain ⊙ x · (mean x² + eps)^(-1/2)) per row (last axis)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return bf16_round(gain * x * r)


def rope_frequencies(d: int, shape) -> np.ndarray:
    """f_t = θ^(-2t/d), t < d/2, with the Llama 3.1 scaling of long wavelengths."""
    t = np.arange(d // 2, dtype=np.float64)
    f = shape.rope_theta ** (-2.0 * t / d)
    if shape.rope_factor <= 0:
        return f
    orig, lo, hi, fac = (shape.rope_original_context, shape.rope_low_freq_factor,
                         shape.rope_high_freq_factor, shape.rope_factor)
    out = np.empty_like(f)
    for i, fi in enumerate(f):
        lam = 2.0 * math.pi / fi
        if lam < orig / hi:
            out[i] = fi
        elif lam > orig / lo:
            out[i] = fi / fac
        else:
            s = (orig / lam - lo) / (hi - lo)
            out[i] = (1.0 - s) * fi / fac + s * fi
    return out


def rope(y: np.ndarray, pos: np.ndarray, freqs: np.ndarray) -> np.ndarray:
    """Rotate pairs (y_t, y_{t+d/2}) of y [..., rows, heads, d] by the angle pos·f_t."""
    d = y.shape[-1]
    ang = pos[:, None].astype(np.float64) * freqs[None, :]  # [rows, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = y[..., : d // 2], y[..., d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def layer(w, shape, weights: dict, dense: bool = False, n_threads: int | None = None):
    """One decoder layer on x (``weights["x"]``): returns x₂ [batch, N, H] as binary64 holding
    bf16 values. ``w`` gives the attention configuration (heads, d, S, B, τ, ...); ``dense``
    replaces the S2O attention by dense causal attention."""
    B, N, Hq, Hkv, d = w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim
    H, I = Hq * d, shape.intermediate
    W = {k: bf16_value(v) for k, v in weights.items()}
    x = W["x"].reshape(B, N, H)
    # 1-2: norm and the q/k/v projection.
    h = rms_norm(x, W["attn_norm"], shape.rms_eps)
    qkv = bf16_round(h @ W["w_qkv"])
    q = qkv[..., : Hq * d].reshape(B, N, Hq, d)
    k = qkv[..., Hq * d: (Hq + Hkv) * d].reshape(B, N, Hkv, d)
    v = qkv[..., (Hq + Hkv) * d:].reshape(B, N, Hkv, d)
    # 3: rotary embedding at each row's position in its sequence.
    freqs = rope_frequencies(d, shape)
    pos = np.arange(N)
    q = bf16_round(np.stack([rope(q[b], pos, freqs) for b in range(B)]))
    k = bf16_round(np.stack([rope(k[b], pos, freqs) for b in range(B)]))
    # 4: attention on the head-major q, k, v.
    Q = np.ascontiguousarray(q.transpose(0, 2, 1, 3))
    K = np.ascontiguousarray(k.transpose(0, 2, 1, 3))
    V = np.ascontiguousarray(v.transpose(0, 2, 1, 3))
    cfg = config(w)
    qb, kb, vb = bf16_bits(Q), bf16_bits(K), bf16_bits(V)
    if dense:
        o = dense_causal(cfg, qb, kb, vb, n_threads=n_threads)
    else:
        idx = build_indices(cfg, qb, kb, n_threads=n_threads)
        o, _ = attention(cfg, qb, kb, vb, idx, n_threads=n_threads)
    O = bf16_round(o).reshape(B, Hq, N, d)
    o_rows = O.transpose(0, 2, 1, 3).reshape(B, N, H)
    # 5-9: output projection with the residual, then the MLP block.
    x1 = bf16_round(x + o_rows @ W["w_o"])
    h2 = rms_norm(x1, W["mlp_norm"], shape.rms_eps)
    gu = bf16_round(h2 @ W["w_gu"])
    a = bf16_round(silu(gu[..., :I]) * gu[..., I:])
    return bf16_round(x1 + a @ W["w_down"])

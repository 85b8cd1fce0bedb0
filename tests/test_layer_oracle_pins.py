"""Pins of the decoder-layer oracle (``oracle/layer.py``) to facts other than itself: bf16
rounding against torch's conversion, RMS norm on rows with a closed form, the rotary embedding's
identity at position 0, norm preservation and relative-position property, the frequency scaling's
regimes and continuity, the silu identity silu(z) − silu(−z) = z, the whole layer with zero
projections (the residual stream passes through unchanged), and, as a library the layer reduces
to, transformers' Llama decoder layer and its "llama3" rotary table run on the same weights
(test_layer_oracle_mutations.py plants mistakes in copies of the layer oracle and checks that
these pins reject each)."""
import math

import numpy as np
import pytest
import torch

import gen
from oracle import layer as L

SHAPE = gen.LAYER_8B


def test_bf16_round_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 7,
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 0.0, 3.0])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(L.bf16_round(x.astype(np.float64)), want)
    # exact ties go to the even neighbour
    assert L.bf16_round(1 + 2 ** -8) == 1.0
    assert L.bf16_round(1 + 3 * 2 ** -8) == 1 + 2 ** -6


def test_bits_round_trip():
    rng = np.random.default_rng(1)
    v = L.bf16_round(rng.standard_normal(5000))
    np.testing.assert_array_equal(L.bf16_value(L.bf16_bits(v)), v)


def test_rms_norm_closed_forms():
    # a constant row c·1 with unit gain normalises to c/sqrt(c² + eps)
    for c in (2.0, -0.5, 8.0):
        x = np.full((1, 64), c)
        got = L.rms_norm(x, np.ones(64), 1e-5)
        np.testing.assert_array_equal(got, L.bf16_round(np.full((1, 64), c / math.sqrt(c * c + 1e-5))))
    # (3, 4): mean square 12.5
    got = L.rms_norm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.0)
    r = 1 / math.sqrt(12.5)
    np.testing.assert_array_equal(got, L.bf16_round(np.array([[3 * r, 8 * r]])))


def test_rope_identity_norm_and_relative_position():
    rng = np.random.default_rng(2)
    d = 128
    f = L.rope_frequencies(d, SHAPE)
    y = rng.standard_normal((5, 3, d))
    np.testing.assert_allclose(L.rope(y, np.zeros(5, np.int64), f), y, rtol=0, atol=0)
    pos = np.array([0, 1, 77, 4096, 131071])
    r = L.rope(y, pos, f)
    pair = lambda a: a[..., : d // 2] ** 2 + a[..., d // 2:] ** 2  # noqa: E731
    np.testing.assert_allclose(pair(r), pair(y), rtol=1e-12)
    # <R(m) q, R(n) k> depends only on m - n
    q, k = rng.standard_normal((1, 1, d)), rng.standard_normal((1, 1, d))
    dot = lambda m, n: float(np.sum(L.rope(q, np.array([m]), f) * L.rope(k, np.array([n]), f)))  # noqa: E731
    for m, n, s in ((5, 2, 1000), (300, 17, 12345), (9, 9, 70000)):
        assert abs(dot(m, n) - dot(m + s, n + s)) < 1e-9 * (1 + abs(dot(m, n)))


def test_rope_frequency_scaling_regimes():
    d = 128
    base = SHAPE.rope_theta ** (-2.0 * np.arange(d // 2) / d)
    f = L.rope_frequencies(d, SHAPE)
    lam = 2 * math.pi / base
    hi = lam < SHAPE.rope_original_context / SHAPE.rope_high_freq_factor
    lo = lam > SHAPE.rope_original_context / SHAPE.rope_low_freq_factor
    assert hi.any() and lo.any() and (~hi & ~lo).any()
    np.testing.assert_array_equal(f[hi], base[hi])
    np.testing.assert_allclose(f[lo], base[lo] / SHAPE.rope_factor, rtol=1e-15)
    mid = ~hi & ~lo
    # between the two: strictly between base/8 and base, and continuous at both ends
    assert np.all(f[mid] < base[mid]) and np.all(f[mid] > base[mid] / SHAPE.rope_factor)
    no_scale = L.rope_frequencies(d, SHAPE.replace(rope_factor=0.0))
    np.testing.assert_array_equal(no_scale, base)
    for edge in (SHAPE.rope_original_context / SHAPE.rope_high_freq_factor,
                 SHAPE.rope_original_context / SHAPE.rope_low_freq_factor):
        fb = 2 * math.pi / edge
        probe = SHAPE.replace()
        # evaluate the mixed formula at the edge through a one-frequency table
        s = (probe.rope_original_context / edge - probe.rope_low_freq_factor) / (
            probe.rope_high_freq_factor - probe.rope_low_freq_factor)
        mixed = (1 - s) * fb / probe.rope_factor + s * fb
        assert abs(mixed - (fb if edge < 4096 else fb / probe.rope_factor)) < 1e-12 * fb


def test_silu_identity_and_limits():
    z = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(L.silu(z) - L.silu(-z), z, atol=1e-12)
    assert L.silu(np.array([0.0]))[0] == 0.0
    assert abs(L.silu(np.array([40.0]))[0] - 40.0) < 1e-12


def test_layer_with_zero_projections_is_identity():
    w = gen.Workload("layer-pin", 1, 2, 1, 256, 64, 128, 64, 0.01, 3)
    shape = SHAPE.replace(intermediate=128)
    wts = gen.make_layer(w, shape)
    for name in ("w_o", "w_down"):
        wts[name] = torch.zeros_like(wts[name])
    x2 = L.layer(w, shape, wts)
    np.testing.assert_array_equal(x2, L.bf16_value(wts["x"]).reshape(x2.shape))


def test_layer_s2o_at_tau_zero_matches_dense_attention():
    w = gen.Workload("layer-pin", 1, 2, 1, 256, 64, 128, 64, 0.0, 4)
    shape = SHAPE.replace(intermediate=128)
    wts = gen.make_layer(w, shape)
    a = L.layer(w, shape, wts)
    b = L.layer(w, shape, wts, dense=True)
    # the same key sets: differences only from the attention's summation order, below one ulp of
    # bf16 on all but a few elements
    assert np.mean(a != b) < 0.01
    assert np.max(np.abs(a - b)) <= 2 ** -6 * max(1.0, np.max(np.abs(a)))


def test_layer_inputs_are_seeded_and_thread_independent():
    w = gen.Workload("layer-pin", 1, 2, 1, 2048, 64, 128, 64, 0.01, 5)
    shape = SHAPE.replace(intermediate=256)
    a = gen.make_layer(w, shape, threads=1)
    b = gen.make_layer(w, shape, threads=7)
    c = gen.make_layer(w, shape, seed=6, threads=3)
    for name in a:
        assert torch.equal(a[name].view(torch.int16), b[name].view(torch.int16)), name
    assert not torch.equal(a["w_qkv"].view(torch.int16), c["w_qkv"].view(torch.int16))
    # projection scale N(0, 1/fan_in), norm gains around 1
    assert abs(float(a["w_gu"].float().std()) * math.sqrt(128) - 1) < 0.05
    assert abs(float(a["attn_norm"].float().mean()) - 1) < 0.05


# ----------------------------------------------------------------------------- against a library

def _hf_layer(w, shape, wts):
    """The same layer in transformers' own Llama implementation (float64, eager attention with a
    causal mask), with the random weights moved into its parameter layout (x·W here, x·Wᵀ
    there). Returns (output rows [N, H], the rotary table's inverse frequencies)."""
    tr = pytest.importorskip("transformers")
    from transformers.models.llama import modeling_llama as ml
    Hq, Hkv, d, N, I = w.n_q_heads, w.n_kv_heads, w.head_dim, w.seq_len, shape.intermediate
    H = Hq * d
    cfg = tr.LlamaConfig(
        hidden_size=H, num_attention_heads=Hq, num_key_value_heads=Hkv, head_dim=d,
        intermediate_size=I, rms_norm_eps=shape.rms_eps, max_position_embeddings=131072,
        rope_theta=shape.rope_theta, attention_bias=False, mlp_bias=False,
        rope_scaling={"rope_type": "llama3", "factor": shape.rope_factor,
                      "low_freq_factor": shape.rope_low_freq_factor,
                      "high_freq_factor": shape.rope_high_freq_factor,
                      "original_max_position_embeddings": shape.rope_original_context})
    cfg._attn_implementation = "eager"
    W = {k: torch.from_numpy(L.bf16_value(v)) for k, v in wts.items()}
    layer = ml.LlamaDecoderLayer(cfg, layer_idx=0).double()
    rot = ml.LlamaRotaryEmbedding(cfg)
    with torch.no_grad():
        a = layer.self_attn
        a.q_proj.weight.copy_(W["w_qkv"][:, :Hq * d].T)
        a.k_proj.weight.copy_(W["w_qkv"][:, Hq * d:(Hq + Hkv) * d].T)
        a.v_proj.weight.copy_(W["w_qkv"][:, (Hq + Hkv) * d:].T)
        a.o_proj.weight.copy_(W["w_o"].T)
        layer.mlp.gate_proj.weight.copy_(W["w_gu"][:, :I].T)
        layer.mlp.up_proj.weight.copy_(W["w_gu"][:, I:].T)
        layer.mlp.down_proj.weight.copy_(W["w_down"].T)
        layer.input_layernorm.weight.copy_(W["attn_norm"])
        layer.post_attention_layernorm.weight.copy_(W["mlp_norm"])
        x = W["x"].reshape(1, N, H)
        pos = torch.arange(N)[None]
        mask = torch.full((N, N), float("-inf"), dtype=torch.float64).triu(1)[None, None]
        out = layer(x, attention_mask=mask, position_ids=pos, position_embeddings=rot(x, pos))
    out = out[0] if isinstance(out, tuple) else out
    return out.numpy().reshape(N, H), rot.inv_freq.double().numpy()


HF_W = gen.Workload("layer-pin", 1, 2, 1, 256, 64, 128, 64, 0.0, 4)
HF_SHAPE = SHAPE.replace(intermediate=128)


def test_rope_frequencies_match_transformers_llama3():
    """The frequency table against transformers' "llama3" rotary scaling (its float32 table)."""
    _, inv = _hf_layer(HF_W, HF_SHAPE, gen.make_layer(HF_W, HF_SHAPE))
    np.testing.assert_allclose(L.rope_frequencies(HF_W.head_dim, HF_SHAPE), inv, rtol=1e-6)


def test_layer_matches_transformers_llama_decoder_layer():
    """The whole layer (dense causal attention) against transformers' LlamaDecoderLayer run in
    float64 on the same bf16 weights and input. The oracle rounds to bf16 at nine points and the
    library at none, so the two agree to a few bf16 ulps: every element within 4 ulps of bf16 at
    max(1, |x₂|) (2^-5 relative; measured 2 ulps) and a mean error below 0.005 (measured 0.0031).
    A swapped operand, a wrong rotation or a dropped term moves the output by 0.4 or more."""
    wts = gen.make_layer(HF_W, HF_SHAPE)
    ref, _ = _hf_layer(HF_W, HF_SHAPE, wts)
    got = L.layer(HF_W, HF_SHAPE, wts, dense=True).reshape(ref.shape)
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -5 * np.maximum(1.0, np.abs(ref))), float(err.max())
    assert err.mean() < 0.005, float(err.mean())

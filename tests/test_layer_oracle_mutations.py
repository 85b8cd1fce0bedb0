"""The layer oracle's pins have teeth: each case plants one plausible mistake in a copy of
``oracle/layer.py`` (operands swapped, a wrong rotation, a dropped term or residual, a transposed
head layout, a wrong activation, the frequency scaling skipped), loads the copy as a module of the
``oracle`` package and checks that the pins of test_layer_oracle_pins.py reject it. The real
oracle is never modified."""
import os
import types

import pytest

import oracle
import test_layer_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "layer.py")

MUTATIONS = {
    "gate-up-swapped": ("a = bf16_round(silu(gu[..., :I]) * gu[..., I:])",
                        "a = bf16_round(silu(gu[..., I:]) * gu[..., :I])"),
    "k-v-swapped": ("k = qkv[..., Hq * d: (Hq + Hkv) * d]", "k = qkv[..., (Hq + Hkv) * d:]"),
    "rope-sign": ("return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)",
                  "return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)"),
    "rope-interleaved-pairs": ("a, b = y[..., : d // 2], y[..., d // 2:]",
                               "a, b = y[..., 0::2], y[..., 1::2]"),
    "no-attention-residual": ('x1 = bf16_round(x + o_rows @ W["w_o"])',
                              'x1 = bf16_round(o_rows @ W["w_o"])'),
    "heads-not-transposed": ("o_rows = O.transpose(0, 2, 1, 3).reshape(B, N, H)",
                             "o_rows = O.reshape(B, N, H)"),
    "norm-gain-dropped": ("return bf16_round(gain * x * r)", "return bf16_round(x * r)"),
    "silu-as-sigmoid": ("return z / (1.0 + np.exp(-z))", "return 1.0 / (1.0 + np.exp(-z))"),
    "mlp-norm-on-layer-input": ('h2 = rms_norm(x1, W["mlp_norm"], shape.rms_eps)',
                                'h2 = rms_norm(x, W["mlp_norm"], shape.rms_eps)'),
    "rope-scaling-skipped": ("if shape.rope_factor <= 0:", "if True:"),
}

PIN_TESTS = [
    pins.test_rms_norm_closed_forms,
    pins.test_rope_identity_norm_and_relative_position,
    pins.test_rope_frequency_scaling_regimes,
    pins.test_silu_identity_and_limits,
    pins.test_layer_with_zero_projections_is_identity,
    pins.test_rope_frequencies_match_transformers_llama3,
    pins.test_layer_matches_transformers_llama_decoder_layer,
]


def mutant(name):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    m = types.ModuleType(f"oracle._layer_mutant_{name.replace('-', '_')}")
    m.__package__ = "oracle"
    exec(compile(text.replace(old, new), f"<{name}>", "exec"), m.__dict__)
    return m


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(monkeypatch, name):
    monkeypatch.setattr(pins, "L", mutant(name))
    caught = []
    for pin in PIN_TESTS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_copy_passes_every_pin(monkeypatch):
    m = types.ModuleType("oracle._layer_copy")
    m.__package__ = "oracle"
    exec(compile(open(SRC).read(), "<copy>", "exec"), m.__dict__)
    monkeypatch.setattr(pins, "L", m)
    for pin in PIN_TESTS:
        pin()

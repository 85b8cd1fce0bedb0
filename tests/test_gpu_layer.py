"""The decoder layer around the attention (C ABI ``s2o_layer_prefill``) against the layer oracle,
at τ = 0 (every causal key) and τ > 1 (the dense local window), where the attention's key sets
do not depend on score rounding, and with the dense causal baseline.

Tolerance, from the arithmetic: GPU and oracle round to bf16 at the same points and differ in
between by fp32 against binary64 and, mainly, by the attention's own parity error (max-abs 2e-2,
mean-abs 1e-3 on O, bf16 probabilities in P·V). Through W_o (H inputs of weight N(0, 1/H)) that
error reaches x₁ = x + O·W_o at about its own size, 1e-3, a quarter of a bf16 ulp of x₁ (2^-8 for
|x₁| in [0.5, 1)): a large share of x₁ lands one ulp apart, and the MLP path (norm, gate and up,
W_down) carries that into x₂ at a similar size before x₂'s own rounding. Bound: one ulp on average
(2^-8 · mean|x₂|) and three ulps of the largest magnitude at most (one from x₁, one from the MLP
term, one from the final rounding: 3 · 2^(⌊log2 max|x₂|⌋ − 7)).
"""
import math

import numpy as np
import pytest
import torch

import gen
import long_context_sparse_stripe_b200 as s2o
from oracle import layer as oracle_layer

pytestmark = pytest.mark.gpu

W_L = gen.Workload("layer-small", batch=1, n_q_heads=4, n_kv_heads=2, seq_len=1024, head_dim=128,
                   segment_len=256, block_size=128, tau=0.0, seed=21)
SHAPE = gen.LAYER_8B.replace(intermediate=1024)


def check(got: torch.Tensor, want: np.ndarray):
    g = got.float().cpu().numpy().astype(np.float64).reshape(want.shape)
    err = np.abs(g - want)
    top = np.max(np.abs(want))
    ulp_max = 2.0 ** (math.floor(math.log2(top)) - 7)
    assert err.max() <= 3 * ulp_max, f"max abs error {err.max():.3g} > {3 * ulp_max:.3g}"
    assert err.mean() <= 2.0 ** -8 * np.mean(np.abs(want)), f"mean abs error {err.mean():.3g}"


@pytest.mark.parametrize("w,dense", [(W_L, False), (W_L.replace(tau=1.5), False), (W_L, True),
                                     (W_L.replace(batch=2, seed=22, tau=1.5), False)],
                         ids=["s2o-tau0", "s2o-local", "dense", "s2o-local-batch2"])
def test_layer_matches_oracle(w, dense):
    wts = gen.make_layer(w, SHAPE)
    want = oracle_layer.layer(w, SHAPE, wts, dense=dense)
    cfg = s2o.Config.of(w)
    dev = {k: v.cuda() for k, v in wts.items()}
    x = dev.pop("x").clone()
    s2o.layer_prefill(cfg, SHAPE, dev, x, dense=dense)
    torch.cuda.synchronize()
    assert s2o.check_device_status() == 0
    check(x, want)


def test_layer_s2o_equals_dense_at_tau_zero_within_attention_rounding():
    """τ = 0 selects every causal key: the S2O layer and the dense-baseline layer agree."""
    w = W_L
    wts = {k: v.cuda() for k, v in gen.make_layer(w, SHAPE).items()}
    cfg = s2o.Config.of(w)
    xs = wts.pop("x")
    a = s2o.layer_prefill(cfg, SHAPE, wts, xs.clone())
    b = s2o.layer_prefill(cfg, SHAPE, wts, xs.clone(), dense=True)
    torch.cuda.synchronize()
    d = (a.float() - b.float()).abs()
    top = float(b.float().abs().max())
    assert float(d.max()) <= 3 * 2.0 ** (math.floor(math.log2(top)) - 7)

"""The pins have teeth: each test plants one plausible mistake in a copy of the oracle's source
(a dropped term, a wrong sign, an off-by-one, a transposed operand, a reversed tie-break), builds
it on the CPU and checks that the pin suite in test_oracle_pins.py rejects it. The real oracle is
never modified."""
import os
import shutil
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "s2o_oracle.c")

MUTATIONS = {
    "u-sign": ("u[t] = kbar_top[t] - kbar_all[t];", "u[t] = kbar_all[t] - kbar_top[t];"),
    "drop-score-scale": ("Kbar + (size_t)c * d, d) * sigma;", "Kbar + (size_t)c * d, d);"),
    "visible-count-le": ("if (perm_k[c * B + e] < s * S) ++cntv;",
                         "if (perm_k[c * B + e] <= s * S) ++cntv;"),
    "tie-break-reversed": ("return (a->idx > b->idx) - (a->idx < b->idx);",
                           "return (a->idx < b->idx) - (a->idx > b->idx);"),
    "local-window-off-by-one": ("for (int j = s0; j <= i; ++j) keys[nk++] = j;",
                                "for (int j = s0; j < i; ++j) keys[nk++] = j;"),
    "gqa-mapping": ("G = Hq / Hkv, g = h / G;", "G = Hq / Hkv, g = h % Hkv;"),
    "no-normalisation": ("double p = any ? w[c] / Z : 0.0;", "double p = any ? w[c] : 0.0;"),
    "transposed-block-score": (
        "dot_f32(Qbar + (size_t)b * d, Kbar + (size_t)c * d, d) * sigma;",
        "dot_f32(Qbar + (size_t)c * d, Kbar + (size_t)b * d, d) * sigma;"),
    "kappa-from-mean-key": ("kappa[j] = dot_f32_bf16(qbar, K + (size_t)j * d, d);",
                            "kappa[j] = dot_f32_bf16(kbar_all, K + (size_t)j * d, d);"),
    "dropped-visibility-weight": (
        "w[c] = ns[c] > 0 ? (double)ns[c] * oracle_exp64((double)rb[c] - (double)M) : 0.0;",
        "w[c] = ns[c] > 0 ? oracle_exp64((double)rb[c] - (double)M) : 0.0;"),
    # Online early stop: the stopping block dropped instead of kept.
    "online-stop-drops-block": ("          kept = x + 1;\n          break;",
                                "          kept = x;\n          break;"),
    # Online early stop: the share's denominator without the block itself.
    "online-share-denominator": ("          den += ek[x];\n          const double share = ek[x] / den;",
                                 "          const double share = ek[x] / den;\n          den += ek[x];"),
    # Online early stop: the smallest share over the rows instead of the largest.
    "online-min-over-rows": ("          if (share > ms[x]) ms[x] = share;",
                             "          if (e == 0 || share < ms[x]) ms[x] = share;"),
    # Pooled means summed in one pass instead of chunks of B list entries.
    "one-chunk-sum": ("  float *total = calloc((size_t)d, sizeof(float));",
                      "  chunk = len;\n  float *total = calloc((size_t)d, sizeof(float));"),
    # The normaliser Z summed in one pass instead of 32-block chunks.
    "one-chunk-normaliser": (
        "for (int c0 = 0; c0 < nB; c0 += 32) {\n      double part = 0.0;\n"
        "      for (int c = c0; c < c0 + 32 && c < nB; ++c)",
        "for (int c0 = 0; c0 < nB; c0 += nB) {\n      double part = 0.0;\n"
        "      for (int c = c0; c < c0 + nB && c < nB; ++c)"),
    # Orderings ascending instead of descending (the shared comparator of both orderings).
    "orderings-ascending": ("return a->key > b->key ? -1 : 1;", "return a->key < b->key ? -1 : 1;"),
    # Selected blocks listed least important first.
    "selection-ascending": ("if (a->p != b->p) return a->p > b->p ? -1 : 1;",
                            "if (a->p != b->p) return a->p < b->p ? -1 : 1;"),
    # A block whose score equals τ dropped (p > τ instead of p ≥ τ).
    "selection-strict": ("if (ns[c] > 0 && p >= tau) {", "if (ns[c] > 0 && p > tau) {"),
    # The query score without the mean key (rho = q·kbar_top).
    "rho-drops-mean-key": ("u[t] = kbar_top[t] - kbar_all[t];", "u[t] = kbar_top[t];"),
    # kbar_top pooled over the second-ranked key block instead of the top one.
    "kbar-top-second-block": ("list_mean(K, d, perm_k, B, B, kbar_top);",
                              "list_mean(K, d, perm_k + B, B, B, kbar_top);"),
    # A selected block's key at the segment start let through (it is already a local key).
    "selected-keys-le": ("if (j < s0) keys[nk++] = j;", "if (j <= s0) keys[nk++] = j;"),
    # The segment-local query ordering never applied.
    "query-order-skipped": (
        "if (cfg->query_perm) qsort(tmp, (size_t)S, sizeof(keyed), cmp_keyed_desc);",
        "if (0 && cfg->query_perm) qsort(tmp, (size_t)S, sizeof(keyed), cmp_keyed_desc);"),
    # Query block means over original-order blocks instead of permuted ones.
    "qbar-original-order": (
        "list_mean(Q, d, perm_q + (size_t)b * B, B, B, Qbar + (size_t)b * d);",
        "list_mean(Q, d, ident + (size_t)b * B, B, B, Qbar + (size_t)b * d);"),
    # Attention logits without the 1/sqrt(d) scale.
    "attention-no-scale": ("    z[a] = acc * inv_sqrt_d;\n    if (z[a] > m) m = z[a];",
                           "    z[a] = acc;\n    if (z[a] > m) m = z[a];"),
    # Attention output not divided by the softmax normaliser.
    "attention-unnormalised": ("  for (int t = 0; t < d; ++t) out[t] /= den;", ""),
    # Attention weights applied to the keys instead of the values.
    "attention-values-from-keys": ("const uint16_t *vj = V + (size_t)keys[a] * d;",
                                   "const uint16_t *vj = K + (size_t)keys[a] * d;"),
    # Dense causal attention without the 1/sqrt(d) scale.
    "dense-no-scale": ("        z[j] = acc * inv_sqrt_d;", "        z[j] = acc;"),
    # 4-bit centroids: codes of the key centroids without the channel's offset.
    "int4-key-code-no-offset": ("float code = rintf((Kbar[(size_t)c * d + t] - mn) / st);",
                                "float code = rintf(Kbar[(size_t)c * d + t] / st);"),
    # 4-bit centroids: the integer product not scaled back by the query step.
    "int4-query-scale-dropped": ("r[(size_t)b * nB + c] = ((float)acc * sq) * sigma;",
                                 "r[(size_t)b * nB + c] = ((float)acc) * sigma;"),
    # 4-bit centroids: sixteen steps over the channel's range instead of fifteen.
    "int4-sixteen-steps": ("float st = (mx - mn) / 15.0f;", "float st = (mx - mn) / 16.0f;"),
    # One key ordering per KV head: the pooled query of the head itself, not of its group.
    "shared-order-own-head": ("for (int hh = g * G; hh < (g + 1) * G; ++hh) {",
                              "for (int hh = h; hh < h + 1; ++hh) {"),
    # One key ordering per KV head: the group's mean queries summed, not averaged.
    "shared-order-sum-not-mean": ("for (int t = 0; t < d; ++t) qsum[t] = qsum[t] / (float)G;",
                                  "for (int t = 0; t < d; ++t) qsum[t] = qsum[t];"),
}

# The pins that run against each mutant (all CPU, seconds each).
PIN_TESTS = [
    pins.test_hand_case_intermediates,
    pins.test_hand_case_probabilities_closed_form,
    lambda: [pins.test_hand_case_selection_and_pairs(t) for t in ("0.0", "0.28", "0.3", "0.4")],
    pins.test_hand_case_key_sets,
    lambda: [pins.test_tau_zero_is_dense_causal_attention(w)
             for w in (pins.gen.workload("tiny"), pins.SMALL_GQA)],
    lambda: [pins.test_tau_above_one_is_local_window_only(w)
             for w in (pins.gen.workload("tiny"), pins.SMALL_GQA)],
    pins.test_threshold_is_inclusive,
    pins.test_index_arrays_are_sorted_permutations,
    pins.test_probabilities_and_selection_rule,
    pins.test_float64_rederivation_of_pooled_quantities,
    pins.test_sum_order_case_chunked_means,
    pins.test_sum_order_case_normaliser_chunks,
    pins.test_shared_key_order_variant,
    pins.test_int4_centroid_variant,
    pins.test_int4_scores_exact_on_grid_aligned_centroids,
    pins.test_online_stop_hand_case,
    lambda: pins.test_online_stop_against_softmax_probabilities(0.03),
]


def build_mutant(tmp_path, name):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new))
    lib = tmp_path / f"{name}.so"
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(lib), str(src), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(tmp_path, name):
    lib = build_mutant(tmp_path, name)
    caught = []
    with oracle.use_library(lib):
        for pin in PIN_TESTS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(getattr(pin, "__name__", "lambda"))
                break  # one rejection is enough
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_copy_passes_every_pin(tmp_path):
    src = tmp_path / "same.c"
    shutil.copy(SRC, src)
    lib = tmp_path / "same.so"
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(lib), str(src), "-lm"], check=True)
    with oracle.use_library(str(lib)):
        for pin in PIN_TESTS:
            pin()

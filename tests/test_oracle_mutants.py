"""Planted mistakes in the oracle must be caught by its pins.

Each case rewrites one spot of a temporary copy of oracle/moe_oracle.c (a
dropped term, a wrong sign or index, a transposed operand, a wrong rule),
compiles it, and runs the pins from tests/pins.py against it: at least one
pin must fail.  The real oracle source is never modified.
"""
import os
import shutil

import pytest

import oracle
import pins

MUTANTS = {
    "nibble_order": ("*hi = j & 1;", "*hi = 1 - (j & 1);"),
    "scale_bias_swapped": ("s = orc_f16_to_f64(rd16(blob + sb));\n    b = orc_f16_to_f64(rd16(blob + sb + 2));",
                           "s = orc_f16_to_f64(rd16(blob + sb + 2));\n    b = orc_f16_to_f64(rd16(blob + sb));"),
    "sb_row_major": ("((size_t)(kk / 64) * 32u + (size_t)r) * 4u",
                     "((size_t)r * (size_t)(ks / 64) + (size_t)(kk / 64)) * 4u"),
    "gate_up_halves": ("r = (n % 16) + 16 * m;", "r = (n % 16) + 16 * (1 - m);"),
    "f16_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "f16_exponent_bias": ("ldexp((double)(1024 + m), e - 25)", "ldexp((double)(1024 + m), e - 24)"),
    "gelu_sign": ("(1.0 + tanh(", "(1.0 - tanh("),
    "gelu_cubic_dropped": ("(v + 0.044715 * v * v * v)", "(v + 0.044715 * v * v)"),
    "down_transposed": ("a += W[(size_t)r * F + n] * h[n];", "a += W[(size_t)(n % D) * F + (r % F)] * h[n];"),
    "up_not_multiplied": ("h[n] = orc_gelu_tanh(g[n]) * u[n];", "h[n] = orc_gelu_tanh(g[n]) + u[n];"),
    "router_bias_sign": ("if (bias) acc = acc + bias[e];", "if (bias) acc = acc - bias[e];"),
    "router_scale_index": ("ws_f16[(size_t)e * ng + g]", "ws_f16[(size_t)e * ng + (ng - 1 - g)]"),
    "topk_tie_high_id": ("if (best < 0 || logits[e] > logits[best]) best = e;",
                         "if (best < 0 || logits[e] >= logits[best]) best = e;"),
    "softmax_not_normalised": ("for (int i = 0; i < K; ++i) w[i] /= z;",
                               "for (int i = 0; i < K; ++i) w[i] /= 1.0;"),
    "combine_weight_order": ("y[r] += gate_w[i] * ye[r];", "y[r] += gate_w[K - 1 - i] * ye[r];"),
    "shared_dropped": ("    if (shared_blob)\n        orc_expert_ffn(shared_blob, D, FS, x, y);\n    else\n",
                       "    if (0)\n        orc_expert_ffn(shared_blob, D, FS, x, y);\n    else\n"),
    "lfu_evicts_most_frequent": ("count[r] < count[victim] ||", "count[r] > count[victim] ||"),
    "lfu_recency_reversed": ("(last_use[r] < last_use[victim] ||", "(last_use[r] > last_use[victim] ||"),
    "lfu_last_use_not_updated": ("last_use[e] = step + 1u;", "last_use[e] = 0u;"),
    "lfu_pinned_ignored": ("if (pinned) continue;", "(void)pinned;"),
    "lfu_highest_empty_slot": ("if (expert_in[s] < 0) { slot = s; break; }", "if (expert_in[s] < 0) { slot = s; }"),
    "lfu_counts_per_expert": ("for (int p = 0; p < T * K; ++p) count[ids[p]] += 1u;",
                              "for (int e2 = 0; e2 < E; ++e2) if (sel[e2]) count[e2] += 1u;"),
    "lru_recency_reversed": ("if (victim < 0 || last_use[victim] > last_use[r] ||",
                             "if (victim < 0 || last_use[victim] < last_use[r] ||"),
    "decay_not_halving": ("for (int e = 0; e < E; ++e) count[e] >>= 1;",
                          "for (int e = 0; e < E; ++e) count[e] >>= 0;"),
    "in_cache_count_kept": ("if (policy == ORC_POLICY_LFU_IN_CACHE) count[victim] = 0u;",
                            "if (policy == ORC_POLICY_LFU_IN_CACHE) count[victim] = count[victim];"),
    "group_unstable": ("        for (int p = 0; p < T * K; ++p)\n            if (ids[p] == e) pairs[pos++] = p;",
                       "        for (int p = T * K - 1; p >= 0; --p)\n            if (ids[p] == e) pairs[pos++] = p;"),
    "attn_gqa_modulo": ("const int g = h / grp;", "const int g = h % Hkv;"),
    "attn_scale_dropped": ("w[i] = scale * a;", "w[i] = a;"),
    "attn_window_short": ("const int first = n > cap ? n - cap : 0;", "const int first = n > cap ? n - cap + 1 : 0;"),
    "attn_not_normalised": ("o[(size_t)h * hd + d] = acc / z;", "o[(size_t)h * hd + d] = acc;"),
    "attn_value_slot_linear": ("acc += w[i] * orc_f16_to_f64(vg[slot * hd + d]);",
                               "acc += w[i] * orc_f16_to_f64(vg[(size_t)i * hd + d]);"),
    "bf16_truncates": ("q = rint(ldexp(a, 8 - e));", "q = floor(ldexp(a, 8 - e));"),
    "bf16_ties_away": ("q = rint(ldexp(a, 8 - e));", "q = round(ldexp(a, 8 - e));"),
    "bf16_no_subnormal_clamp": ("if (e < -125) e = -125;", "(void)0;"),
    "rms_eps_dropped": ("rms = sqrt(ss / (double)D + 1e-6);", "rms = sqrt(ss / (double)D);"),
    "rms_sum_not_mean": ("rms = sqrt(ss / (double)D + 1e-6);", "rms = sqrt(ss + 1e-6);"),
    "residual_dropped": ("r_out[i] = r_in[i] + y[i];", "r_out[i] = y[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / "moe_oracle.c"
    mpath.write_text(src.replace(old, new))
    shutil.copy(os.path.join(os.path.dirname(oracle.SRC), "moe_oracle.h"), tmp_path / "moe_oracle.h")
    lib = oracle.build(str(mpath), str(tmp_path / "libmut.so"), extra=("-I", str(tmp_path)))
    M = oracle.Oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(M)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
            break
    assert failed, f"planted mistake '{name}' passed every pin"

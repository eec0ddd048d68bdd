"""Plant plausible mistakes in copies of the oracle (on the CPU) and require the
pins to catch every one: a dropped term, a wrong sign or index, a swapped operand.
Each mutant is a single textual edit of oracle.c, compiled to a temp library."""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "bf16_truncation": ("const double kr = nearbyint(k);", "const double kr = trunc(k);"),
    "bf16_ties_away_from_zero": ("const double kr = nearbyint(k);", "const double kr = round(k);"),
    "rope_sign": ("out[j] = x[j] * c - x[j + half] * s;", "out[j] = x[j] * c + x[j + half] * s;"),
    "rope_freq_full_dim": ("-2.0 * (double)j / (double)rope_dims", "-2.0 * (double)j / (double)dim"),
    "rope_interleaved_pairs": ("out[j] = x[j] * c - x[j + half] * s;\n        out[j + half] = x[j] * s + x[j + half] * c;",
                               "out[2 * j] = x[2 * j] * c - x[2 * j + 1] * s;\n        out[2 * j + 1] = x[2 * j] * s + x[2 * j + 1] * c;"),
    "key_rope_last_position": ("w, b * c->r, NULL, NULL,\n                              NULL,",
                               "w, b * c->r + c->r - 1, NULL, NULL,\n                              NULL,"),
    "query_not_rotated": ("qsa_oracle_rotate_query(c, idx_q_row, i, qrot);",
                          "qsa_oracle_rotate_query(c, idx_q_row, 0, qrot);"),
    "pool_divisor": ("kbar[j] = s / (double)c->r;", "kbar[j] = s / (double)(c->r + 1);"),
    "rms_no_eps": ("sqrt(ms + c->rms_eps)", "sqrt(ms)"),
    "rms_no_sqrt": ("const double rms = sqrt(ms + c->rms_eps);", "const double rms = ms + c->rms_eps;"),
    "relu_dropped": ("if (dot > 0.0) I += dot;", "I += dot;"),
    "score_one_head": ("dot += bf(qrot[(size_t)h * dim + j])", "dot += bf(qrot[(size_t)0 * dim + j])"),
    "mask_includes_own_block": ("const int64_t n_vis = i / c->r;\n    const int64_t k_b",
                                "const int64_t n_vis = (i + 1) / c->r;\n    const int64_t k_b"),
    "target_includes_own_block": ("const int64_t n_vis = i / c->r;\n    if (n_vis <= 0) return;",
                                  "const int64_t n_vis = (i + 1) / c->r;\n    if (n_vis <= 0) return;"),
    "tie_to_higher_index": ("return (a->b > b->b) - (a->b < b->b);", "return (a->b < b->b) - (a->b > b->b);"),
    "budget_off_by_one": ("const int64_t m = n_vis < k_b ? n_vis : k_b;",
                          "const int64_t m = n_vis < k_b ? n_vis : k_b - 1;"),
    "tail_excludes_query": ("for (int64_t t = cur * c->r; t <= i; ++t)", "for (int64_t t = cur * c->r; t < i; ++t)"),
    "no_softmax_scale": ("logit[t] = dot * scale;", "logit[t] = dot;"),
    "gqa_modulo": ("const int kvh = h / g;\n        double m = -INFINITY;",
                   "const int kvh = h % c->kv_heads;\n        double m = -INFINITY;"),
    "bwd_gqa_modulo": ("const int kvh = h / g;\n        const double* qh", "const int kvh = h % c->kv_heads;\n        const double* qh"),
    "values_from_keys": ("const uint16_t* vr = vc +", "const uint16_t* vr = kc +"),
    "decode_pool_early": ("if ((p + 1) % c->r == 0) {", "if (p % c->r == 0) {"),
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_ties_up": ("if (a > mid || (a == mid && (c & 1) == 0)) best", "if (a >= mid) best"),
    "quant_scale_max_normal_240": ("fl32_div(amax, 448.0)", "fl32_div(amax, 240.0)"),
    "q8_value_scale_dropped": ("o[j] += w * (qsa_oracle_e4m3_value(vc[row * d + j]) * vs[row]);",
                               "o[j] += w * qsa_oracle_e4m3_value(vc[row * d + j]);"),
    "bwd_softmax_jacobian_no_delta": ("const double dz = p * (gv - delta);", "const double dz = p * gv;"),
    "bwd_dk_unscaled": ("dkr[j] += scale * dz * qh[j];", "dkr[j] += dz * qh[j];"),
    "bwd_dv_from_dz": ("dvr[j] += p * gh[j];", "dvr[j] += dz * gh[j];"),
    "bwd_gather_first_token": ("kt[(size_t)t * row + j] = bf(kc[(size_t)tokens[t] * row + j]);",
                               "kt[(size_t)t * row + j] = bf(kc[(size_t)tokens[0] * row + j]);"),
    "target_mean_pool": ("if (avg[b * c->r + e] > best) best = avg[b * c->r + e];", "best += avg[b * c->r + e];"),
    "target_max_over_heads": ("avg[j] += exp(z[j] - mx) / den;", "avg[j] = fmax(avg[j], exp(z[j] - mx) / den);"),
    "target_not_normalised": ("for (int64_t b = 0; b < n_vis; ++b) t[b] /= mass;", ";"),
    "target_unscaled_logits": ("z[j] = dot * scale;", "z[j] = dot;"),
    "target_keys_shifted_past_query": ("const uint16_t* kr = kc + ((size_t)j * hkv + h / g) * d;",
                                       "const uint16_t* kr = kc + ((size_t)(j + 1) * hkv + h / g) * d;"),
    "kl_gradient_sign": ("if (ds) ds[b] = tsum * exp(log_soft) - t[b];", "if (ds) ds[b] = t[b] - tsum * exp(log_soft);"),
    "kl_reversed": ("if (t[b] > 0.0) kl += t[b] * (log(t[b]) - log_soft);",
                    "if (t[b] > 0.0) kl += exp(log_soft) * (log_soft - log(t[b]));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/present"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    so = str(tmp_path / "liboracle_mutant.so")
    subprocess.check_call(["gcc", *oracle.GCC_FLAGS, "-o", so, str(path), "-lm"])

    def make(**kw):
        return oracle.Oracle(lib_path=so, **kw)

    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(make)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"

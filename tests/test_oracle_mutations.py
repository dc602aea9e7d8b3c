"""The oracle's pins against planted slips (CPU only).

Each case below plants one plausible mistake in a copy of ``oracle/oracle.c`` (the same
mistake in the incremental step and in the full-sequence recompute where both hold the
step, so that their agreement cannot hide it), builds the copy, and runs
``tests/test_oracle_pins.py`` against it in a fresh process. Every slip must make at
least one pin fail. A pattern that no longer occurs in the oracle fails the case, so a
change to the oracle's text asks for its slips to be restated.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

SLIPS = {
    # wiring of the layer
    "gate_up_swapped": [("gt[i] = orc_silu(gt[i]) * up[i];", "gt[i] = orc_silu(up[i]) * gt[i];"),
                        ("G[i] = orc_silu(G[i]) * U[i];", "G[i] = orc_silu(U[i]) * G[i];")],
    "query_not_rotated": [("for (int hh = 0; hh < Hq; hh++) orc_rope(D, pos, c->rope_theta, q + hh * D);", ""),
                          ("for (int hh = 0; hh < Hq; hh++) orc_rope(D, t, c->rope_theta, Q + ((int64_t)t * Hq + hh) * D);",
                           "")],
    "key_stored_before_rotation": [("for (int g = 0; g < Hkv; g++) orc_rope(D, pos, c->rope_theta, k + g * D);\n", ""),
                                   ("                orc_rope(D, t, c->rope_theta, Kf + g * D);\n", "")],
    "value_rotated_too": [("for (int g = 0; g < Hkv; g++) orc_rope(D, pos, c->rope_theta, k + g * D);",
                           "for (int g = 0; g < Hkv; g++) { orc_rope(D, pos, c->rope_theta, k + g * D); "
                           "orc_rope(D, pos, c->rope_theta, v + g * D); }"),
                          ("                orc_rope(D, t, c->rope_theta, Kf + g * D);",
                           "                orc_rope(D, t, c->rope_theta, Kf + g * D); orc_rope(D, t, c->rope_theta, Vf + g * D);")],
    "value_rounding_off_by_one_bit": [
        ("vcache[kv_index(c, max_ctx, l, g, pos) + i] = orc_store(v[g * D + i], dt);",
         "vcache[kv_index(c, max_ctx, l, g, pos) + i] = (uint16_t)(orc_store(v[g * D + i], dt) ^ (dt ? 1u : 0u));"),
        ("Vs[((int64_t)g * n + t) * D + i] = orc_store(Vf[g * D + i], dt);",
         "Vs[((int64_t)g * n + t) * D + i] = (uint16_t)(orc_store(Vf[g * D + i], dt) ^ (dt ? 1u : 0u));")],
    "attention_skips_current_position": [("orc_attention(D, pos + 1,", "orc_attention(D, pos > 0 ? pos : 1,"),
                                         ("orc_attention(D, t + 1,", "orc_attention(D, t > 0 ? t : 1,")],
    "kv_head_map_modulo": [("int g = (int)(((int64_t)hh * Hkv) / Hq);", "int g = hh % Hkv;")],
    "mlp_norm_uses_attention_gain": [("L[W_MLP_NORM]", "L[W_ATTN_NORM]")],
    "final_norm_uses_last_mlp_gain": [
        ("orc_rmsnorm(d, x, w->final_norm,",
         "orc_rmsnorm(d, x, w->layers[(int64_t)(c->n_layers - 1) * W_PER_LAYER + W_MLP_NORM],"),
        ("orc_rmsnorm(d, X + (int64_t)t * d, w->final_norm,",
         "orc_rmsnorm(d, X + (int64_t)t * d, w->layers[(int64_t)(c->n_layers - 1) * W_PER_LAYER + W_MLP_NORM],")],
    "no_final_norm": [("        orc_rmsnorm(d, x, w->final_norm, dt, c->rms_eps, h);\n"
                       "        head_matvec(c, w, h, logits);",
                       "        head_matvec(c, w, x, logits);"),
                      ("        head_matvec(c, w, H + (int64_t)t * d, logits + (int64_t)t * c->vocab);",
                       "        head_matvec(c, w, X + (int64_t)t * d, logits + (int64_t)t * c->vocab);")],
    "residual_overwritten_after_attention": [
        ("        layer_matvec(c, w, l, W_O, d, Hq * D, o, y);\n        for (int i = 0; i < d; i++) x[i] += y[i];",
         "        layer_matvec(c, w, l, W_O, d, Hq * D, o, y);\n        for (int i = 0; i < d; i++) x[i] = y[i];"),
        ("            for (int i = 0; i < d; i++) x[i] += Y[i];\n            orc_rmsnorm",
         "            for (int i = 0; i < d; i++) x[i] = Y[i];\n            orc_rmsnorm")],
    "lm_head_is_the_embedding": [("else orc_matvec(c->vocab, c->d_model, w->lm_head,", "else orc_matvec(c->vocab, c->d_model, w->tok_emb,")],
    # FP8 weights
    "e4m3_exponent_bias": [("else v = ldexp((double)(8 + m), e - 10);", "else v = ldexp((double)(8 + m), e - 11);")],
    "e4m3_encode_rounds_half_up": [("    if (rem > 0.5 || (rem == 0.5 && (qi & 1u))) qi++;\n    if (exp8 == -6",
                                    "    if (rem >= 0.5) qi++;\n    if (exp8 == -6")],
    "e4m3_scale_from_mean": [("const float s = amax > 0.f ? amax / 448.0f : 1.0f;", "const float s = amax > 0.f ? amax / 440.0f : 1.0f;")],
    "q8_scale_divides": [("y[n] = (double)scale[n] * acc;", "y[n] = acc / (double)scale[n];")],
    "q8_gate_is_up": [("    if (w->q8) orc_matvec_q8(N, K, w->q8[i], w->q8_scale[i], x, y);",
                       "    if (w->q8) orc_matvec_q8(N, K, w->q8[j == W_GATE ? i + 1 : i], w->q8_scale[j == W_GATE ? i + 1 : i], x, y);")],
    "q8_head_reads_16bit_weights": [("if (w->q8) orc_matvec_q8(c->vocab, c->d_model, w->q8_head, w->q8_head_scale, x, y);",
                                     "if (0 && w->q8) orc_matvec_q8(c->vocab, c->d_model, w->q8_head, w->q8_head_scale, x, y);")],
    "embedding_row_off_by_one": [("x[i] = orc_value(w->tok_emb[(int64_t)token * d + i], dt);",
                                  "x[i] = orc_value(w->tok_emb[(int64_t)(token + (token + 1 < c->vocab)) * d + i], dt);")],
    "rope_position_off_by_one": [("orc_rope(D, pos, c->rope_theta, q + hh * D);", "orc_rope(D, pos + 1, c->rope_theta, q + hh * D);"),
                                 ("orc_rope(D, pos, c->rope_theta, k + g * D);", "orc_rope(D, pos + 1, c->rope_theta, k + g * D);"),
                                 ("orc_rope(D, t, c->rope_theta, Q + ((int64_t)t * Hq + hh) * D);",
                                  "orc_rope(D, t + 1, c->rope_theta, Q + ((int64_t)t * Hq + hh) * D);"),
                                 ("orc_rope(D, t, c->rope_theta, Kf + g * D);", "orc_rope(D, t + 1, c->rope_theta, Kf + g * D);")],
    "attention_skips_position_zero": [
        ("orc_attention(D, pos + 1, q + hh * D, kcache + kv_index(c, max_ctx, l, g, 0),\n"
         "                          vcache + kv_index(c, max_ctx, l, g, 0), dt, o + hh * D);",
         "orc_attention(D, pos > 0 ? pos : 1, q + hh * D, kcache + kv_index(c, max_ctx, l, g, pos > 0 ? 1 : 0),\n"
         "                          vcache + kv_index(c, max_ctx, l, g, pos > 0 ? 1 : 0), dt, o + hh * D);"),
        ("orc_attention(D, t + 1, Q + ((int64_t)t * Hq + hh) * D, Ks + (int64_t)g * n * D,\n"
         "                              Vs + (int64_t)g * n * D, dt, O + ((int64_t)t * Hq + hh) * D);",
         "orc_attention(D, t > 0 ? t : 1, Q + ((int64_t)t * Hq + hh) * D, Ks + ((int64_t)g * n + (t > 0)) * D,\n"
         "                              Vs + ((int64_t)g * n + (t > 0)) * D, dt, O + ((int64_t)t * Hq + hh) * D);")],
    # building blocks
    "rmsnorm_fixed_eps": [("double r = 1.0 / sqrt(ss / n + eps);", "double r = 1.0 / sqrt(ss / n + 1e-6);")],
    "score_scale_missing": [("double scale = 1.0 / sqrt((double)D)", "double scale = 1.0")],
    "softmax_denominator_wrong": [("s[j] = exp(s[j] - m); sum += s[j];",
                                   "s[j] = exp(s[j] - m); sum += s[j] * 0.5 + 0.5 * s[j] * (j == 0);")],
    "rope_angle_exponent": [("pow(theta, -2.0 * i / D)", "pow(theta, -1.0 * i / D)")],
    "rope_rotation_sign": [("v[i] = a * c - b * s;", "v[i] = a * c + b * s;"),
                           ("v[i + half] = b * c + a * s;", "v[i + half] = b * c - a * s;")],
    "rope_interleaved_pairs": [("double a = v[i], b = v[i + half];", "double a = v[2 * i], b = v[2 * i + 1];"),
                               ("v[i] = a * c - b * s;", "v[2 * i] = a * c - b * s;"),
                               ("v[i + half] = b * c + a * s;", "v[2 * i + 1] = b * c + a * s;")],
    "rmsnorm_eps_outside_sqrt": [("double r = 1.0 / sqrt(ss / n + eps);", "double r = 1.0 / (sqrt(ss / n) + eps);")],
    "rmsnorm_sum_not_mean": [("double r = 1.0 / sqrt(ss / n + eps);", "double r = 1.0 / sqrt(ss + eps);")],
    "silu_is_sigmoid": [("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));")],
    "argmax_last_of_ties": [("if (v[i] > v[best]) best = i;", "if (v[i] >= v[best]) best = i;")],
    "matvec_transposed": [("const uint16_t *row = W + (int64_t)n * K;", "const uint16_t *row = W + (int64_t)n;"),
                          ("for (int k = 0; k < K; k++) acc += tv[row[k]] * x[k];",
                           "for (int k = 0; k < K; k++) acc += tv[row[(int64_t)k * N]] * x[k];")],
    # sampling
    "sample_temperature_multiplies": [("total += exp((logits[cand[k]] - logits[cand[0]]) / temperature);",
                                       "total += exp((logits[cand[k]] - logits[cand[0]]) * temperature);")],
    "sample_ties_to_highest_index": [("if (best < 0 || v > (isnan(logits[best]) ? -INFINITY : logits[best])) best = i;",
                                      "if (best < 0 || v >= (isnan(logits[best]) ? -INFINITY : logits[best])) best = i;")],
    "sample_boundary_inclusive": [("            if (cum[k] > r) {", "            if (cum[k] >= r) {")],
    "sample_draw_uses_output_pos": [("return (double)(orc_splitmix64(seed, (uint64_t)pos + 1) >> 40) / 16777216.0;",
                                     "return (double)(orc_splitmix64(seed, (uint64_t)pos) >> 40) / 16777216.0;")],
    "sample_cumulative_from_last_candidate": [("        const double r = u * total;", "        const double r = (1.0 - u) * total;")],
    "splitmix64_second_shift": [("z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;", "z = (z ^ (z >> 28)) * 0x94D049BB133111EBull;")],
    # storage types
    "bf16_store_truncates": [("return (uint16_t)((x + 0x7FFFu + lsb) >> 16);", "return (uint16_t)(x >> 16);")],
    "fp16_store_rounds_half_up": [("if (rem > 0.5 || (rem == 0.5 && (qi & 1u))) qi++;", "if (rem >= 0.5) qi++;")],
    "fp16_subnormal_scale": [("if (e == 0) v = ldexp((double)m, -24);", "if (e == 0) v = ldexp((double)m, -25);")],
}

# runs the pins against a given oracle library (the oracle's build step is replaced by that path)
_RUNNER = r"""
import sys, pytest
import oracle.build as ob
ob.build = lambda force=False: sys.argv[1]
sys.exit(pytest.main(["-q", "-x", "-p", "no:cacheprovider", "tests/test_oracle_pins.py"]))
"""


def _plant(name, tmpdir):
    src = open(SRC).read()
    for old, new in SLIPS[name]:
        if old not in src:
            return ("missing", old)
        src = src.replace(old, new)
    c, so = os.path.join(tmpdir, f"orc_{name}.c"), os.path.join(tmpdir, f"orc_{name}.so")
    with open(c, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", so, c, "-lm"])
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", _RUNNER, so], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return (r.returncode, r.stdout[-2000:])


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    tmpdir = str(tmp_path_factory.mktemp("slips"))
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:  # each case is its own process
        futs = {name: ex.submit(_plant, name, tmpdir) for name in SLIPS}
        return {name: f.result() for name, f in futs.items()}


@pytest.mark.parametrize("name", list(SLIPS))
def test_planted_slip_fails_a_pin(outcomes, name):
    code, detail = outcomes[name]
    assert code != "missing", f"the oracle no longer contains {detail!r}: restate this slip"
    # pytest exit status 1: tests ran and at least one failed (0 would mean the slip went unnoticed)
    assert code == 1, f"slip {name!r} left every pin green (exit {code}):\n{detail}"

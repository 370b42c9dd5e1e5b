"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and runs the pin suite against that
build: the suite must fail.  The mistakes are the ones a transcription of the
pages could plausibly make: a dropped or misplaced term of the recurrence, a
wrong sign, an off-by-one grid, a transposed group index, the wrong rounding
rule or the wrong read point of the output.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssq_oracle.c")

MUTATIONS = {
    "z_sign": ("z = (float)rint(-(double)lo * (double)inv) + 0.0f;",
               "z = (float)rint((double)lo * (double)inv) + 0.0f;"),
    "asym_levels_2b": ("return (float)((1 << b) - 1);", "return (float)(1 << b);"),
    "sym_levels_2b1": ("return (float)((1 << (b - 1)) - 1);",
                       "return (float)(1 << (b - 1));"),
    "no_dt_on_input": ("const float dtx = dt[h] * x[r];", "const float dtx = x[r];"),
    "decay_not_exp": ("double e = exp((double)dA);", "double e = 1.0 + (double)dA;"),
    "group_map": ("const int g = h / heads_per_group;",
                  "const int g = h % G;"),
    "round_half_away": ("float r = (float)rint(p);", "float r = (float)round(p);"),
    "y_before_rounding": ("acc += (double)Cg[n] * (double)stored[n];",
                          "acc += (double)Cg[n] * (double)sn[n];"),
    "no_skip_term": ("acc += (double)D[h] * (double)x[r];", "acc += 0.0;"),
    "no_clamp": ("if (c > qm) c = qm;\n        }", "}"),
    "truncate": ("float r = (float)rint(p);", "float r = (float)trunc(p);"),
    "deq_drop_zero": ("float d = (float)q[n] - zero;", "float d = (float)q[n];"),
    "swap_B_C": ("float w = dtx * Bg[n];", "float w = dtx * Cg[n];"),
    "constant_row_step": ("if (delta == 0.0f) delta = fabsf(lo);",
                          "if (delta == 0.0f) delta = 1.0f;"),
    "sr_ignores_draw": ("const double k = floor(p + (double)u16[n] / 65536.0);",
                        "const double k = floor(p + 0.5);"),
    "sr_no_low_clamp": ("            if (c < 0.0f) c = 0.0f;\n", ""),
    "diag_err_sign": ("const float e = deq[n] - sn[n];", "const float e = sn[n] - deq[n];"),
    "diag_rev_same_sign": ("(w[n] > 0.0f && inc < 0.0f) || (w[n] < 0.0f && inc > 0.0f)",
                           "(w[n] > 0.0f && inc > 0.0f) || (w[n] < 0.0f && inc < 0.0f)"),
    "diag_rev_error_only": ("const float inc = e + w[n];", "const float inc = e;"),
    "diag_signal_before_update": ("signal += (double)Cg[n] * (double)sn[n];",
                                  "signal += (double)Cg[n] * (double)s[n];"),
    "damp_hadamard_sign": ("return (__builtin_popcount((unsigned)(a & b)) & 1) ? -1 : 1;",
                           "return (__builtin_popcount((unsigned)(a | b)) & 1) ? -1 : 1;"),
    "damp_y_no_inverse_scale": ("acc /= (double)P;", "acc /= 1.0;"),
    "damp_fwht_butterfly_sign": ("                a[i + h] = x - y;", "                a[i + h] = y - x;"),
    "damp_fwht_skips_last_stage": ("for (int h = 1; h < P; h *= 2)", "for (int h = 1; 2 * h < P; h *= 2)"),
    "damp_input_not_rotated": ("const float dtx = dt[h] * xr[k];",
                               "const float dtx = dt[h] * x[(size_t)h * P + k];"),
    "damp_B_by_position": ("const float b = B[(size_t)g * N + ch[m]];",
                           "const float b = B[(size_t)g * N + m];"),
    "damp_protected_not_fp16": ("hi[(size_t)m * P + k] = oref_fp16_round(t[(size_t)m * P + k]);",
                                "hi[(size_t)m * P + k] = t[(size_t)m * P + k];"),
    "philox_round_multiplier": ("(uint64_t)0xD2511F53u * (uint64_t)c0",
                                "(uint64_t)0xD2511F57u * (uint64_t)c0"),
    "philox_weyl_constant": ("k1 += 0xBB67AE85u;", "k1 += 0xBB67AE87u;"),
    "philox_nine_rounds": ("for (int round = 0; round < 10; ++round)",
                           "for (int round = 0; round < 9; ++round)"),
    "philox_output_words_swapped": ("out[0] = c0; out[1] = c1;", "out[0] = c1; out[1] = c0;"),
    "philox_key_words_swapped": ("const uint32_t key[2] = {(uint32_t)r->seed, (uint32_t)(r->seed >> 32)};",
                                 "const uint32_t key[2] = {(uint32_t)(r->seed >> 32), (uint32_t)r->seed};"),
    "sr_draw_other_half": ("return (out[(n % 8) / 2] >> (16 * (n % 2))) & 0xFFFFu;",
                           "return (out[(n % 8) / 2] >> (16 * (1 - n % 2))) & 0xFFFFu;"),
    "decode_batch_layer0_decay": ("dt + lb * H, A + l * H, D + l * H,",
                                  "dt + lb * H, A, D + l * H,"),
    "damp_y_before_store": ("        /* readout from the stored state, rotated back */\n"
                            "        damp_load_head(c, hi, q, dl, z, t);\n",
                            "        /* readout from the stored state, rotated back */\n"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {name}"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "ssq_oracle.c")
        open(c, "w").write(mutated)
        subprocess.check_call(["cp", os.path.join(ROOT, "oracle", "ssq_oracle.h"), d])
        so = os.path.join(d, "liboref_mut.so")
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-std=c11",
                               "-shared", "-fPIC", "-o", so, c, "-lm"])
        env = dict(os.environ, SSQ_ORACLE_LIB=so)
        r = subprocess.run(
            [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
             os.path.join(ROOT, "tests", "test_oracle_pins.py"),
             os.path.join(ROOT, "tests", "test_oracle_damp.py"),
             os.path.join(ROOT, "tests", "test_oracle_philox.py")],
            cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"

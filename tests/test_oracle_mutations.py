"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of moe_oracle.c (on the CPU), builds
it into a temporary library and runs the pin suite against it; the suite must
fail. The committed oracle itself is untouched.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTATIONS = {
    "silu_on_up_operand": ("return g * sigmoid(g) * u;", "return u * sigmoid(u) * g;"),
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    "no_renormalisation": ("w[j] = scale * order[j].s / sel_sum;", "w[j] = scale * order[j].s;"),
    "tie_break_to_higher_index": ("return (a->e < b->e) ? -1 : (a->e > b->e);",
                                  "return (a->e > b->e) ? -1 : (a->e < b->e);"),
    "down_weight_transposed": ("acc += hh[f] * weight_at(wd, s_d, e, d, F, i, f);",
                               "acc += hh[f] * weight_at(wd, s_d, e, F, d, f, i);"),
    "gate_and_up_rows_swapped": ("g += xc * weight_at(wgu, s_gu, e, 2L * F, d, f, c);",
                                 "g += xc * weight_at(wgu, s_gu, e, 2L * F, d, (long)F + f, c);"),
    "combine_drops_weight": ("a += w[j] * y[(long)j * d + i];", "a += y[(long)j * d + i];"),
    "rounding_ties_down": ("return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "return fl;"),
    "bias_dropped": ("logit += (double)gate_bias[e];", "logit += 0.0 * gate_bias[e];"),
    "fp8_scale_dropped": ("* (double)scales[e * rows + r];", "* 1.0;"),
    "e4m3_subnormal_exponent": ("v = ldexp((double)mant / 8.0, -6);", "v = ldexp((double)mant / 8.0, -7);"),
    "gap_wrong_neighbour": ("order[k - 1].v - order[k].v", "order[0].v - order[k].v"),
    "rank_by_rounded_score": ("order[e].key = score_bias ? order[e].v : logit;",
                              "order[e].key = order[e].v;"),
    "score_bias_dropped": ("order[e].s + (double)score_bias[e]", "order[e].s"),
    "score_bias_in_the_weights": ("sel_sum += order[j].s;", "sel_sum += order[j].key;"),
    "shared_expert_dropped": ("a += y_shared[i];", "a += 0.0 * y_shared[i];"),
    "shared_expert_scaled": ("a += y_shared[i];", "a += 2.826 * y_shared[i];"),
    "route_norm_not_normalising": ("xr[c] = xr[c] * inv * (double)norm_w[c];",
                                   "xr[c] = xr[c] * (double)norm_w[c];"),
    "route_norm_weight_dropped": ("xr[c] = xr[c] * inv * (double)norm_w[c];", "xr[c] = xr[c] * inv;"),
    "route_norm_eps_outside_root": ("inv = 1.0 / sqrt(ms / d + norm_eps);",
                                    "inv = 1.0 / (sqrt(ms / d) + norm_eps);"),
    "sqrt_softplus_without_root": ("return score_fn == 1 ? sqrt(softplus(z)) : sigmoid(z);",
                                   "return score_fn == 1 ? softplus(z) : sigmoid(z);"),
    "e2m1_exponent_bias": ("ldexp(1.0 + 0.5 * mant, ex - 1)", "ldexp(1.0 + 0.5 * mant, ex - 2)"),
    "e8m0_bias": ("ldexp(1.0, (int)b - 127)", "ldexp(1.0, (int)b - 128)"),
    "fp4_nibble_order": ("(off & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF)",
                         "(off & 1) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4)"),
    "fp4_block_size": ("(cols / 32) + c / 32]", "(cols / 32) + c / 64]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_fail_on_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mutated = tmp_path / "moe_oracle_mutated.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmoe_oracle_mutated.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib),
                    str(mutated), "-lm"], check=True)
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"pins did not catch {name}:\n{res.stdout[-2000:]}"

"""Plant plausible mistakes in copies of the oracle and check the pins catch them.

Each mutation is a one-line change to rpk_oracle.c (a flipped sign, a dropped
term, a wrong index); the copy is compiled on the CPU into a temporary
library and the pin and brute-force suites are run against it in a child
process. Every mutation must make them fail.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rpk_oracle.c")

MUTATIONS = {
    "rotation_sign": ("out[base + i1] = a * c - bb * s;", "out[base + i1] = a * c + bb * s;"),
    "pairing_swapped": ("int i1 = interleaved ? 2 * j : j;", "int i1 = interleaved ? j : 2 * j;"),
    "frequency_exponent": ("pow(base, -2.0 * (double)j / (double)rotary_dim)",
                           "pow(base, -(double)j / (double)rotary_dim)"),
    "implicit_position": ("if (!position_ids) pos = cache_lens[b] + i;",
                          "if (!position_ids) pos = i;"),
    "mrope_section_edge": ("if (j < acc) return s;", "if (j <= acc) return s;"),
    "scale_dropped": ("double s = J->scale * acc;", "double s = acc;"),
    "gqa_mapping": ("int kvh = h / group;", "int kvh = h % J->n_kv_heads;"),
    "window_off_by_one": ("int64_t l = window > 0 ? p - (window - 1) : 0;",
                          "int64_t l = window > 0 ? p - window : 0;"),
    "query_alignment": ("int64_t p = (int64_t)r + k_len - q_len;", "int64_t p = (int64_t)r;"),
    "rounding_ties_away": ("double r = rint(a / ulp) * ulp;",
                           "double r = floor(a / ulp + 0.5) * ulp;"),
    "running_sum_not_rescaled": ("*l = *l * alpha + p;", "*l = *l + p;"),
    "slot_row": ("int32_t row = slot % page_size;", "int32_t row = (slot + 1) % page_size;"),
    "value_weight_unnormalised": ("double wj = w[i++] / den;", "double wj = w[i++];"),
    "visible_window_off_by_one": ("return j >= pos - (window - 1) || j < sinks;",
                                  "return j >= pos - window || j < sinks;"),
    "visible_alignment": ("int64_t pos = (int64_t)r + k_len - q_len;", "int64_t pos = (int64_t)r;"),
    "sinks_one_too_many": ("return j >= pos - (window - 1) || j < sinks;",
                           "return j >= pos - (window - 1) || j <= sinks;"),
    "sinks_not_causal": ("if (j < 0 || j >= k_len || j > pos) return 0;",
                         "if (j < 0 || j >= k_len || (j > pos && j >= sinks)) return 0;"),
    "p_rope_denominator": ("double omega = pow(base, -2.0 * (double)j / (double)head_dim);",
                           "double omega = pow(base, -2.0 * (double)j / (2.0 * rotated_pairs));"),
    "p_rope_tail_rotated": ("      if (j < rotated_pairs) {", "      if (j <= rotated_pairs) {"),
    "lse_log_base": ("if (lse) *lse = m + log(den);", "if (lse) *lse = m + log2(den);"),
    "lse_max_dropped": ("if (lse) *lse = m + log(den);", "if (lse) *lse = log(den);"),
    "e4m3_exponent_bias": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_ties_away": ("double units = rint(a / ulp);", "double units = floor(a / ulp + 0.5);"),
    "e4m3_no_saturation": ("if (a >= 448.0) return sign | 0x7E;",
                           "if (a >= 480.0) return sign | 0x7E;"),
    "e4m3_key_scale_multiplied": ("rpko_f64_to_e4m3(k_rot[src + c] / (double)k_scale[kh]);",
                                  "rpko_f64_to_e4m3(k_rot[src + c] * (double)k_scale[kh]);"),
    "e4m3_slot_row": ("int32_t row = slot - pi * page_size;",
                      "int32_t row = (slot + 1) % page_size;"),
    "backward_delta_dropped": ("double ds = p[i] * (dp[i] - D);", "double ds = p[i] * dp[i];"),
    "backward_key_scale_dropped": ("d_k[base[i] + c] += scale * ds * load_elt(q, dtype, qb + c);",
                                   "d_k[base[i] + c] += ds * load_elt(q, dtype, qb + c);"),
    "backward_value_weight_dropped": ("d_v[base[i] + c] += p[i] * load_elt(d_out, dtype, qb + c);",
                                      "d_v[base[i] + c] += load_elt(d_out, dtype, qb + c);"),
    "e4m3_read_scale_dropped": ("return rpko_e4m3_to_f64(((const uint8_t*)pool)[idx]) * (double)scale[kvh];",
                                "return rpko_e4m3_to_f64(((const uint8_t*)pool)[idx]);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mutated = tmp_path / "rpk_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "librpk_oracle_mut.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", str(mutated),
                    "-o", str(so), "-lm"], check=True)
    env = dict(os.environ, RPK_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_bruteforce.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutation {name} survived the pins:\n{r.stdout[-2000:]}"

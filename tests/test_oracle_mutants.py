"""Planted mistakes: each mutant is a copy of the oracle's C source with one plausible
error (a dropped term, a wrong sign or index, an off-by-one).  The pins in
test_oracle_pins.py must reject every one of them.  CPU only."""
import os
import subprocess
import sys
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "mla_oracle.c")

MUTANTS = {
    "dropped_softmax_scale": ("s_buf[t] = softmax_scale * descale_q * acc;",
                              "s_buf[t] = descale_q * acc;"),
    "causal_off_by_one": ("int64_t lim = causal ? L - q_len + i + 1 : L;",
                          "int64_t lim = causal ? L - q_len + i : L;"),
    "value_columns_shifted": ("o[d] += w * vd;", "o[d] += w * (d + 1 < dv ? vd : 0.0);"),
    "page_of_wrong_position": ("[req_pool_indices[b] * r2t_stride + p * page_size]",
                               "[req_pool_indices[b] * r2t_stride + p]"),
    "planner_zero_block_piece": ("if (budget - fixed_overhead > 0) {",
                                 "if (budget - fixed_overhead >= 0) {"),
    "e4m3_exponent_bias": ("v = ldexp((double)(8 + m), e - 10);",
                           "v = ldexp((double)(8 + m), e - 9);"),
    "lse_without_max": ("double l = m + log(sum);\n    for (int64_t d = 0; d < dv; ++d) o[d] = 0.0;",
                        "double l = log(sum);\n    for (int64_t d = 0; d < dv; ++d) o[d] = 0.0;"),
    "merge_weight_uses_max": ("double w = exp(lse_parts[k] - l);",
                              "double w = exp(lse_parts[k] - m);"),
    "fp8_query_neighbours_swapped": ("qd[d] = q_is_fp8 ? e4m3_bits_to_double(((const uint8_t*)q_row)[d])",
                                     "qd[d] = q_is_fp8 ? e4m3_bits_to_double(((const uint8_t*)q_row)[d ^ 1])"),
    "descale_k_dropped": ("? fp8_bits_to_double(kv[slot * dq + d], kv_format) * descale_k\n                                  : bf16_bits_to_double(((const uint16_t*)kv)[slot * dq + d]);\n            acc",
                          "? fp8_bits_to_double(kv[slot * dq + d], kv_format)\n                                  : bf16_bits_to_double(((const uint16_t*)kv)[slot * dq + d]);\n            acc"),
    "e5m2_exponent_bias": ("v = ldexp((double)(4 + m), e - 17);", "v = ldexp((double)(4 + m), e - 16);"),
    "quantize_ties_away_from_zero": ("if (err < best_err || (err == best_err && (code & 1) == 0)) {",
                                     "if (err < best_err || (err == best_err && code > best)) {"),
    "set_kv_slot_ignored": ("int64_t slot = cache_loc[i];", "int64_t slot = i;"),
    "set_kv_scale_multiplied": ("if (has_scale) x = x / k_scale;", "if (has_scale) x = x * k_scale;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    with tempfile.TemporaryDirectory() as tmp:
        c_path = os.path.join(tmp, "mutant.c")
        so_path = os.path.join(tmp, "libmutant.so")
        open(c_path, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so_path,
                        c_path, "-lm"], check=True)
        env = dict(os.environ, MLA_ORACLE_LIB_OVERRIDE=so_path)
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(HERE, "test_oracle_pins.py")],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"pins accepted the planted mistake {name}:\n{r.stdout[-2000:]}"

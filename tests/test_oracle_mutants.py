"""The oracle's pins must reject plausible mistakes (CPU only).

Each case plants one mistake in a copy of oracle/moe_oracle.c, builds it, and
runs the pin suite against that build in a fresh process: the suite has to fail.
"""
import os
import subprocess
import sys

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "tie_to_higher_index": ("if (best < 0 || ranks_above(z[e], z[best])) best = e;",
                            "if (best < 0 || !ranks_above(z[best], z[e])) best = e;"),
    "nan_not_ranked_first": ("    if (isnan(a)) return 1;", "    if (isnan(a)) return 0;"),
    "nan_compared_as_number": ("    if (isnan(b)) return 0;\n    if (isnan(a)) return 1;\n",
                               ""),
    "weights_not_shifted": ("(float)(exp((double)z[ids[(int64_t)t * k + j]] - zmax) / denom)",
                            "(float)(exp((double)z[ids[(int64_t)t * k + j]]) / denom)"),
    "capacity_off_by_one": ("if (capacity <= 0 || p < capacity) {",
                            "if (capacity <= 0 || p <= capacity) {"),
    "inclusive_offsets": ("        offsets[e] = total;\n        total += kept[e];",
                          "        total += kept[e];\n        offsets[e] = total;"),
    "bias_ignored": ("float b = bias ? bias[e] : 0.0f;", "float b = 0.0f;"),
    "w1_transposed": ("load_elem(W1, dtype, w1base + (int64_t)f * d + c)",
                      "load_elem(W1, dtype, w1base + (int64_t)c * F + f)"),
    "relu_missing": ("double r = acc > 0.0 ? acc : 0.0;", "double r = acc;"),
    "h_not_rounded": ("h[f] = bf16_bits_to_double(double_to_bf16_bits(r));", "h[f] = r;"),
    "h_fp32_not_rounded": ("h[f] = (double)(float)r;", "h[f] = r;"),
    "w2_wrong_expert": ("w2base = (int64_t)e * d * F;", "w2base = 0;"),
    "combine_first_weight_only": ("double wj = (double)w[(int64_t)t * k + j];",
                                  "double wj = (double)w[(int64_t)t * k];"),
    "dispatch_wrong_token": ("int t = row_slot[row] / k;", "int t = row_slot[row] % T;"),
    "gate_transposed": ("*\n                       load_elem(Wg, dtype, (int64_t)e * d + c);",
                        "*\n                       load_elem(Wg, dtype, (int64_t)c * E + e);"),
    "window_not_clamped": ("int64_t n = step + 1 < W ? step + 1 : W;", "int64_t n = W;"),
    "hot_tie_to_higher": ("if (best < 0 || sum[e] > sum[best]) best = e;",
                          "if (best < 0 || sum[e] >= sum[best]) best = e;"),
    "bf16_double_rounding": ("double a = fabs(v);", "double a = (double)(float)fabs(v);"),
    "bf16_ties_away": ("double r = rint(ldexp(a, -q));", "double r = round(ldexp(a, -q));"),
    "corr_transposed": ("C[(int64_t)i * E + h] += 1;", "C[(int64_t)h * E + i] += 1;"),
    "corr_first_choice_only": ("for (int b = 0; b < k_next; ++b) {",
                               "for (int b = 0; b < 1; ++b) {"),
    "forecast_no_k_prev": ("((double)s * (double)k_prev)", "((double)s)"),
    "aux_bias_ignored": ("float z = logits[(int64_t)t * E + e] + (bias ? bias[e] : 0.0f);",
                         "float z = logits[(int64_t)t * E + e];"),
    "aux_f_not_over_k": ("(double)counts[e] / ((double)T * (double)k)",
                         "(double)counts[e] / (double)T"),
    "aux_unnormalised_softmax": ("for (int e = 0; e < E; ++e) P[e] += ex[e] / D;",
                                 "for (int e = 0; e < E; ++e) P[e] += ex[e];"),
    "bwd_no_relu_mask": ("if (load_elem(H, dtype, (int64_t)r * F + f) > 0.0)", "if (1)"),
    "bwd_w1_transposed": ("acc += g[f] * load_elem(W1, dtype, w1b + (int64_t)f * d + c);",
                          "acc += g[f] * load_elem(W1, dtype, w1b + (int64_t)c * F + f);"),
    "bwd_route_no_centering": ("((double)dw[(int64_t)t * k + j] - s)",
                               "((double)dw[(int64_t)t * k + j])"),
    "bwd_dispatch_first_slot": ("if (row >= 0) acc += load_elem(dXp",
                                "if (row >= 0 && j == 0) acc += load_elem(dXp"),
    "bwd_combine_unweighted": ("store_elem(dYp, dtype, (int64_t)row * d + o, (double)w[s] * g);",
                               "store_elem(dYp, dtype, (int64_t)row * d + o, g);"),
    "bwd_gate_wrong_operand": (
        "acc += (double)dlogits[(int64_t)t * E + e] * load_elem(x, dtype, (int64_t)t * d + c);",
        "acc += (double)dlogits[(int64_t)t * E + e] * load_elem(Wg, dtype, (int64_t)e * d + c);"),
    "bwd_relu_mask_at_zero": ("if (load_elem(H, dtype, (int64_t)r * F + f) > 0.0)",
                              "if (load_elem(H, dtype, (int64_t)r * F + f) >= 0.0)"),
    "bwd_dw2_from_dh": ("load_elem(H, dtype, (int64_t)r * F + f);",
                        "load_elem(dH, dtype, (int64_t)r * F + f);"),
    "bwd_dbias_dropped": ("db[e] += dz;", "(void)dz;"),
    "bwd_route_first_slot_only": (
        "for (int i = 0; i < k; ++i) s += (double)w[(int64_t)t * k + i] * (double)dw[(int64_t)t * k + i];",
        "for (int i = 0; i < 1; ++i) s += (double)w[(int64_t)t * k + i] * (double)dw[(int64_t)t * k + i];"),
    "bwd_gate_dx_overwritten": ("double acc = load_elem(dx, dtype, (int64_t)t * d + c);",
                                "double acc = 0.0;"),
    "bwd_dw_token_row": ("dot += g * load_elem(Yp, dtype, (int64_t)row * d + o);",
                         "dot += g * load_elem(Yp, dtype, (int64_t)t * d + o);"),
    "combine_dropped_slot_read": ("                if (row < 0) continue;\n                double wj",
                                  "                if (row < 0) row = 0;\n                double wj"),
    "forecast_column_sum": ("a += q[i] * (double)C[(int64_t)i * E + h];",
                            "a += q[i] * (double)C[(int64_t)h * E + i];"),
}


# Mutants inside the loops the OpenMP build runs in parallel, planted again in
# that build (the pins then run on four threads).
PARALLEL_LOOP_MUTANTS = ["w1_transposed", "relu_missing", "h_not_rounded", "w2_wrong_expert",
                         "combine_first_weight_only", "combine_dropped_slot_read",
                         "dispatch_wrong_token", "gate_transposed"]
CASES = [(n, False) for n in sorted(MUTANTS)] + [(n, True) for n in PARALLEL_LOOP_MUTANTS]


@pytest.mark.parametrize("name,parallel", CASES)
def test_pins_reject_mutant(name, parallel, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "moe_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", *(["-fopenmp"] if parallel else []), "-shared", "-o",
                           str(lib), str(mutated), "-lm"])
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib), OMP_NUM_THREADS="4")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                          os.path.join(ROOT, "tests", "test_oracle_backward.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode != 0, f"pins accepted the mutant {name}:\n{res.stdout[-2000:]}"

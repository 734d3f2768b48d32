"""The pins must catch plausible mistakes: each case below compiles a copy of the oracle
with one planted slip (CPU only, in a temporary directory) and runs the pin suite
against it in a subprocess; the suite has to fail for every mutant."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "drop_up_projection": ("h[n] = silu(g) * u;", "h[n] = silu(g);"),
    "silu_sign": ("return z * sigmoid(z);", "return z * sigmoid(-z);"),
    "up_reads_gate_rows": ("w_gu + (size_t)(f + n) * D", "w_gu + (size_t)n * D"),
    "down_transposed": ("s += bf16_to_double(row[n]) * h[n];",
                        "s += bf16_to_double(w_d[(size_t)n * D + d]) * h[n];"),
    "drop_routing_weight": ("acc[d] += a * s;", "acc[d] += s;"),
    "no_renormalisation": ("double a = p[idx[(size_t)t * K + k]] / sel_sum;",
                           "double a = p[idx[(size_t)t * K + k]];"),
    "ties_to_higher_index": ("key[e] > key[best]", "key[e] >= key[best]"),
    "selection_bias_in_weights": ("sel_sum += p[best];", "sel_sum += key[best];"),
    "sigmoid_scores_as_softmax": ("for (int e = 0; e < E; ++e) p[e] = sigmoid(p[e]);",
                                  "for (int e = 0; e < E; ++e) p[e] = exp(p[e] - m);"),
    "bf16_weights_truncated": ("u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;",
                               "u = u & 0xFFFF0000u;"),
    "shared_gate_no_sigmoid": ("sgate[t] = w_sg ? sigmoid(dot_bf16(xt, w_sg, D)) : 0.0;",
                               "sgate[t] = w_sg ? dot_bf16(xt, w_sg, D) : 0.0;"),
    "drop_logit_bias": ("+ (bias ? bias[e] : 0.0)", "+ 0.0"),
    "drop_shared_expert": ("if (w_s_gu) expert_accumulate(xt, w_s_gu, w_s_d, D, f_s, sgate[t], h, acc);",
                           ";"),
    "unstable_permutation": ("sorted_token[row] = t;", "sorted_token[row] = T - 1 - t;"),
    "softmax_without_exp": ("p[e] = exp(p[e] - m);", "p[e] = 1.0 + (p[e] - m);"),
    "capacity_keeps_one_more": ("keep[(size_t)t * K + k] = seen[e] < C ? 1 : 0;",
                                "keep[(size_t)t * K + k] = seen[e] <= C ? 1 : 0;"),
    "capacity_floor_not_ceil": ("const double c = ceil(capacity_factor * (double)T * (double)K / (double)E);",
                                "const double c = floor(capacity_factor * (double)T * (double)K / (double)E);"),
    "capacity_counts_tokens": ("const double c = ceil(capacity_factor * (double)T * (double)K / (double)E);",
                               "const double c = ceil(capacity_factor * (double)T / (double)E);"),
    "capacity_ignores_minimum": ("if (cap < min_capacity) cap = min_capacity;", ";"),
    "capacity_keeps_latest": ("keep[(size_t)t * K + k] = seen[e] < C ? 1 : 0;",
                              "keep[(size_t)t * K + k] = seen[e] >= C ? 1 : 0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    find, repl = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    assert find in src, f"mutation site of {name} not found"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(find, repl, 1), encoding="utf-8")
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                           "-std=c11", str(mut), "-o", str(lib), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"

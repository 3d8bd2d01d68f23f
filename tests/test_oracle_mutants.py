"""Mutation check of the oracle pins.

Each mutant is a copy of ``oracle/fwpkm_oracle.c`` with one plausible mistake
planted (a flipped sign, a dropped factor, a swapped index ...), compiled on
the CPU.  The pin suite is run against it in a child process and must fail;
so must the hand-worked examples of ``tests/golden/`` on their own.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fwpkm_oracle.c")

MUTANTS = {
    "key_grad_sign": ("G1[c] += c1 * (q[c] - K1[c]);", "G1[c] += c1 * (K1[c] - q[c]);"),
    "second_half_uses_first_query_half": ("G2[c] += c2 * (q[dh + c] - K2[c]);",
                                          "G2[c] += c2 * (q[c] - K2[c]);"),
    "entropy_term_dropped": ("if (lam != 0.0) gam[r] +=", "if (0) gam[r] +="),
    "heads_summed_not_averaged": ("for (int c = 0; c < dv; ++c) y[c] /= Hd;", ""),
    "no_row_contribution_average": ("vr[c] -= eta * GV[u * dv + c] / Csum[u];",
                                    "vr[c] -= eta * GV[u * dv + c];"),
    "gate_not_weighting_mse": ("GV[u * dv + c] += (2.0 * om / Hd) * wr * ev[c];",
                               "GV[u * dv + c] += (2.0 / Hd) * wr * ev[c];"),
    "softmax_not_normalised": ("for (int r = 0; r < k; ++r) w[r] /= z;", ""),
    "slot_index_transposed": ("cand[a * k + b].idx = top1[a] * (int64_t)n + top2[b];",
                              "cand[a * k + b].idx = top2[b] * (int64_t)n + top1[a];"),
    "ties_by_index_desc": ("return (x->idx < y->idx) ? -1 : (x->idx > y->idx ? 1 : 0);",
                           "return (x->idx < y->idx) ? 1 : (x->idx > y->idx ? -1 : 0);"),
    "eps_dropped_from_score": ("s[i] = -log(eps + d);", "s[i] = -log(d + 1e-300);"),
    "marginal_not_normalised": ("for (int64_t u = 0; u < U; ++u) psum[u] /= (double)M;",
                                "for (int64_t u = 0; u < U; ++u) psum[u] /= (double)(M + 1);"),
    "distance_of_wrong_half_index": ("d1[m * k + r] = dd1[a_[r]];", "d1[m * k + r] = dd1[b_[r]];"),
    "mse_grad_factor_two_dropped": ("gam[r] = (2.0 * om / Hd) * dot;",
                                    "gam[r] = (1.0 * om / Hd) * dot;"),
    "count_divisor_is_the_weight": ("if (dm->variant & ORC_AGG_COUNT) Csum[u] = Cnt[u];", ""),
    "summed_heads_still_averaged": ("(dm->variant & ORC_HEADS_SUM) ? 1.0 : (double)H;",
                                    "(double)H;"),
    "keys_not_updated": ("if (ktouched[row])", "if (0)"),
    "dot_key_grad_of_the_first_half": ("G2[c] += dLds * q[dh + c];", "G2[c] += dLds * q[c];"),
    "dot_score_ignored_in_selection": ("orc_half_scores_dot(q + dh, K2, n, dh, s2);", ""),
}


def _fails(test_file, env) -> tuple:
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        os.path.join(ROOT, "tests", test_file)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode != 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not found exactly once"
    mut_c = tmp_path / "mutant.c"
    mut_c.write_text(src.replace(before, after))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-shared", "-fPIC", "-o",
                           str(so), str(mut_c), "-lm"])
    env = dict(os.environ, FWPKM_ORACLE_LIB=str(so), OMP_NUM_THREADS="2")
    failed, out = _fails("test_oracle_pins.py", env)
    assert failed, f"mutant {name} survived the pins:\n{out}"
    failed, out = _fails("test_golden.py", env)
    assert failed, f"mutant {name} survived the hand-worked examples:\n{out}"

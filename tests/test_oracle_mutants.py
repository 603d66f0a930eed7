"""Planted mistakes in a copy of the oracle must fail the pins.

Each mutant is the oracle's C source with one plausible mistake (a dropped
term, a wrong sign or index, a transposed operand, a wrong divisor, a wrong
tie-break). It is compiled into a temporary folder and the pin tests are run
against it in a subprocess; every mutant must make them fail. The oracle
itself is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "seer_oracle.c")

MUTANTS = {
    "pool_divides_by_block_size": [("pooled[d] /= (double)n;", "pooled[d] /= (double)blk;")],
    "w_k_transposed": [("acc += (double)W[(size_t)e * D + d] * pooled[d];",
                        "acc += (double)W[(size_t)d * dg + e] * pooled[d];")],
    "w_q_transposed": [("acc += (double)W[(size_t)e * D + d] * bf16_to_double(qh[d]);",
                        "acc += (double)W[(size_t)d * dg + e] * bf16_to_double(qh[d]);")],
    "gate_scale_dropped": [("s += sh * inv_sqrt_dg;", "s += sh;")],
    "heads_summed_not_averaged": [("*out = s / (double)G;", "*out = s;")],
    "gate_reads_next_block": [("const double* kp = kpool + ((size_t)row * NBmax + j) * dg;",
                               "const double* kp = kpool + ((size_t)row * NBmax + (j + 1 < NB ? j + 1 : j)) * dg;")],
    "last_block_not_forced": [("for (int j = 0; j < NB - 1; ++j) { cand[j].score",
                               "for (int j = 0; j < NB; ++j) { cand[j].score"),
                              ("qsort(cand, (size_t)(NB - 1),", "qsort(cand, (size_t)NB,"),
                              ("out[n++] = NB - 1;", "out[n++] = cand[kb - 1].index;"),
                              ("(size_t)(NB > 1 ? NB - 1 : 1)", "(size_t)(NB > 0 ? NB : 1)")],
    "tie_break_reversed": [("return (a->index < b->index) ? -1 : (a->index > b->index);",
                            "return (a->index > b->index) ? -1 : (a->index < b->index);")],
    "softmax_scale_dropped": [("z[i] = acc * scale;", "z[i] = acc;")],
    "lse_missing_max": [("lse[(size_t)b * Hq + hq] = m + log(denom);",
                         "lse[(size_t)b * Hq + hq] = log(denom);")],
    "attend_reads_past_length": [("const int t1 = (j * blk + blk < L) ? j * blk + blk : L;\n            for (int t",
                                  "const int t1 = j * blk + blk;\n            for (int t")],
    "merge_weight_sign": [("const double w = exp(lse_parts[s] - M);", "const double w = exp(M - lse_parts[s]);")],
    "block_mass_scale_dropped": [("z[t] = acc * scale;", "z[t] = acc;")],
    "block_mass_next_block": [("mh[t / blk] += exp(z[t] - m) / denom;",
                               "mh[(t + 1) / blk < NBmax ? (t + 1) / blk : t / blk] += exp(z[t] - m) / denom;")],
    "block_mass_ignores_length": [("L = L < 0 ? 0 : (L > Lmax ? Lmax : L);\n        double* z",
                                   "L = Lmax;\n        double* z")],
    "block_mass_lse_missing_max": [("const double lse_h = m + log(denom);", "const double lse_h = log(denom);")],
    "agg_max_takes_min": [("if (agg == 1) a = v > a ? v : a;", "if (agg == 1) a = v < a ? v : a;")],
    "agg_softmax_over_candidates_only": [("for (int j = 0; j < NB; ++j) den += exp(sh[(size_t)h * NB + j] - m);",
                                          "for (int j = 0; j < NB - 1; ++j) den += exp(sh[(size_t)h * NB + j] - m);")],
    "agg_mean_not_divided": [("out[j] = (agg == 1) ? a : a / (double)G;", "out[j] = a;")],
    "threshold_strict": [("if (s[j] >= threshold)", "if (s[j] > threshold)")],
    "prefill_not_causal": [("for (int u = j * blk; u < (j + 1) * blk && u <= t && u < L; ++u) tok[n++] = u;",
                            "for (int u = j * blk; u < (j + 1) * blk && u < L; ++u) tok[n++] = u;")],
    "prefill_w_q_transposed": [("acc += qbar[d] * (double)W[(size_t)e * D + d];",
                                "acc += qbar[d] * (double)W[(size_t)d * dg + e];")],
    "prefill_query_pool_summed": [("qbar[d] = acc / (double)(t1 - t0);", "qbar[d] = acc;")],
    "prefill_diagonal_not_forced": [("            out[n] = i;\n            *ns = n + 1;",
                                     "            out[n] = (i > 0 && n > 0) ? out[n - 1] : i;\n            *ns = n + 1;")],
    "value_row_of_wrong_head": [("const uint16_t* vt = v_cache + ((size_t)row * Lmax + tok[i]) * D;",
                                 "const uint16_t* vt = v_cache + ((size_t)(row ^ 1) * Lmax + tok[i]) * D;")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation site for {name} not found once: {old!r}"
        src = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "libmutant.so"
    c_path.write_text(src)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so_path),
                    str(c_path), "-lm"], check=True)
    env = dict(os.environ, SEER_ORACLE_LIB=str(so_path), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"

"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of the oracle's C source
(a dropped term, an off-by-one, a wrong index, a flipped sign, a swapped
operand), builds it, and runs the pin suite against that build.  The pins
must reject every mutant.  Mistakes are planted only in the oracle copy,
never in the CUDA library.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nsa_oracle.c")

MUTANTS = {
    "mean_divides_by_l_minus_1": ("round_store(sk / l, c->kv_round)",
                                  "round_store(sk / (l - 1), c->kv_round)"),
    "incomplete_block_visible": ("if (t < c->cmp_block - 1) return 0;\n  int n = (t - c->cmp_block + 1) / c->cmp_stride + 1;",
                                 "if (t < 0) return 0;\n  int n = t / c->cmp_stride + 1;"),
    "score_wrong_group": ("score_tok[(size_t)(h / G) * nc + j] += p_row[j];",
                          "score_tok[(size_t)(h % c->Hkv) * nc + j] += p_row[j];"),
    "tie_goes_to_higher_block": ("(sr == sb && cand[r] < cand[best])",
                                 "(sr == sb && cand[r] > cand[best])"),
    "first_block_not_forced": ("for (int i = 0; i < m; ++i) cand[i] = i + 1;",
                               "for (int i = 0; i < m; ++i) cand[i] = i + 1;\n  if (m > 0) cand[0] = 0;"),
    "sel_sees_next_token": ("if (p <= t && p < c->T) pos[n++] = p;",
                            "if (p <= t + 1 && p < c->T) pos[n++] = p;"),
    "window_one_too_long": ("int lo = t - c->window + 1;", "int lo = t - c->window;"),
    "lse_drops_max": ("*lse = mx + log(sum);", "*lse = log(sum);"),
    "bwd_delta_sign": ("double ds = p[s] * (dp - delta);", "double ds = p[s] * (dp + delta);"),
    "combine_swaps_gates": ("if (c->branch_mask & ORC_SWA) acc += g3[2] * ow[d];",
                            "if (c->branch_mask & ORC_SWA) acc += g3[1] * ow[d];"),
    "pool_bwd_not_spread": ("dk[KI(c, b, j * dstr + i, g) + d] += dkc[(size_t)j * D + d] / l;",
                            "dk[KI(c, b, j * dstr + i, g) + d] += dkc[(size_t)j * D + d];"),
    "dv_without_prob": ("dvrows[s][d] += p[s] * dO[d];", "dvrows[s][d] += dO[d];"),
    "dk_uses_key_not_query": ("dkrows[s][d] += scale * ds * qrow[d];",
                              "dkrows[s][d] += scale * ds * krows[s][d];"),
    "softmax_scale_dropped": ("logit[s] = scale * dot(qrow, krows[s], D);",
                              "logit[s] = dot(qrow, krows[s], D);"),
    "bf16_round_truncates": ("double r = nearbyint(ldexp(m, 8));", "double r = trunc(ldexp(m, 8));"),
    "gate_grad_reads_exact_outputs": ("    o_sel[i] = round_store(o_sel[i], c->o_round);\n",
                                      "    o_sel[i] = o_sel[i];\n"),
    "moba_gate_first_head_only": ("      acc += dot(q + QI(c, b, t, h), kc + CI(c, nc, b, j, g), D);",
                                  "      if (h == g * G) acc += dot(q + QI(c, b, t, h), kc + CI(c, nc, b, j, g), D);"),
    "moba_own_block_not_forced": ("  idx_row[n - 1] = cur;\n", "  idx_row[n - 1] = cand[n - 1];\n"),
    "moba_ties_to_higher_block": ("(gr == gb && cand[r] < cand[best])", "(gr == gb && cand[r] > cand[best])"),
    "mlp_ignores_stride": ("              sk += k[KI(c, b, j * dstr + i, g) + e] * wk[((size_t)i * D + e) * D + n];",
                           "              sk += k[KI(c, b, j * l + i, g) + e] * wk[((size_t)i * D + e) * D + n];"),
    "mlp_weight_transposed": ("              sv += v[KI(c, b, j * dstr + i, g) + e] * wv[((size_t)i * D + e) * D + n];",
                              "              sv += v[KI(c, b, j * dstr + i, g) + e] * wv[((size_t)i * D + n) * D + e];"),
    "mlp_bwd_drops_weight_grad_row": ("              dwk[((size_t)i * D + e) * D + n] += k[rowi] * gk;",
                                      "              dwk[((size_t)i * D + e) * D + n] += k[rowi] * gk * (i > 0);"),
    "cmp_bwd_kc_swaps_key_value_grads": ("      dkr[j] = dkc + CI(c, nc, b, j, g);\n      dvr[j] = dvc + CI(c, nc, b, j, g);",
                                         "      dkr[j] = dvc + CI(c, nc, b, j, g);\n      dvr[j] = dkc + CI(c, nc, b, j, g);"),
    "remap_overlap_off_by_one": ("if (clo < hi && chi > lo) acc += cmp_score_row[i];",
                                 "if (clo <= hi && chi > lo) acc += cmp_score_row[i];"),
    "remap_first_block_only": ("if (clo < hi && chi > lo) acc += cmp_score_row[i];",
                               "if (clo >= lo && clo < hi) { acc += cmp_score_row[i]; break; }"),
    "current_block_not_forced": ("idx_row[cnt++] = cur;", "idx_row[cnt++] = cur - 1;"),
    "dq_uses_query_not_key": ("dq[d] += scale * ds * krows[s][d];", "dq[d] += scale * ds * qrow[d];"),
    "softmax_not_normalised": ("double p = logit[s] / sum;", "double p = logit[s];"),
    "delta_uses_first_value_row": ("double delta = dot(dO, o, D);",
                                   "double delta = dot(dO, vrows[0], D);"),
    "pool_key_ignores_stride": ("sk += k[KI(c, b, j * dstr + i, g) + d];",
                                "sk += k[KI(c, b, j * l + i, g) + d];"),
    "window_excludes_query": ("for (int p = lo; p <= t; ++p) pos[n++] = p;",
                              "for (int p = lo; p < t; ++p) pos[n++] = p;"),
    "decode_reads_previous_row": ("b, L - 1, oc,", "b, L - 2, oc,"),
    "gate_bwd_ignores_branch_mask": ("dob[i][d] = on ? gates[(size_t)r * 3 + i] * dO[d] : 0.0;",
                                     "dob[i][d] = gates[(size_t)r * 3 + i] * dO[d];"),
    "dgates_scaled_by_gate": ("dgates[(size_t)r * 3 + i] = on ? dot(dO, ob[i], D) : 0.0;",
                              "dgates[(size_t)r * 3 + i] = on ? gates[(size_t)r * 3 + i] * dot(dO, ob[i], D) : 0.0;"),
    "moba_prefers_lowest_gate": ("    gate[j] = acc;", "    gate[j] = -acc;"),
    "mlp_bwd_row_grad_transposed": ("ak += wk[((size_t)i * D + e) * D + n] * gk;",
                                    "ak += wk[((size_t)i * D + n) * D + e] * gk;"),
    "mlp_bwd_row_grad_first_block_only": ("            dk[rowi] += ak;",
                                          "            if (j == 0) dk[rowi] += ak;"),
}


def _run_mutant(name: str, workdir: str) -> tuple:
    """Build the oracle with mutant `name` planted and run the pin suite on
    it; returns (pin-suite exit code, the end of its output)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return None, f"mutation site for {name} not found exactly once"
    mut = os.path.join(workdir, f"{name}.c")
    with open(mut, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(workdir, f"lib{name}.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib, mut,
                    "-lm"], check=True)
    env = dict(os.environ, NSA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(request, tmp_path_factory):
    """The selected mutants, run a few at a time (each pin run is one
    process with two OpenMP threads)."""
    names = sorted({item.callspec.params["name"] for item in request.session.items
                    if item.originalname == "test_pins_reject_mutant"})
    workdir = str(tmp_path_factory.mktemp("mutants"))
    workers = max(1, min(4, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {n: ex.submit(_run_mutant, n, workdir) for n in names}
        return {n: f.result() for n, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, mutant_results):
    code, out = mutant_results[name]
    assert code is not None, out
    assert code != 0, f"pins accepted mutant {name}:\n{out}"

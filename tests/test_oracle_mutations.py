"""The pins in ``test_oracle.py`` must be able to fail.

Each case plants one plausible mistake in a copy of ``oracle/la_oracle.c``
(on the CPU), builds it into a temporary shared object and runs the pin tests
against it in a subprocess; every mutant must make at least one pin fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "la_oracle.c")

MUTANTS = {
    # ELU+1
    "elu_eps_dropped": ("den += eps;", "den += 0.0 * eps;"),
    "elu_phi_missing_plus_one": ("x > 0.0 ? x + 1.0 : exp(x)", "x > 0.0 ? x : exp(x)"),
    "elu_query_feature_in_state": ("S[d * dv + j] += pk[d] * vt[j];", "S[d * dv + j] += pq[d] * vt[j];"),
    "elu_normaliser_not_updated": ("z[d] += pk[d];", "z[d] += 0.0 * pk[d];"),
    # GLA
    "gla_gate_on_columns": ("S[d * dv + j] = gt[d] * S[d * dv + j] + kt[d] * vt[j];",
                            "S[d * dv + j] = gt[j % dk] * S[d * dv + j] + kt[d] * vt[j];"),
    "gla_gate_on_new_term": ("S[d * dv + j] = gt[d] * S[d * dv + j] + kt[d] * vt[j];",
                             "S[d * dv + j] = gt[d] * (S[d * dv + j] + kt[d] * vt[j]);"),
    "gla_read_with_key": ("for (int64_t j = 0; j < dv; ++j) acc[j] += qt[d] * S[d * dv + j];\n            memcpy(o + IDX4(b, t, h, 0, T, H, dv), acc, sizeof(double) * (size_t)dv);\n        }\n        store_state(S_out, S, b, h, H, dk * dv);\n        free(S);\n    }\n}\n\n/* Gated delta",
                          "for (int64_t j = 0; j < dv; ++j) acc[j] += kt[d] * S[d * dv + j];\n            memcpy(o + IDX4(b, t, h, 0, T, H, dv), acc, sizeof(double) * (size_t)dv);\n        }\n        store_state(S_out, S, b, h, H, dk * dv);\n        free(S);\n    }\n}\n\n/* Gated delta"),
    # gated delta rule
    "gdn_correction_sign": ("a * (S[d * dv + j] - be * kt[d] * kS[j])", "a * (S[d * dv + j] + be * kt[d] * kS[j])"),
    "gdn_decay_skips_correction": ("a * (S[d * dv + j] - be * kt[d] * kS[j])", "(a * S[d * dv + j] - be * kt[d] * kS[j])"),
    "gdn_write_not_scaled_by_beta": ("+ be * kt[d] * vt[j];", "+ kt[d] * vt[j];"),
    "gdn_alpha_beta_swapped": ("const double a = alpha[IDX3(b, t, h, T, H)];\n            const double be = beta[IDX3(b, t, h, T, H)];",
                               "const double a = beta[IDX3(b, t, h, T, H)];\n            const double be = alpha[IDX3(b, t, h, T, H)];"),
    "gdn_prediction_transposed": ("for (int64_t j = 0; j < dv; ++j) kS[j] += kt[d] * S[d * dv + j];",
                                  "for (int64_t j = 0; j < dv; ++j) kS[j] += kt[j % dk] * S[d * dv + j];"),
    # KDA
    "kda_decay_on_columns": ("S[d * dv + j] *= at[d];", "S[d * dv + j] *= at[j % dk];"),
    "kda_decay_skipped": ("S[d * dv + j] *= at[d];", "S[d * dv + j] *= 1.0;"),
    "kda_residual_sign": ("(vt[j] - pred[j])", "(vt[j] + pred[j])"),
    "kda_write_not_scaled_by_beta": ("S[d * dv + j] += be * kt[d] * (vt[j] - pred[j]);",
                                     "S[d * dv + j] += kt[d] * (vt[j] - pred[j]);"),
    # output RMS normalisation
    "norm_eps_outside_root": ("1.0 / sqrt(ss / (double)dv + eps)", "1.0 / (sqrt(ss / (double)dv) + eps)"),
    "norm_sum_not_mean": ("1.0 / sqrt(ss / (double)dv + eps)", "1.0 / sqrt(ss + eps)"),
    "norm_weight_ignored": ("xr[j] * scale * (w ? w[j] : 1.0)", "xr[j] * scale"),
    "norm_over_all_rows": ("        double ss = 0.0;\n        for (int64_t j = 0; j < dv; ++j) ss += xr[j] * xr[j];",
                           "        static double ss = 0.0;\n        for (int64_t j = 0; j < dv; ++j) ss += xr[j] * xr[j];"),
    "norm_weight_per_row": ("xr[j] * scale * (w ? w[j] : 1.0)", "xr[j] * scale * (w ? w[r % dv] : 1.0)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    mutated = tmp_path / "la_oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", str(mutated), "-o", str(lib), "-lm"])
    env = dict(os.environ, LA_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"

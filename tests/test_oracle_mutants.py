"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pin suite catches every one of them: a pin that cannot fail pins nothing."""
import os

import pytest

import oracle
import oracle_pins as P

# (name, text in gdr_oracle.c, replacement)
MUTANTS = [
    ("delta_sign", "S[i * dv + n] += bk * (vt[n] - r[n]);", "S[i * dv + n] += bk * (vt[n] + r[n]);"),
    ("beta_dropped", "const double bk = bt * kt[i];", "const double bk = kt[i];"),
    ("group_index", "f[i] = exp(gt[(long)i * G / dk]);", "f[i] = exp(gt[0]);"),
    ("decay_sign", "f[i] = exp(gt[(long)i * G / dk]);", "f[i] = exp(-gt[(long)i * G / dk]);"),
    ("readout_wrong_vector", "ot[n] += S[i * dv + n] * qt[i];", "ot[n] += S[i * dv + n] * kt[i];"),
    ("chunk_E_no_beta", "E[t * dv + n] = bc[t] * acc;", "E[t * dv + n] = acc;"),
    ("chunk_L_strict", "L[t * Cl + j] = (j <= t) ? l : 0.0;", "L[t * Cl + j] = (j < t) ? l : 0.0;"),
    ("chunk_M_beta_on_row", "M[t * Cl + j] = (j < t) ? bc[j] * m : 0.0;",
     "M[t * Cl + j] = (j < t) ? bc[t] * m : 0.0;"),
    ("chunk_Khat_pivot", "Kh[t * dk + i] = kc[t * dk + i] * exp(LamC - Lam[t * dk + i]);",
     "Kh[t * dk + i] = kc[t * dk + i] * exp(Lam[t * dk + i]);"),
    ("chunk_F_missing", "double acc = F[i] * S[i * dv + n];", "double acc = S[i * dv + n];"),
    ("tril_inverse_sign", "acc -= N[t * n + j] * X[j * n + c];", "acc += N[t * n + j] * X[j * n + c];"),
    ("neumann_odd_sign", "const double sgn = (p % 2 == 0) ? 1.0 : -1.0;",
     "const double sgn = 1.0;"),
    ("neumann_mask_off_by_one", "if (i - j < p)\n                    T1[i * n + j] = 0.0;",
     "if (i - j <= p)\n                    T1[i * n + j] = 0.0;"),
    ("neumann_resid_sign", "X[e] += T1[e];", "X[e] -= T1[e];"),
    ("lam_not_cumulative", "acc += gc[(long)t * G + (long)i * G / dk];",
     "acc = gc[(long)t * G + (long)i * G / dk];"),
    ("neumann1_sign", "X[e] = Dinv[e] - X[e];", "X[e] = Dinv[e] + X[e];"),
    ("epilogue_gate_sign", "const double gate = 1.0 / (1.0 + exp(-z[(size_t)r * dv + i]));",
     "const double gate = 1.0 / (1.0 + exp(z[(size_t)r * dv + i]));"),
    ("gva_mapping_recurrent", "hk = hv / R;\n        double *S = (double *)malloc",
     "hk = hv % Hk;\n        double *S = (double *)malloc"),
    ("gva_mapping_chunked", "hk = hv / R;\n        const long kh = b * Hk + hk;\n        const size_t CC",
     "hk = hv % Hk;\n        const long kh = b * Hk + hk;\n        const size_t CC"),
    ("epilogue_eps_outside_root", "const double inv = 1.0 / sqrt(ss / dv + eps);",
     "const double inv = 1.0 / (sqrt(ss / dv) + eps);"),
    ("epilogue_gate_index", "const double gate = 1.0 / (1.0 + exp(-z[(size_t)r * dv + i]));",
     "const double gate = 1.0 / (1.0 + exp(-z[(size_t)r * dv]));"),
    ("momentum_velocity_sign", "Z[i * dv + n] = mk * Z[i * dv + n] + (S[i * dv + n] - fs);",
     "Z[i * dv + n] = mk * Z[i * dv + n] + (S[i * dv + n] + fs);"),
    ("momentum_no_carry", "Z[i * dv + n] = mk * Z[i * dv + n] + (S[i * dv + n] - fs);",
     "Z[i * dv + n] = (S[i * dv + n] - fs);"),
    ("grad_decay_group", "f[i] = exp(gt[grp]);", "f[i] = exp(gt[0]);"),
    ("grad_dk_drops_state_term", "dkt[i] += bt * a1 - a2;", "dkt[i] += bt * a1;"),
    ("grad_dS_misses_write", "const double dsp = dS[i * dv + n] - kt[i] * du[n];",
     "const double dsp = dS[i * dv + n];"),
    ("grad_dg_no_factor", "dgt[(long)i * G / dk] += df * f[i];", "dgt[(long)i * G / dk] += df;"),
    ("grad_dq_old_state", "acc += Snew[i * dv + n] * dot[n];", "acc += Sprev[i * dv + n] * dot[n];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdr_oracle.c")).read()
    assert src.count(old) == 1, "mutation site not unique: " + name
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(mut_src), out=str(tmp_path / "mutant.so"))
    with oracle.using_library(lib):
        failed = P.failing_pins()
    assert failed, "no pin caught mutant " + name

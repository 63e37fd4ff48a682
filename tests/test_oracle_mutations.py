"""Plant plausible mistakes in copies of the oracle and check that the pins catch
every one: each mutant is compiled on the host from an edited copy of
oracle/gdr_oracle.c, and at least one check of tests/oracle_pins.py must fail
on it.  Nothing here touches a GPU."""
import os
import shutil

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "gdr_oracle.c")

# (name, exact text in the oracle, replacement)
MUTANTS = [
    ("no_decay", "for (int i = 0; i < dv * dk; ++i) S[i] *= alpha;", ""),
    ("delta_sign", "double delta = beta * (vt[i] - u[i]);", "double delta = beta * (vt[i] + u[i]);"),
    ("beta_dropped", "double delta = beta * (vt[i] - u[i]);", "double delta = (vt[i] - u[i]);"),
    ("readout_transposed", "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qh[j];\n            ot[i] = acc;",
     "for (int j = 0; j < dk; ++j) acc += S[j * dk + i] * qh[j];\n            ot[i] = acc;"),
    ("readout_with_k", "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qh[j];\n            ot[i] = acc;",
     "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kh[j];\n            ot[i] = acc;"),
    ("retrieval_transposed", "for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kh[j];\n            u[i] = acc;",
     "for (int j = 0; j < dk; ++j) acc += S[j * dk + i] * kh[j];\n            u[i] = acc;"),
    ("gva_modulo", "return (int)(((int64_t)hv * p->H_k) / p->H_v);", "return hv % p->H_k;"),
    ("l2_no_sqrt", "double f = on ? mult / sqrt(ss + eps) : mult;", "double f = on ? mult / (ss + eps) : mult;"),
    ("scale_on_k", "p->scale, out);\n}\n\nstatic void load_k_hat", "1.0, out);\n}\n\nstatic void load_k_hat"),
    ("rms_no_mean", "    ms /= n;\n", ""),
    ("gate_sigmoid_only", "double silu = z[i] / (1.0 + exp(-z[i]));", "double silu = 1.0 / (1.0 + exp(-z[i]));"),
    ("eps_outside_root", "double r = 1.0 / sqrt(ms + eps);", "double r = 1.0 / sqrt(ms) + eps;"),
    ("chunk_decay_off_by_one", "for (int j = s + 1; j <= r; ++j) d *= alpha[j];", "for (int j = s; j <= r; ++j) d *= alpha[j];"),
    ("chunk_solve_sign", "for (int s = c; s < r; ++s) acc -= A[r * C + s] * T[s * C + c];",
     "for (int s = c; s < r; ++s) acc += A[r * C + s] * T[s * C + c];"),
    ("chunk_w_no_decay", "acc += T[r * C + s] * beta[s] * eg[s] * K[(size_t)s * dk + j];",
     "acc += T[r * C + s] * beta[s] * K[(size_t)s * dk + j];"),
    ("chunk_p_strict", "P[r * C + s] = (s <= r) ?", "P[r * C + s] = (s < r) ?"),
    ("chunk_state_no_decay", "double acc = eg[L - 1] * S[(size_t)i * dk + j];", "double acc = S[(size_t)i * dk + j];"),
    ("brute_sign", "a * ((i == j ? 1.0 : 0.0) - b * kh[s * dk + i] * kh[s * dk + j]);",
     "a * ((i == j ? 1.0 : 0.0) + b * kh[s * dk + i] * kh[s * dk + j]);"),
    ("brute_product_order", "for (int r = s + 1; r <= t; ++r) {", "for (int r = s; r <= t; ++r) {"),
    ("gate_softplus_mirrored", "fmax(x, 0.0) + log1p(exp(-fabs(x)))", "fmax(-x, 0.0) + log1p(exp(-fabs(x)))"),
    ("gate_alog_not_exponentiated", "g[i] = -exp(A_log[h]) * softplus;", "g[i] = -A_log[h] * softplus;"),
    ("gate_decay_positive", "g[i] = -exp(A_log[h]) * softplus;", "g[i] = exp(A_log[h]) * softplus;"),
    ("gate_bias_dropped", "const double x = a[i] + dt_bias[h];", "const double x = a[i];"),
    ("gate_beta_mirrored", "beta[i] = 1.0 / (1.0 + exp(-b[i]));", "beta[i] = 1.0 / (1.0 + exp(b[i]));"),
]


def test_mutations_are_well_formed():
    src = open(SRC).read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, f"mutation {name}: text must occur exactly once"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1
    mutated = tmp_path / "gdr_oracle.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / "liboracle_mutant.so")
    oracle.build(src=str(mutated), out=so, force=True, werror=False)
    lib = oracle.load(so)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"

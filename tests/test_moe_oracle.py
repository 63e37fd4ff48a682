"""The fp64 oracle of the routed-expert MoE block against its pins
(tests/moe_oracle_pins.py), and planted mistakes in copies of
oracle/moe_oracle.c that the pins must catch.  CPU only."""
import os

import pytest

import moe_oracle_pins
import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "moe_oracle.c")


@pytest.mark.parametrize("check", moe_oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_moe_pin(check):
    check(oracle.load())


# (name, exact text in the oracle, replacement)
MUTANTS = [
    ("no_renormalisation", "w[(size_t)t * K + k] = pt[idx[(size_t)t * K + k]] / sum;",
     "w[(size_t)t * K + k] = pt[idx[(size_t)t * K + k]];"),
    ("ties_to_higher_index", "if (!taken[e] && (best < 0 || pt[e] > pt[best])) best = e;",
     "if (!taken[e] && (best < 0 || pt[e] >= pt[best])) best = e;"),
    ("softmax_not_normalised", "for (int e = 0; e < E; ++e) pt[e] = exp(lg[e] - m) / z;",
     "for (int e = 0; e < E; ++e) pt[e] = exp(lg[e] - m);"),
    ("silu_as_sigmoid", "static double silu(double u) { return u / (1.0 + exp(-u)); }",
     "static double silu(double u) { return 1.0 / (1.0 + exp(-u)); }"),
    ("gate_up_swapped", "h[j] = silu(g) * u;", "h[j] = silu(u) * g;"),
    ("down_transposed", "for (int j = 0; j < I; ++j) s += wd[(size_t)i * I + j] * h[j];",
     "for (int j = 0; j < I; ++j) s += wd[(size_t)j * H + i] * h[j];"),
    ("shared_gate_sign", "1.0 / (1.0 + exp(-s))", "1.0 / (1.0 + exp(s))"),
    ("expert_off_by_one", "const size_t off = (size_t)e * I * H;",
     "const size_t off = (size_t)((e + 1) % p->n_exp) * I * H;"),
    ("weight_dropped", "w[(size_t)t * K + k], h, yt);", "1.0, h, yt);"),
]


def test_moe_mutations_are_well_formed():
    src = open(SRC).read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, f"mutation {name}: text must occur exactly once"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_moe_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    mutated = tmp_path / "moe_oracle.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / "liboracle_moe_mutant.so")
    oracle.build(moe_src=str(mutated), out=so, force=True, werror=False)
    lib = oracle.load(so)
    failed = []
    for check in moe_oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"

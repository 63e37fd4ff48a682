"""The fp64 oracle of the gated full-attention decode step against its pins
(tests/attn_oracle_pins.py), and planted mistakes in copies of
oracle/gattn_oracle.c that the pins must catch.  CPU only."""
import os

import pytest

import attn_oracle_pins
import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "gattn_oracle.c")


@pytest.mark.parametrize("check", attn_oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_attn_pin(check):
    check(oracle.load())


# (name, exact text in the oracle, replacement)
MUTANTS = [
    ("rope_not_a_rotation", "yr[i + half] = b * c + a * s;", "yr[i + half] = b * c - a * s;"),
    ("rope_frequency", "pow(theta, -2.0 * i / rot_dim)", "pow(theta, -1.0 * i / rot_dim)"),
    ("rope_position_off_by_one", "const double pos = (double)L;", "const double pos = (double)(L + 1);"),
    ("query_not_rotated",
     "orc_rope_partial(p->q + ((size_t)b * p->H_q + h) * d, 1, d, p->rot_dim, pos, p->theta,",
     "orc_rope_partial(p->q + ((size_t)b * p->H_q + h) * d, 1, d, 0, pos, p->theta,"),
    ("gqa_modulo", "const int g = (int)(((int64_t)h * p->H_kv) / p->H_q);", "const int g = h % p->H_kv;"),
    ("new_key_from_cache", "const double *kt = t < L ? kc + t * d : kr;", "const double *kt = kc + t * d;"),
    ("new_value_from_cache", "const double *vt = t < L ? vc + t * d : vn;", "const double *vt = vc + t * d;"),
    ("no_scale", "score[t] = p->scale * s;", "score[t] = s;"),
    ("gate_silu", "yrow[i] = oi / (1.0 + exp(-gt[i]));", "yrow[i] = oi * gt[i] / (1.0 + exp(-gt[i]));"),
    ("no_normalisation", "const double oi = acc[i] / l;", "const double oi = acc[i];"),
]


def test_attn_mutations_are_well_formed():
    src = open(SRC).read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, f"mutation {name}: text must occur exactly once"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_attn_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    mutated = tmp_path / "gattn_oracle.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / "liboracle_attn_mutant.so")
    oracle.build(attn_src=str(mutated), out=so, force=True, werror=False)
    lib = oracle.load(so)
    failed = []
    for check in attn_oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"

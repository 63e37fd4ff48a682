"""The fp64 oracle against closed forms, a hand-worked example and invariants
(see tests/oracle_pins.py for what each check pins)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(lib, check):
    check(lib)


def test_threads_do_not_change_results(lib):
    import numpy as np
    rng = np.random.default_rng(20)
    p = oracle_pins._rand_problem(rng, [30, 17, 5], H_k=2, H_v=4, d=8)
    a = oracle.gdr_recurrent(**p, threads=1, lib=lib)
    b = oracle.gdr_recurrent(**p, threads=4, lib=lib)
    assert np.array_equal(a.o, b.o) and np.array_equal(a.state, b.state)
    c = oracle.gdr_chunked(**p, chunk=8, threads=3, lib=lib)
    d = oracle.gdr_chunked(**p, chunk=8, threads=1, lib=lib)
    assert np.array_equal(c.o, d.o)


def test_rejects_bad_arguments(lib):
    import numpy as np
    rng = np.random.default_rng(21)
    p = oracle_pins._rand_problem(rng, [10], d=4)
    with pytest.raises(ValueError):
        oracle.gdr_bruteforce(**p, lib=lib)  # longer than 8 tokens
    with pytest.raises(ValueError):
        oracle.gdr_chunked(**p, chunk=0, lib=lib)
    with pytest.raises(ValueError):
        oracle.gdr_recurrent(**dict(p, cu_seqlens=[0, 3]), lib=lib)


# ---------------------------------------------------------------- raw gates
# g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b): pinned by closed
# forms, not by re-typing the formula.
import numpy as np  # noqa: E402

def test_gate_from_raw_closed_forms():
    a = np.array([[0.0, -3.0], [50.0, -800.0], [800.0, 2.0]])
    b = np.array([[0.0, 1.0], [-1.0, 40.0], [-800.0, 3.0]])
    A_log = np.array([0.0, np.log(2.0)])
    dt_bias = np.array([0.0, 3.0])
    g, beta = oracle.gate_from_raw(a, b, A_log, dt_bias)
    # x = a + dt_bias: 0 -> softplus = ln 2; head 1 scales by exp(ln 2) = 2.
    assert g[0, 0] == pytest.approx(-np.log(2.0), rel=1e-15)
    assert g[0, 1] == pytest.approx(-2.0 * np.log(2.0), rel=1e-15)   # -3 + 3 = 0
    assert g[1, 0] == pytest.approx(-(50.0 + np.log1p(np.exp(-50.0))), rel=1e-15)
    assert g[1, 1] == 0.0                                              # e^-797 underflows
    assert g[2, 0] == pytest.approx(-800.0, rel=1e-15)                # no overflow
    assert beta[0, 0] == 0.5 and beta[2, 0] == 0.0 and beta[1, 1] == pytest.approx(1.0, abs=1e-15)
    assert beta[0, 1] == pytest.approx(1.0 / (1.0 + np.exp(-1.0)), rel=1e-15)


def test_gate_from_raw_identities():
    rng = np.random.default_rng(5)
    a = rng.normal(size=(40, 3)) * 4
    b = rng.normal(size=(40, 3)) * 4
    zero = np.zeros(3)
    g_pos, beta_pos = oracle.gate_from_raw(a, b, zero, zero)
    g_neg, beta_neg = oracle.gate_from_raw(-a, -b, zero, zero)
    # softplus(x) - softplus(-x) = x  and  sigmoid(x) + sigmoid(-x) = 1.
    np.testing.assert_allclose(-g_pos + g_neg, a, rtol=0, atol=1e-13)
    np.testing.assert_allclose(beta_pos + beta_neg, 1.0, rtol=0, atol=1e-15)
    # A_log = -inf switches the decay off (g = 0); decays are never positive.
    g_off, _ = oracle.gate_from_raw(a, b, np.full(3, -np.inf), zero)
    assert np.all(g_off == 0.0) and np.all(g_pos < 0)
    # dt_bias shifts the argument: g(a, dt_bias=c) == g(a + c, 0).
    c = np.array([0.5, -1.0, 2.0])
    g1, _ = oracle.gate_from_raw(a, b, zero, c)
    g2, _ = oracle.gate_from_raw(a + c, b, zero, zero)
    np.testing.assert_array_equal(g1, g2)

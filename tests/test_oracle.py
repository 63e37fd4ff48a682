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

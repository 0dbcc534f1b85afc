"""The fp64 oracle against facts it does not compute itself (CPU only)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load_library()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)


def test_oracle_threads_do_not_change_results(lib):
    """Rows spread over threads give the same bits as one thread."""
    import numpy as np
    rng = np.random.default_rng(5)
    p = oracle_pins._rand_problem(rng, 3, 7, 33, 16)
    o1, s1 = oracle.scan(**p, nthreads=1, lib=lib)
    o8, s8 = oracle.scan(**p, nthreads=8, lib=lib)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)

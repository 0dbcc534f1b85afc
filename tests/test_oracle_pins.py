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


def test_complex_oracle_threads_do_not_change_results(lib):
    """Complex mode: rows spread over threads give the same bits as one thread."""
    import numpy as np
    p = oracle_pins._cplx_problem(np.random.default_rng(6), 2, 5, 40, 4)
    o1, s1 = oracle.scan_complex(**p, nthreads=1, lib=lib)
    o8, s8 = oracle.scan_complex(**p, nthreads=8, lib=lib)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)


def test_backward_oracle_threads_only_reorder_sums(lib):
    """Backward: per-row gradients are the same bits on any thread count; the
    gradients summed over rows (dA, dB, dC, dD, dbias) add the threads'
    partial sums in thread order, so they may differ by rounding only."""
    import numpy as np
    p, h0, dout, dlast = oracle_pins._bwd_problem(307, batch=3, dim=5, L=12, N=4)
    r1 = oracle.scan_bwd(dout, **p, h0=h0, dlast=dlast, nthreads=1, lib=lib)
    r8 = oracle.scan_bwd(dout, **p, h0=h0, dlast=dlast, nthreads=8, lib=lib)
    for k in ("du", "ddelta", "dz", "dh0"):
        assert np.array_equal(r1[k], r8[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        np.testing.assert_allclose(r8[k], r1[k], rtol=1e-12, atol=1e-14, err_msg=k)

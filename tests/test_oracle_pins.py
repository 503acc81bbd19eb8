"""The fp64 oracle against the pages' closed forms, special cases and printed values."""
import pytest

import oracle
import oracle_pins as P


def _fwd(form, q, k, v, log_w, e1, e2, S0):
    return oracle.forward(form, q, k, v, log_w, e1, e2, S0)


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(_fwd)


def test_block_inverse_identities():
    e12, e11 = P.check_block_inverses()
    assert e12 < 1e-13 and e11 < 1e-13


def test_zero_length_and_empty_batch():
    import numpy as np
    z = np.zeros((2, 0, 3, 4))
    S0 = np.arange(2 * 3 * 4 * 4, dtype=np.float64).reshape(2, 3, 4, 4)
    o, S_T = oracle.forward("gla", z, z, z, z, None, None, S0)
    assert o.shape == (2, 0, 3, 4) and (S_T == S0).all()
    e = np.zeros((0, 5, 3, 4))
    o, S_T = oracle.forward("gla", e, e, e, e)
    assert o.shape == (0, 5, 3, 4) and S_T.shape == (0, 3, 4, 4)

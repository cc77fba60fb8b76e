"""The oracle's probe projection and prefill gradients against their pins
(CPU only; the pins live in oracle_pins_ext.py)."""
import numpy as np
import pytest

import oracle
import oracle_pins_ext


@pytest.fixture(scope="module")
def O():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins_ext.ALL_EXT_PINS, ids=lambda p: p.__name__)
def test_pin(O, pin):
    pin(O)


def test_bwd_threads_do_not_change_results(O):
    rng = np.random.default_rng(5)
    q, rho, g = (rng.standard_normal((2, 9, 4, 3)) for _ in range(3))
    k, v = (rng.standard_normal((2, 9, 2, 3)) for _ in range(2))
    a = O.prefill_bwd(q, rho, k, v, g, True, 0.7, threads=1)
    b = O.prefill_bwd(q, rho, k, v, g, True, 0.7, threads=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_bwd_rejects_bad_heads(O):
    q = np.zeros((1, 2, 3, 2))
    k = np.zeros((1, 2, 2, 2))
    with pytest.raises(AssertionError):
        O.prefill_bwd(q, q, k, k, q, True, 1.0)

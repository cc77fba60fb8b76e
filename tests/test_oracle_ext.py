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


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_bwd_sampled_matches_full_routine(O, causal):
    """prefill_bwd_sampled (numpy, row by row) gives, at every query row and
    key row of a small GQA problem, the same gradients as the C routine
    (itself pinned by finite differences and fp64 autograd)."""
    rng = np.random.default_rng(11)
    B, L, Hq, Hkv, d = 2, 23, 4, 2, 8
    q, rho, g = (rng.standard_normal((B, L, Hq, d)) for _ in range(3))
    k, v = (rng.standard_normal((B, L, Hkv, d)) for _ in range(2))
    rho *= 0.7
    dq, drho, dk, dv = O.prefill_bwd(q, rho, k, v, g, causal, 0.4)
    rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(L)])
    keys = np.array([(b, hk, j) for b in range(B) for hk in range(Hkv) for j in range(L)])
    sq, sr, sk, sv = oracle.prefill_bwd_sampled(q, rho, k, v, g, causal, 0.4, rows, keys)
    for got, ref, idx in ((sq, dq, rows), (sr, drho, rows)):
        want = ref[idx[:, 0], idx[:, 2], idx[:, 1]]
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    for got, ref in ((sk, dk), (sv, dv)):
        want = ref[keys[:, 0], keys[:, 2], keys[:, 1]]
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)

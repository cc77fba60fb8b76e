"""The oracle against its pins (CPU only).

The pins live in oracle_pins.py; this file runs each of them on both oracle
forms, plus the hand-derived worked examples under tests/golden/.
"""
import json
import os

import numpy as np
import pytest

import oracle
import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def O():
    return oracle.get()


@pytest.mark.parametrize("form", ["explicit", "expanded"])
@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(O, pin, form):
    pin(O, form)


@pytest.mark.parametrize("form", ["explicit", "expanded"])
def test_worked_examples(O, form):
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        ex = json.load(f)["examples"]
    for e in ex:
        k = np.array(e["k"], dtype=np.float64)
        v = np.array(e["v"], dtype=np.float64)
        q = np.array(e["q"], dtype=np.float64)
        rho = np.array(e["rho"], dtype=np.float64)
        out, lse = O.rows(q[None], rho[None], k[None], v[None], [0], [len(k)], e["scale"], form)
        np.testing.assert_allclose(out[0], e["out"], rtol=0, atol=1e-12, err_msg=e["name"])
        np.testing.assert_allclose(lse[0], e["lse"], rtol=0, atol=1e-12, err_msg=e["name"])


def test_regression_values(O):
    """Values written by tests/golden/make_oracle_golden.py (calls only the
    oracle) at the time the oracle was pinned: a change to the oracle's
    arithmetic must show up here and be justified."""
    path = os.path.join(GOLDEN, "oracle_regression.json")
    with open(path) as f:
        g = json.load(f)
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_oracle_golden",
                                                  os.path.join(GOLDEN, "make_oracle_golden.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    for case in g["cases"]:
        out, lse = mk.evaluate(O, case["name"])
        np.testing.assert_allclose(out, np.array(case["out"]), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, np.array(case["lse"]), rtol=1e-12, atol=1e-12)


def test_rejects_bad_arguments(O):
    q = np.zeros((1, 2))
    k = np.zeros((1, 3, 2))
    with pytest.raises(ValueError):
        O.rows(q, q, k, k, [0], [4], 1.0)  # more keys than the stream holds
    with pytest.raises(ValueError):
        O.rows(q, q, k, k, [1], [1], 1.0)  # stream index out of range


def test_threads_do_not_change_results(O):
    rng = np.random.default_rng(3)
    q, rho = rng.standard_normal((37, 8)), rng.standard_normal((37, 8))
    K, V = rng.standard_normal((4, 50, 8)), rng.standard_normal((4, 50, 8))
    rs, rn = rng.integers(0, 4, 37), rng.integers(0, 51, 37)
    a, la = O.rows(q, rho, K, V, rs, rn, 0.3, threads=1)
    b, lb = O.rows(q, rho, K, V, rs, rn, 0.3, threads=7)
    assert np.array_equal(a, b) and np.array_equal(la, lb)

"""Planted mistakes in copies of the oracle must each fail at least one pin.

Each mutant is a one-place text edit of oracle/plx_oracle.c (a dropped term, a
flipped sign, a missing centring, a transposed contraction, unnormalised
weights, an ignored scale, a wrong lse), compiled into a temporary library on
the CPU.  The real oracle passes every pin (test_oracle.py); a pin set that
let one of these through would be too weak to trust.
"""
import os
import tempfile

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "plx_oracle.c")

MUTANTS = {
    "sign_flip": ("out[c] = o[c] - corr;", "out[c] = o[c] + corr;"),
    # Centring one side suffices for a cross-covariance (sum a (k - mu) v^T equals
    # sum a (k - mu)(v - o)^T), so the mistake to catch is centring neither.
    "neither_side_centred": [("a[j] * (kj[r] - mu[r])", "a[j] * (kj[r])"),
                             ("row[c] += wr * (vj[c] - o[c]);", "row[c] += wr * vj[c];")],
    "value_side_contraction": ("corr += cov[(int64_t)r * dv + c] * rho[r];",
                               "corr += cov[(int64_t)c * dv + r] * rho[r % dk];"),
    "weights_not_normalised": ("for (int64_t j = 0; j < n; ++j) a[j] /= l;", ""),
    "scale_ignored": ("s *= scale;", ""),
    "lse_without_log": ("*lse = m + log(l);", "*lse = m + l;"),
    "expanded_tbar_sign": ("out[c] = o[c] - (ubuf[c] - tbar * o[c]);",
                           "out[c] = o[c] - (ubuf[c] + tbar * o[c]);"),
    "expanded_tbar_dropped": ("out[c] = o[c] - (ubuf[c] - tbar * o[c]);",
                              "out[c] = o[c] - ubuf[c];"),
    "expanded_t_unweighted": ("tbar += a[j] * t;", "tbar += t;"),
    "first_key_skipped": ("for (int64_t j = 0; j < n; ++j) {\n        const double *vj = v + j * dv;\n        for (int c = 0; c < dv; ++c) o[c] += a[j] * vj[c];",
                          "for (int64_t j = 1; j < n; ++j) {\n        const double *vj = v + j * dv;\n        for (int c = 0; c < dv; ++c) o[c] += a[j] * vj[c];"),
}


# Mistakes in the probe projection and the prefill gradients; each must fail
# at least one pin of oracle_pins_ext.
EXT_MUTANTS = {
    "probe_transposed": ("acc += w[n * K + kk] * x[m * K + kk];",
                         "acc += w[kk * N + n] * x[m * K + kk];"),
    "bwd_dt_sign": ("const double dt = a[j] * (go - gv);", "const double dt = a[j] * (gv - go);"),
    "bwd_dsum_tbar_term_dropped": ("const double dsum = gout + tbar * go;",
                                   "const double dsum = gout;"),
    "bwd_da_t_term_dropped": ("const double da = cj * gv + t[j] * go;",
                              "const double da = cj * gv;"),
    "bwd_dv_coefficient_dropped": ("DVROW(j)[c] += a[j] * cj * gi[c];",
                                   "DVROW(j)[c] += a[j] * gi[c];"),
    "bwd_dk_probe_term_dropped": ("DKROW(j)[c] += jb->scale * ds * qi[c] + dt * ri[c];",
                                  "DKROW(j)[c] += jb->scale * ds * qi[c];"),
    "bwd_dq_scale_dropped": ("dqi[c] += jb->scale * ds * KROW(j)[c];",
                             "dqi[c] += ds * KROW(j)[c];"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def _catches(O, form):
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(O, form)
        except (AssertionError, ValueError, FloatingPointError) as e:
            failures.append(f"{pin.__name__}: {str(e)[:80]}")
    return failures


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(source, name):
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    mutated = source
    for old, new in edits:
        assert mutated.count(old) == 1, f"mutant anchor for {name} not unique in oracle source"
        mutated = mutated.replace(old, new)
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "mutant.c")
        with open(src, "w") as f:
            f.write(mutated)
        lib = oracle.build(src=src, out=os.path.join(td, "libmutant.so"))
        O = oracle.Oracle(lib)
        form = "expanded" if name.startswith("expanded") else "explicit"
        caught = _catches(O, form)
        assert caught, f"mutant {name} passed every pin"


@pytest.mark.parametrize("name", sorted(EXT_MUTANTS))
def test_ext_mutant_is_caught(source, name):
    import oracle_pins_ext
    old, new = EXT_MUTANTS[name]
    assert source.count(old) == 1, f"mutant anchor for {name} not unique in oracle source"
    with tempfile.TemporaryDirectory() as td:
        src = os.path.join(td, "mutant.c")
        with open(src, "w") as f:
            f.write(source.replace(old, new))
        O = oracle.Oracle(oracle.build(src=src, out=os.path.join(td, "libmutant.so")))
        caught = []
        for pin in oracle_pins_ext.ALL_EXT_PINS:
            try:
                pin(O)
            except (AssertionError, ValueError, FloatingPointError) as e:
                caught.append(f"{pin.__name__}: {str(e)[:80]}")
        assert caught, f"mutant {name} passed every pin"

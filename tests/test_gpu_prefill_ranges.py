"""plx_prefill_fwd (bf16, tcgen05 path) on inputs that drive the kernel's range
handling, against the fp64 oracle at the plain bf16 bar (fp32 output, so the
bar measures the arithmetic alone):

* a large probe: rho ~ N(0, 30^2) gives |rho . k| in the hundreds, past the
  fp16 range of P t; the per-row power-of-two scale of P t must grow mid-row
  and the U accumulator and its z column be rescaled with it.  A learned probe
  is large on purpose: under Muon the correction becomes significantly
  non-zero (page 1 "Parallax: Parameterized Local Linear Attention Gives
  Transformers a 'Second Eye'", section 2.3).
* a negative softmax scale: the running extreme of the raw scores is then a
  minimum, not a maximum.
* values far outside fp16's normal range (|v| ~ 1e-6 and ~1e5), and values
  whose magnitude spans eleven decades within one row: the PV products run in
  fp16, so V is carried with a power-of-two block scale.

Shapes span many 64-key tiles with a ragged tail (L = 1100), causal and not,
GQA and d = 64.
"""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx
from parity_util import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def _inputs(B, L, Hq, Hkv, d, seed, rho_std=0.1, v_scale=None, outliers=True):
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    q = (torch.randn(B, L, Hq, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    k32 = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    if outliers:
        hit = torch.rand((B, L, Hkv, 1), generator=g, device=DEV) < 0.01
        k32 = torch.where(hit, k32 * 8.0, k32)
    k = k32.to(torch.bfloat16)
    v32 = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    if v_scale == "mixed":
        # each key row scaled by 10^u, u uniform in [-6, 5]
        u = torch.rand((B, L, Hkv, 1), generator=g, device=DEV) * 11.0 - 6.0
        v32 = v32 * torch.pow(10.0, u)
    elif v_scale is not None:
        v32 = v32 * v_scale
    v = v32.to(torch.bfloat16)
    rho = (torch.randn(B, L, Hq, d, generator=g, device=DEV) * rho_std).to(torch.bfloat16)
    return q, rho, k, v


def _rows(B, L, Hq, n, seed):
    rng = np.random.default_rng(seed)
    i = np.concatenate([[0, 1, 63, 64, L - 1], rng.integers(0, L, n - 5)])
    return np.stack([rng.integers(0, B, n), rng.integers(0, Hq, n), i], axis=1).astype(np.int64)


def _run(q, rho, k, v, causal, scale, nrows=192, seed=0):
    B, L, Hq, _ = q.shape
    out, lse = plx.prefill(q, rho, k, v, causal=causal, softmax_scale=scale,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = _rows(B, L, Hq, nrows, seed)
    ref, ref_lse = oracle.prefill(q, rho, k, v, causal, scale, rows=rows)
    b, h, i = (torch.as_tensor(rows[:, c]) for c in range(3))
    return to_np(out[b, i, h]), ref, to_np(lse[b, h, i]), ref_lse


SHAPES = [(2, 1100, 4, 2, 128), (1, 1100, 2, 1, 64)]
IDS = ["gqa_d128", "d64"]


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_large_probe_rescales_pt_mid_row(shape, causal):
    q, rho, k, v = _inputs(*shape, seed=31, rho_std=30.0)
    tmax = float((torch.einsum("blhd,bmkd->blhm", rho[:, :, :1].float(),
                               k[:, :, :1].float())).abs().max())
    assert tmax > 128.0  # past the initial fp16 range kept for P t
    got, ref, gl, rl = _run(q, rho, k, v, causal, 1.0)
    check_out(got, ref, bf16=True, what=f"rho~N(0,30^2) {shape} causal={causal}")
    check_lse(gl, rl, bf16=True, what="lse")


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_negative_softmax_scale(shape, causal):
    d = shape[-1]
    q, rho, k, v = _inputs(*shape, seed=32, rho_std=0.3)
    for scale in (-1.0, -1.0 / np.sqrt(d)):
        got, ref, gl, rl = _run(q, rho, k, v, causal, scale)
        check_out(got, ref, bf16=True, what=f"scale={scale} {shape} causal={causal}")
        check_lse(gl, rl, bf16=True, what=f"lse scale={scale}")


@pytest.mark.parametrize("v_scale", [1e-6, 1e5, "mixed"], ids=["v1e-6", "v1e5", "v_mixed"])
@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_values_outside_fp16_range(shape, causal, v_scale):
    q, rho, k, v = _inputs(*shape, seed=33, rho_std=0.3, v_scale=v_scale)
    got, ref, _, _ = _run(q, rho, k, v, causal, 1.0)
    check_out(got, ref, bf16=True, what=f"v scale {v_scale} {shape} causal={causal}")


def test_values_outside_fp16_range_bf16_output_is_finite():
    """The default bf16 output of a 1e5-scaled V: finite and within the bar
    plus the output format's own rounding."""
    q, rho, k, v = _inputs(1, 700, 4, 2, 128, seed=34, v_scale=1e5)
    out, _ = plx.prefill(q, rho, k, v, causal=True, softmax_scale=1.0)
    torch.cuda.synchronize()
    rows = _rows(1, 700, 4, 128, seed=1)
    ref, _ = oracle.prefill(q, rho, k, v, True, 1.0, rows=rows)
    b, h, i = (torch.as_tensor(rows[:, c]) for c in range(3))
    check_out(to_np(out[b, i, h]), ref, bf16=True, what="v1e5 bf16 out", output_rounding=True)

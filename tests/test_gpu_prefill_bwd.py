"""plx_prefill_bwd (CUDA, through the C ABI) against the fp64 oracle's
gradients of the prefill operator (the pages print no gradient; the oracle's
derivation is pinned by finite differences and fp64 autograd of the
explicit-covariance definition).  The loss is sum(dout * out) with a seeded
dout."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def _dout(shape, seed, dt):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return torch.randn(shape, generator=g, device=DEV).to(dt)


def _compare(inp, dout, causal, scale, bf16, what):
    q, rho, k, v = inp["q"], inp["rho"], inp["k"], inp["v"]
    grads = plx.prefill_bwd(q, rho, k, v, dout, causal=causal, softmax_scale=scale)
    torch.cuda.synchronize()
    refs = oracle.prefill_bwd(q, rho, k, v, dout, causal, scale)
    for name, got, ref in zip(("dq", "drho", "dk", "dv"), grads, refs):
        check_out(to_np(got), ref, bf16=bf16, what=f"{what} {name}")


@pytest.mark.parametrize("rho_zero", [False, True], ids=["rho", "rho0"])
def test_bwd_prefill_tiny_fp32(rho_zero):
    """The tiny fp32 prefill (B=1, H=1, L=128, d=64, causal, seed 0), at the
    fp32 bar (max abs error 1e-4) for every gradient."""
    shape = W.WORKLOADS["prefill_tiny_fp32"]
    inp = W.make_prefill(shape, seed=0, device=DEV, rho_zero=rho_zero)
    _compare(inp, _dout(inp["q"].shape, 1, torch.float32), True, 1.0, False, "tiny fp32")


CASES = [(1, 65, 4, 2, 64, True), (2, 33, 2, 1, 128, False), (1, 200, 3, 3, 128, True),
         (1, 1, 2, 1, 64, True)]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_bwd_fp32_shapes(case):
    B, L, Hq, Hkv, d, causal = case
    shape = W.PrefillShape(B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, dtype=torch.float32, rho_std=0.3)
    inp = W.make_prefill(shape, seed=L + Hq, device=DEV)
    _compare(inp, _dout(inp["q"].shape, 2, torch.float32), causal, 1.0 / np.sqrt(d), False,
             str(case))


@pytest.mark.parametrize("causal", [True, False], ids=["causal", "full"])
def test_bwd_bf16_l1024_outlier_keys(causal):
    """bf16 inputs with the prefill workload's distributions (1% of key rows x8,
    rho ~ N(0, 0.1^2)), B=1, L=1024, H_q=4, H_kv=2, d=128: every gradient at the
    bf16 bar (2e-2 of its RMS)."""
    shape = W.PrefillShape(B=1, L=1024, Hq=4, Hkv=2, d=128, outlier_frac=0.01, causal=causal)
    inp = W.make_prefill(shape, seed=5, device=DEV)
    _compare(inp, _dout(inp["q"].shape, 3, torch.bfloat16), causal, 1.0, True, "bf16 L=1024")


BF16_CASES = [(1, 1, 2, 1, 64, True), (1, 65, 4, 2, 64, True), (2, 200, 2, 1, 128, False),
              (1, 300, 3, 3, 128, True), (1, 520, 4, 2, 128, True), (2, 129, 2, 2, 64, False)]


@pytest.mark.parametrize("case", BF16_CASES, ids=[f"b{i}" for i in range(len(BF16_CASES))])
def test_bwd_bf16_shapes(case):
    """bf16 inputs (the tensor-core kernels) over ragged lengths that span
    several 64- and 128-row tiles and their partial tails, GQA groups of 1-2,
    d = 64 and 128, causal and not: every gradient at the bf16 bar."""
    B, L, Hq, Hkv, d, causal = case
    shape = W.PrefillShape(B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, rho_std=0.3)
    inp = W.make_prefill(shape, seed=7 * L + d, device=DEV)
    _compare(inp, _dout(inp["q"].shape, 4, torch.bfloat16), causal, 1.0 / np.sqrt(d), True,
             str(case))


def test_bwd_bf16_negative_scale():
    """A negative softmax scale (the softmax favours the smallest scores)."""
    shape = W.PrefillShape(B=1, L=257, Hq=2, Hkv=1, d=128, rho_std=0.3)
    inp = W.make_prefill(shape, seed=11, device=DEV)
    _compare(inp, _dout(inp["q"].shape, 5, torch.bfloat16), True, -0.2, True, "negative scale")


def test_bwd_bf16_full_size_sampled():
    """The backward at the full prefill workload (B=8, L=4096, H_q=16, H_kv=8,
    d=128, causal, 1% outlier keys), in the configuration the benchmark times:
    dq and drho at 48 stratified query rows and dk, dv at 16 key rows among the
    last 64 positions (the rows that see them are few), against the oracle's
    row-by-row gradients, at the bf16 bar."""
    shape = W.WORKLOADS["prefill_b8_l4096"]
    x = W.make_prefill(shape, seed=40, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(41)
    dout = torch.randn(x["q"].shape, generator=gen, device=DEV).to(torch.bfloat16)
    dq, drho, dk, dv = plx.prefill_bwd(x["q"], x["rho"], x["k"], x["v"], dout, causal=True,
                                       softmax_scale=1.0)
    torch.cuda.synchronize()
    rows = W.sample_rows_prefill(shape, 48, seed=42)
    rng = np.random.default_rng(43)
    keys = np.stack([rng.integers(0, shape.B, 16), rng.integers(0, shape.Hkv, 16),
                     rng.integers(shape.L - 64, shape.L, 16)], axis=1)
    rq, rr, rk, rv = oracle.prefill_bwd_sampled(x["q"], x["rho"], x["k"], x["v"], dout, True,
                                                1.0, rows, keys)
    b, h, i = (torch.as_tensor(rows[:, c], device=DEV) for c in range(3))
    kb, kh, kj = (torch.as_tensor(keys[:, c], device=DEV) for c in range(3))
    check_out(to_np(dq[b, i, h]), rq, bf16=True, what="full-size dq")
    check_out(to_np(drho[b, i, h]), rr, bf16=True, what="full-size drho")
    check_out(to_np(dk[kb, kj, kh]), rk, bf16=True, what="full-size dk")
    check_out(to_np(dv[kb, kj, kh]), rv, bf16=True, what="full-size dv")

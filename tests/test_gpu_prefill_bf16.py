"""plx_prefill_fwd with bf16 inputs (tcgen05 tensor-core path) against the
fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def _rand(B, L, Hq, Hkv, d, seed, rho_std=0.1):
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    q = (torch.randn(B, L, Hq, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    rho = (torch.randn(B, L, Hq, d, generator=g, device=DEV) * rho_std).to(torch.bfloat16)
    k = (torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    v = (torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    return q, rho, k, v


SHAPES = [(B, L, Hq, Hkv, d, causal)
          for (B, L, Hq, Hkv, d) in [(1, 1, 1, 1, 128), (1, 2, 2, 1, 64), (2, 3, 2, 2, 128),
                                     (1, 17, 4, 1, 128), (1, 64, 2, 2, 64), (1, 127, 2, 1, 128),
                                     (2, 128, 4, 2, 128), (1, 129, 3, 3, 64),
                                     (1, 255, 8, 2, 128), (2, 300, 4, 4, 128),
                                     (1, 520, 2, 1, 64)]
          for causal in (True, False)]


OUT = [torch.float32, torch.bfloat16]


def _check(out, ref, what):
    """fp32 output: the stated bar on the arithmetic alone.  bf16 output: the
    same bar plus the output format's own rounding (2^-8 |ref|)."""
    check_out(to_np(out), ref, bf16=True, what=f"{what} out={out.dtype}",
              output_rounding=(out.dtype == torch.bfloat16))


@pytest.mark.parametrize("odt", OUT, ids=["out_f32", "out_bf16"])
@pytest.mark.parametrize("case", SHAPES, ids=[f"c{i}" for i in range(len(SHAPES))])
def test_prefill_bf16_shapes(case, odt):
    B, L, Hq, Hkv, d, causal = case
    q, rho, k, v = _rand(B, L, Hq, Hkv, d, seed=L * 13 + Hq + d)
    scale = 1.0 / np.sqrt(d)
    out, lse = plx.prefill(q, rho, k, v, causal=causal, softmax_scale=scale, out_dtype=odt)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(q, rho, k, v, causal, scale)
    _check(out, ref, str(case))
    check_lse(to_np(lse), ref_lse, bf16=True, what=str(case))


def test_prefill_bf16_rho_zero_is_softmax():
    """rho = 0: plain softmax attention (page 3, W_R = 0)."""
    q, rho, k, v = _rand(2, 333, 4, 2, 128, seed=5)
    rho = torch.zeros_like(rho)
    out, _ = plx.prefill(q, rho, k, v, causal=True, softmax_scale=1.0, out_dtype=torch.float32)
    ref, _ = oracle.prefill(q, rho, k, v, True, 1.0)
    _check(out, ref, "rho=0")


def test_prefill_last_row_equals_decode():
    """Causal prefill row L-1 and a decode over the same L keys agree."""
    B, L, Hq, Hkv, d = 3, 700, 16, 8, 128
    q, rho, k, v = _rand(B, L, Hq, Hkv, d, seed=11, rho_std=0.3)
    out, _ = plx.prefill(q, rho, k, v, causal=True, softmax_scale=1.0, out_dtype=torch.float32)
    sl = torch.full((B,), L, dtype=torch.int32, device=DEV)
    dec = plx.decode(q[:, -1].contiguous(), rho[:, -1].contiguous(), k, v, sl, softmax_scale=1.0)
    ref, _ = oracle.decode(q[:, -1], rho[:, -1], k, v, sl, 1.0)
    check_out(to_np(out[:, -1]), ref, bf16=True, what="prefill last row")
    check_out(to_np(dec), ref, bf16=True, what="decode")


@pytest.mark.parametrize("odt", OUT, ids=["out_f32", "out_bf16"])
def test_prefill_b8_l4096_sampled_rows(odt):
    """Prefill workload B=8, L=4096, H_q=16, H_kv=8, d=128, causal, 1% outlier
    keys: 512 seeded rows against the explicit-covariance oracle."""
    shape = W.WORKLOADS["prefill_b8_l4096"]
    inp = W.make_prefill(shape, seed=0, device=DEV)
    out, lse = plx.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], causal=True,
                           softmax_scale=1.0, out_dtype=odt)
    torch.cuda.synchronize()
    rows = W.sample_rows_prefill(shape, 512, seed=1)
    ref, ref_lse = oracle.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], True, 1.0, rows=rows)
    b, h, i = (torch.as_tensor(rows[:, c]) for c in range(3))
    _check(out[b, i, h], ref, "prefill_b8_l4096 rows")
    check_lse(to_np(lse[b, h, i]), ref_lse, bf16=True, what="prefill_b8_l4096 lse")


def test_prefill_b8_l4096_all_rows_expanded():
    """Every row of the same workload against the oracle's expanded form."""
    shape = W.WORKLOADS["prefill_b8_l4096"]
    inp = W.make_prefill(shape, seed=0, device=DEV)
    out, lse = plx.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], causal=True,
                           softmax_scale=1.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], True, 1.0,
                                  form="expanded")
    _check(out, ref, "prefill_b8_l4096 all rows")
    check_lse(to_np(lse), ref_lse, bf16=True, what="prefill_b8_l4096 all lse")


@pytest.mark.parametrize("odt", OUT, ids=["out_f32", "out_bf16"])
def test_prefill_b1_l32768_sampled_rows(odt):
    """Long-context prefill B=1, L=32768, H_q=32, H_kv=8: out and lse on 256
    seeded rows stratified over the sequence."""
    shape = W.WORKLOADS["prefill_b1_l32768"]
    inp = W.make_prefill(shape, seed=0, device=DEV)
    out, lse = plx.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], causal=True,
                           softmax_scale=1.0, out_dtype=odt)
    torch.cuda.synchronize()
    rows = W.sample_rows_prefill(shape, 256, seed=1, stratified=True)
    ref, ref_lse = oracle.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], True, 1.0, rows=rows)
    b, h, i = (torch.as_tensor(rows[:, c]) for c in range(3))
    _check(out[b, i, h], ref, "prefill_b1_l32768 rows")
    check_lse(to_np(lse[b, h, i]), ref_lse, bf16=True, what="prefill_b1_l32768 lse")


def test_prefill_bf16_deterministic():
    q, rho, k, v = _rand(2, 1000, 8, 2, 128, seed=21)
    a, la = plx.prefill(q, rho, k, v, causal=True, softmax_scale=0.1)
    b, lb = plx.prefill(q, rho, k, v, causal=True, softmax_scale=0.1)
    assert torch.equal(a, b) and torch.equal(la, lb)

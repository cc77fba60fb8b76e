"""plx_prefill_fwd with fp32 inputs (CUDA-core path) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("rho_zero", [False, True])
def test_prefill_tiny_fp32(rho_zero):
    """B=1, H=1, L=128, d=64, causal, seed 0; also rho = 0, which must give
    softmax attention."""
    shape = W.WORKLOADS["prefill_tiny_fp32"]
    inp = W.make_prefill(shape, seed=0, device=DEV, rho_zero=rho_zero)
    scale = 1.0
    out, lse = plx.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], causal=True,
                           softmax_scale=scale)
    ref, ref_lse = oracle.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], True, scale)
    check_out(to_np(out), ref, bf16=False, what="prefill tiny")
    check_lse(to_np(lse), ref_lse, bf16=False, what="prefill tiny lse")
    if rho_zero:
        q = inp["q"].double().permute(0, 2, 1, 3)
        k = inp["k"].double().permute(0, 2, 1, 3)
        v = inp["v"].double().permute(0, 2, 1, 3)
        sdpa = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
        check_out(to_np(out), to_np(sdpa.permute(0, 2, 1, 3)), bf16=False, what="rho=0 vs sdpa")


CASES = [(B, L, Hq, Hkv, d, causal)
         for (B, L, Hq, Hkv, d) in [(1, 1, 1, 1, 64), (1, 2, 2, 1, 128), (2, 3, 2, 2, 64),
                                    (1, 17, 4, 1, 128), (1, 127, 2, 1, 64), (2, 128, 4, 2, 128),
                                    (1, 129, 3, 3, 64), (1, 255, 8, 2, 128)]
         for causal in (True, False)]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_prefill_fp32_shapes(case):
    B, L, Hq, Hkv, d, causal = case
    g = torch.Generator(device=DEV).manual_seed(L * 7 + Hq)
    s = d ** -0.25
    q = torch.randn(B, L, Hq, d, generator=g, device=DEV) * s
    rho = torch.randn(B, L, Hq, d, generator=g, device=DEV) * 0.1
    k = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    v = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    scale = 1.0 / np.sqrt(d)
    out, lse = plx.prefill(q, rho, k, v, causal=causal, softmax_scale=scale)
    ref, ref_lse = oracle.prefill(q, rho, k, v, causal, scale)
    check_out(to_np(out), ref, bf16=False, what=str(case))
    check_lse(to_np(lse), ref_lse, bf16=False, what=str(case))
    assert plx.device_error() == 0

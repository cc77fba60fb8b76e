"""plx_prefill_varlen (CUDA, through the C ABI): every packed sequence's rows
equal plx_prefill_fwd on that sequence alone, and match the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx
from parity_util import check_out, check_lse, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t):
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32).cpu()


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def _packed(lens, Hq, Hkv, d, seed, outliers=False):
    T = sum(lens)
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    q = (torch.randn(T, Hq, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    rho = (torch.randn(T, Hq, d, generator=g, device=DEV) * 0.1).to(torch.bfloat16)
    k32 = torch.randn(T, Hkv, d, generator=g, device=DEV) * s
    if outliers:
        hit = torch.rand((T, Hkv, 1), generator=g, device=DEV) < 0.01
        k32 = torch.where(hit, k32 * 8.0, k32)
    k = k32.to(torch.bfloat16)
    v = (torch.randn(T, Hkv, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=DEV)
    return q, rho, k, v, cu


CASES = [
    # lengths, Hq, Hkv, d, causal, out fp32
    ([1, 127, 128, 129, 300, 0, 517], 4, 2, 128, True, False),
    ([200, 64, 1000], 8, 2, 64, True, True),
    ([333, 5, 256], 4, 4, 128, False, False),
    ([2048, 77], 16, 8, 128, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_prefill_varlen_equals_per_sequence(case):
    lens, Hq, Hkv, d, causal, f32 = case
    q, rho, k, v, cu = _packed(lens, Hq, Hkv, d, seed=sum(lens) + Hq, outliers=True)
    scale = 1.0
    od = torch.float32 if f32 else None
    out, lse = plx.prefill_varlen(q, rho, k, v, cu, max(lens), causal=causal,
                                  softmax_scale=scale, out_dtype=od)
    torch.cuda.synchronize()
    for s, n in enumerate(lens):
        if n == 0:
            continue
        a, b = int(cu[s]), int(cu[s + 1])
        o1, l1 = plx.prefill(q[a:b][None].contiguous(), rho[a:b][None].contiguous(),
                             k[a:b][None].contiguous(), v[a:b][None].contiguous(),
                             causal=causal, softmax_scale=scale, out_dtype=od)
        torch.cuda.synchronize()
        assert torch.equal(_bits(out[a:b]), _bits(o1[0])), f"sequence {s} (length {n})"
        assert torch.equal(_bits(lse[:, a:b]), _bits(l1[0])), f"lse of sequence {s}"


def test_prefill_varlen_oracle_rows():
    lens = [130, 1, 400]
    Hq, Hkv, d = 4, 2, 128
    q, rho, k, v, cu = _packed(lens, Hq, Hkv, d, seed=21)
    out, lse = plx.prefill_varlen(q, rho, k, v, cu, 400, causal=True, softmax_scale=1.0,
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    a, b = int(cu[2]), int(cu[3])
    ref, rl = oracle.prefill(q[a:b][None], rho[a:b][None], k[a:b][None], v[a:b][None], True, 1.0)
    check_out(to_np(out[a:b][None]), ref, bf16=True, what="varlen sequence 2 (fp32 out)")
    check_lse(to_np(lse[:, a:b][None]), rl, bf16=True)


def test_prefill_varlen_too_long_sequence_is_reported():
    lens = [300]
    q, rho, k, v, cu = _packed(lens, 2, 1, 64, seed=2)
    plx.prefill_varlen(q, rho, k, v, cu, 128, causal=True, softmax_scale=0.125)
    assert plx.device_error(clear=True) == 2

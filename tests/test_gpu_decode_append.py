"""plx_decode_append (CUDA, through the C ABI): the KV-cache append is exact and
the decode that follows matches the fp64 oracle over the updated cache."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"

CASES = [
    # B, Hq, Hkv, d, S_max, lengths (counting the new token), dtype
    (3, 4, 2, 128, 200, [200, 1, 77], torch.bfloat16),
    (4, 16, 8, 128, 129, [129, 0, 96, 97], torch.bfloat16),
    (2, 2, 2, 64, 64, [64, 33], torch.bfloat16),
    (3, 6, 2, 128, 150, [150, 2, 0], torch.float32),
    (2, 4, 1, 64, 40, [45, 40], torch.float32),   # 45 > S_max: clamped, row 39 written
]


def _inputs(case, seed):
    B, Hq, Hkv, d, S, lens, dt = case
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    kn = (torch.randn(B, Hkv, d, generator=g, device=DEV) * s).to(dt)
    vn = (torch.randn(B, Hkv, d, generator=g, device=DEV) * s).to(dt)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return q, rho, k, v, kn, vn, sl


def _expected_caches(k, v, kn, vn, lens, S):
    ke, ve = k.clone(), v.clone()
    for b, n in enumerate(lens):
        n = min(max(n, 0), S)
        if n > 0:
            ke[b, n - 1] = kn[b]
            ve[b, n - 1] = vn[b]
    return ke, ve


def _bits(t):
    """The tensor's raw bits (bit-exact comparison)."""
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32).cpu()


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_decode_append(case):
    B, Hq, Hkv, d, S, lens, dt = case
    q, rho, k, v, kn, vn, sl = _inputs(case, 11 + B * 7 + S)
    ke, ve = _expected_caches(k, v, kn, vn, lens, S)
    scale = 1.0 / np.sqrt(d)
    out = plx.decode_append(q, rho, kn, vn, k, v, sl, softmax_scale=scale)
    torch.cuda.synchronize()
    # the append: exactly the new rows, nothing else
    assert torch.equal(_bits(k), _bits(ke)) and torch.equal(_bits(v), _bits(ve))
    # the decode: same bits as plx_decode on the updated cache, and parity with the oracle
    ref_gpu = plx.decode(q, rho, ke, ve, sl, softmax_scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref_gpu))
    inp = dict(q=q, rho=rho, k_cache=ke, v_cache=ve, seqlens=sl)
    ref, _ = oracle.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"],
                           inp["seqlens"], scale)
    check_out(to_np(out), ref, bf16=(dt == torch.bfloat16), what=str(case[:5]),
              output_rounding=True)


def test_decode_append_steps_grow_the_cache():
    """Three serving steps, each appending one token, equal one decode over the
    final cache with the same lengths."""
    B, Hq, Hkv, d, S = 2, 4, 2, 128, 100
    dt = torch.bfloat16
    q, rho, k, v, _, _, _ = _inputs((B, Hq, Hkv, d, S, [1, 1], dt), 5)
    k0, v0 = k.clone(), v.clone()
    lens = torch.tensor([60, 90], dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(9)
    for step in range(3):
        kn = (torch.randn(B, Hkv, d, generator=g, device=DEV) * d ** -0.25).to(dt)
        vn = (torch.randn(B, Hkv, d, generator=g, device=DEV) * d ** -0.25).to(dt)
        out = plx.decode_append(q, rho, kn, vn, k, v, lens, softmax_scale=1.0)
        for b in range(B):
            n = int(lens[b])
            k0[b, n - 1] = kn[b]
            v0[b, n - 1] = vn[b]
        lens += 1
    torch.cuda.synchronize()
    assert torch.equal(_bits(k), _bits(k0)) and torch.equal(_bits(v), _bits(v0))
    last = plx.decode(q, rho, k0, v0, lens - 1, softmax_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(last))

"""plx_decode_state + plx_merge_states (CUDA, through the C ABI): a context
split into slices and decoded slice by slice merges to the full decode, and to
the fp64 oracle."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t):
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32).cpu()


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def _inputs(B, Hq, Hkv, d, S, lens, dt, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return q, rho, k, v, sl


def _slices(k, v, lens, bounds):
    """Per slice [a, b): contiguous caches and the slice's filled lengths."""
    out = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        kl, vl = k[:, a:b].contiguous(), v[:, a:b].contiguous()
        sl = torch.tensor([min(max(n - a, 0), b - a) for n in lens], dtype=torch.int32,
                          device=DEV)
        out.append((kl, vl, sl))
    return out


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_single_state_merges_to_the_same_bits(dt):
    B, Hq, Hkv, d, S = 4, 16, 8, 128, 700
    lens = [700, 0, 96, 333]
    q, rho, k, v, sl = _inputs(B, Hq, Hkv, d, S, lens, dt, seed=3)
    st = plx.decode_state(q, rho, k, v, sl, softmax_scale=1.0)
    out = plx.merge_states(st[None].contiguous(), out_dtype=dt)
    ref = plx.decode(q, rho, k, v, sl, softmax_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref))
    assert torch.isinf(st[1, :, 0]).all() and (st[1, :, 1:] == 0).all()  # empty sequence


@pytest.mark.parametrize("case", [
    (3, 8, 2, 128, 1000, [1000, 999, 1], [0, 256, 640, 1000], torch.bfloat16),
    (2, 4, 4, 64, 300, [300, 150], [0, 100, 200, 300], torch.float32),
    (2, 16, 8, 128, 4096, [4096, 3000], [0, 1024, 2048, 3072, 4096], torch.bfloat16),
], ids=["bf16_3slices", "fp32_3slices", "bf16_4slices_ctx4096"])
def test_split_context_merges_to_full_decode(case):
    B, Hq, Hkv, d, S, lens, bounds, dt = case
    q, rho, k, v, sl = _inputs(B, Hq, Hkv, d, S, lens, dt, seed=S + B)
    scale = 1.0 / np.sqrt(d)
    states = torch.stack([plx.decode_state(q, rho, kl, vl, sll, softmax_scale=scale)
                          for kl, vl, sll in _slices(k, v, lens, bounds)]).contiguous()
    out = plx.merge_states(states, out_dtype=torch.float32)
    full = plx.decode(q, rho, k, v, sl, softmax_scale=scale)
    torch.cuda.synchronize()
    ref, _ = oracle.decode(q, rho, k, v, sl, scale)
    check_out(to_np(out), ref, bf16=(dt == torch.bfloat16), what=f"merged {case[:5]}")
    # the merge only reorders fp32 sums: close to the single-pass decode
    tol = 1e-5 if dt == torch.float32 else 1e-2
    np.testing.assert_allclose(to_np(out), to_np(full.float()), atol=tol * max(1.0, float(np.abs(ref).max())))


def test_context_parallel_decode_one_rank():
    """The torch.distributed helper on a one-rank NCCL group."""
    import torch.distributed as dist
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        B, Hq, Hkv, d, S = 2, 8, 4, 128, 500
        q, rho, k, v, sl = _inputs(B, Hq, Hkv, d, S, [500, 77], torch.bfloat16, seed=9)
        out = plx.context_parallel_decode(q, rho, k, v, sl, softmax_scale=1.0)
        ref = plx.decode(q, rho, k, v, sl, softmax_scale=1.0)
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), _bits(ref))
    finally:
        dist.destroy_process_group()

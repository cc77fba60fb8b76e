"""plx_decode_static_ws, the decode entry point for callers that cannot
allocate device memory (a per-token serving loop that must stay out of the
allocator, a plugin whose host owns the device memory pool, a C caller with no
device allocator).  It runs the plx_decode kernels with a fixed workspace
array inside the library, so its output must equal plx_decode's bit for bit,
call after call, while the shared array carries state from one call to the
next: a full-grid call first, then calls whose grids are smaller (their CTAs
must not read slots that the earlier, larger grid left behind), with ragged
lengths, an fp32 cache and d = 64.

This file is collected last on purpose: it must pass both on its own in a
fresh process (where its first call does the per-device set-up) and after
every other test.
"""
import ctypes

import pytest
import torch

from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def static_decode(inp, scale):
    """Call the entry point through the C ABI; returns (status, out)."""
    f = plx.lib().plx_decode_static_ws
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp]
    f.restype = i
    q, k = inp["q"], inp["k_cache"]
    B, Hq, d = q.shape
    S_max, Hkv = k.shape[1], k.shape[2]
    out = torch.full_like(q, float("nan"))
    dtype = plx.PLX_BF16 if q.dtype == torch.bfloat16 else plx.PLX_F32
    st = f(q.data_ptr(), inp["rho"].data_ptr(), k.data_ptr(), inp["v_cache"].data_ptr(),
           inp["seqlens"].data_ptr(), out.data_ptr(), B, Hq, Hkv, d, S_max, dtype, scale,
           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st, out


def _small(B, Hq, Hkv, d, S, lens, dt, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    s = d ** -0.25
    return dict(q=(torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt),
                rho=(torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt),
                k_cache=(torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt),
                v_cache=(torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt),
                seqlens=torch.tensor(lens, dtype=torch.int32, device=DEV))


def test_static_workspace_decode_matches_plx_decode_call_after_call():
    calls = [
        ("decode_b32_ctx4096 (full grid)",
         W.make_decode(W.WORKLOADS["decode_b32_ctx4096"], seed=0, device=DEV)),
        ("B=5 ragged, S_max=777 (full grid)",
         W.make_decode(W.DecodeShape(B=5, Hq=16, Hkv=8, d=128, S_max=777, ctx=777, ragged=True),
                       seed=3, device=DEV)),
        ("B=1, H_q=2, H_kv=1, 64 keys (one tile, grid of 1)",
         _small(1, 2, 1, 128, 64, [64], torch.bfloat16, seed=4)),
        ("B=3 fp32, d=64, ragged (small grid)",
         _small(3, 4, 2, 64, 150, [150, 0, 49], torch.float32, seed=5)),
        ("B=2, 300 keys (a few tiles, split segments)",
         _small(2, 16, 8, 128, 300, [300, 97], torch.bfloat16, seed=6)),
    ]
    for n, (what, inp) in enumerate(calls):
        ref = plx.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                         softmax_scale=1.0)
        torch.cuda.synchronize()
        st, out = static_decode(inp, 1.0)
        assert st == plx.PLX_OK, f"call {n} ({what}): {plx.status_string(st)}"
        if not torch.equal(out, ref):
            # say by how much before failing on the bit comparison
            check_out(to_np(out), to_np(ref), bf16=out.dtype == torch.bfloat16,
                      what=f"static-workspace call {n} ({what})")
        assert torch.equal(out, ref), f"call {n} ({what}): not bit-identical to plx_decode"
    assert plx.device_error() == 0

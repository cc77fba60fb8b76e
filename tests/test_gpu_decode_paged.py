"""plx_decode_paged (CUDA, through the C ABI): over a paged KV cache it gives the
same bits as plx_decode over the same rows stored contiguously, and matches
the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t):
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32).cpu()


def paginate(k, v, lens, page_size, seed, spare_pages=3):
    """Scatter the contiguous caches [B, S_max, Hkv, d] into shuffled page pools;
    block-table entries past each sequence's last page are -1 (never read)."""
    B, S_max = k.shape[0], k.shape[1]
    max_pages = -(-S_max // page_size)
    used = [-(-min(max(n, 0), S_max) // page_size) for n in lens]
    num_pages = sum(used) + spare_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g).tolist()
    kp = torch.zeros((num_pages, page_size) + tuple(k.shape[2:]), dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    bt = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for i in range(used[b]):
            pg = perm[nxt]
            nxt += 1
            bt[b, i] = pg
            lo, hi = i * page_size, min((i + 1) * page_size, S_max)
            kp[pg, :hi - lo] = k[b, lo:hi]
            vp[pg, :hi - lo] = v[b, lo:hi]
    return kp, vp, bt.to(k.device)


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


CASES = [
    # B, Hq, Hkv, d, S_max, lengths, page_size, dtype
    (3, 4, 2, 128, 300, [300, 17, 0], 16, torch.bfloat16),
    (2, 16, 8, 128, 520, [520, 255], 32, torch.bfloat16),
    (4, 4, 4, 64, 200, [200, 96, 97, 1], 48, torch.bfloat16),
    (2, 6, 2, 128, 700, [700, 513], 128, torch.bfloat16),
    (2, 4, 2, 128, 600, [600, 300], 256, torch.bfloat16),
    (3, 4, 2, 128, 150, [150, 49, 0], 16, torch.float32),
    (2, 8, 2, 64, 250, [250, 64], 64, torch.float32),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_decode_paged_matches_contiguous(case):
    B, Hq, Hkv, d, S, lens, ps, dt = case
    g = torch.Generator(device=DEV).manual_seed(3 + B * 5 + S + ps)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    kp, vp, bt = paginate(k, v, lens, ps, seed=ps + S)
    scale = 1.0 / np.sqrt(d)
    out = plx.decode_paged(q, rho, kp, vp, bt, sl, softmax_scale=scale)
    # the paged cache's S_max is a whole number of pages: the contiguous call
    # gets the same S_max (zero rows appended), hence the same split of the
    # work over CTAs and the same bits
    S_pad = bt.shape[1] * ps
    kc = torch.zeros((B, S_pad, Hkv, d), dtype=dt, device=DEV)
    vc = torch.zeros_like(kc)
    kc[:, :S] = k
    vc[:, :S] = v
    ref_gpu = plx.decode(q, rho, kc, vc, sl, softmax_scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref_gpu))
    ref, _ = oracle.decode(q, rho, k, v, sl, scale)
    check_out(to_np(out), ref, bf16=(dt == torch.bfloat16), what=str(case[:7]),
              output_rounding=True)


def test_decode_paged_workload_b32_ctx4096_pages16():
    """The decode workload (B=32, H_q=16, H_kv=8, d=128, context 4096) in
    16-token pages: same bits as the contiguous decode; sampled rows vs oracle."""
    shape = W.WORKLOADS["decode_b32_ctx4096"]
    inp = W.make_decode(shape, seed=4, device=DEV)
    lens = inp["seqlens"].tolist()
    kp, vp, bt = paginate(inp["k_cache"], inp["v_cache"], lens, 16, seed=11, spare_pages=0)
    out = plx.decode_paged(inp["q"], inp["rho"], kp, vp, bt, inp["seqlens"], softmax_scale=1.0)
    ref_gpu = plx.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                         softmax_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(_bits(out), _bits(ref_gpu))
    rows = W.sample_rows_decode(shape.B, shape.Hq, 48, seed=5)
    ref, _ = oracle.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                           1.0, rows=rows)
    got = to_np(out)[rows[:, 0], rows[:, 1]]
    check_out(got, ref, bf16=True, what="decode_b32_ctx4096 paged")


def test_decode_paged_bad_page_index_is_reported():
    """A block-table entry outside the pool for a live position: device error 2,
    the chunk reads as zeros, and the call still completes."""
    B, Hq, Hkv, d, S, ps = 1, 2, 1, 64, 64, 16
    dt = torch.bfloat16
    q = torch.randn(B, Hq, d, device=DEV).to(dt)
    rho = torch.zeros(B, Hq, d, device=DEV).to(dt)
    k = torch.randn(B, S, Hkv, d, device=DEV).to(dt)
    v = torch.randn(B, S, Hkv, d, device=DEV).to(dt)
    kp, vp, bt = paginate(k, v, [S], ps, seed=1)
    bt[0, 2] = kp.shape[0] + 5  # out of range
    plx.decode_paged(q, rho, kp, vp, bt, torch.tensor([S], dtype=torch.int32, device=DEV),
                     softmax_scale=0.125)
    assert plx.device_error(clear=True) == 2

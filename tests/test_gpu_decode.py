"""plx_decode (CUDA, through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_decode(inp, scale=1.0):
    out = plx.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                     softmax_scale=scale)
    torch.cuda.synchronize()
    return out


def oracle_rows(inp, scale, rows=None):
    return oracle.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                         scale, rows=rows)


@pytest.fixture(autouse=True)
def _no_device_error():
    yield
    assert plx.device_error(clear=True) == 0


def test_decode_b32_ctx4096_all_rows():
    """Decode workload: B=32, H_q=16, H_kv=8, d=128, context 4096, rho = x W_R^T;
    every (b, h) row against the explicit-covariance oracle."""
    shape = W.WORKLOADS["decode_b32_ctx4096"]
    inp = W.make_decode(shape, seed=0, device=DEV)
    out = run_decode(inp, 1.0)
    ref, _ = oracle_rows(inp, 1.0)
    check_out(to_np(out), ref, bf16=True, what="decode_b32_ctx4096")


SMALL = [
    # B, Hq, Hkv, d, S_max, lengths, dtype
    (1, 1, 1, 64, 1, [1], torch.float32),
    (2, 2, 1, 128, 70, [70, 1], torch.float32),
    (3, 4, 2, 64, 200, [200, 0, 129], torch.float32),
    (2, 3, 1, 128, 129, [64, 129], torch.float32),       # G = 3: one head per pass
    (4, 8, 2, 128, 300, [300, 257, 63, 64], torch.float32),  # G = 4: two passes of two
    (1, 2, 2, 128, 1000, [1000], torch.float32),
    (1, 1, 1, 128, 5, [3], torch.bfloat16),
    (5, 16, 8, 128, 333, [333, 1, 65, 128, 200], torch.bfloat16),
    (3, 4, 4, 64, 257, [257, 256, 0], torch.bfloat16),
    (2, 6, 2, 128, 4100, [4100, 2049], torch.bfloat16),
    (64, 16, 8, 128, 96, None, torch.bfloat16),
]


@pytest.mark.parametrize("case", SMALL, ids=[f"c{i}" for i in range(len(SMALL))])
def test_decode_small_shapes(case):
    B, Hq, Hkv, d, S, lens, dt = case
    g = torch.Generator(device=DEV).manual_seed(7 + B * 31 + S)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    if lens is None:
        sl = torch.randint(0, S + 1, (B,), generator=g, device=DEV, dtype=torch.int32)
    else:
        sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    inp = dict(q=q, rho=rho, k_cache=k, v_cache=v, seqlens=sl)
    scale = 1.0 / np.sqrt(d)
    out = run_decode(inp, scale)
    ref, _ = oracle_rows(inp, scale)
    check_out(to_np(out), ref, bf16=(dt == torch.bfloat16), what=str(case[:5]),
              output_rounding=True)


@pytest.mark.parametrize("case", [c for c in SMALL if c[-1] == torch.bfloat16],
                         ids=[f"c{i}" for i, c in enumerate(SMALL) if c[-1] == torch.bfloat16])
def test_decode_small_shapes_fp32_result_strict_bar(case):
    """The bf16 edge shapes above at the plain 2e-2 RMS bar, with no allowance
    for the output format: the result is taken in fp32 through the state path
    (plx_decode_state, then plx_merge_states of the single slice into fp32),
    which runs the same main kernel and merge arithmetic as plx_decode."""
    B, Hq, Hkv, d, S, lens, dt = case
    g = torch.Generator(device=DEV).manual_seed(7 + B * 31 + S)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(dt)
    if lens is None:
        sl = torch.randint(0, S + 1, (B,), generator=g, device=DEV, dtype=torch.int32)
    else:
        sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    scale = 1.0 / np.sqrt(d)
    st = plx.decode_state(q, rho, k, v, sl, softmax_scale=scale)
    out = plx.merge_states(st[None].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, _ = oracle.decode(q, rho, k, v, sl, scale)
    check_out(to_np(out), ref, bf16=True, what=f"fp32 result {case[:5]}")
    # and plx_decode's bf16 output is that fp32 result rounded once
    bf = plx.decode(q, rho, k, v, sl, softmax_scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(bf, out.to(torch.bfloat16))


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_decode_ignores_rows_beyond_seqlen(dt):
    """Cache rows past seqlens[b] (here NaN and inf) never reach the output."""
    B, Hq, Hkv, d, S = 3, 4, 2, 128, 200
    g = torch.Generator(device=DEV).manual_seed(3)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(dt) * 0.3
    rho = torch.randn(B, Hq, d, generator=g, device=DEV).to(dt) * 0.3
    k = torch.randn(B, S, Hkv, d, generator=g, device=DEV).to(dt) * 0.3
    v = torch.randn(B, S, Hkv, d, generator=g, device=DEV).to(dt) * 0.3
    sl = torch.tensor([150, 1, 77], dtype=torch.int32, device=DEV)
    clean = dict(q=q, rho=rho, k_cache=k.clone(), v_cache=v.clone(), seqlens=sl)
    for b in range(B):
        k[b, sl[b]:] = float("nan")
        v[b, sl[b]:] = float("inf")
    dirty = dict(q=q, rho=rho, k_cache=k, v_cache=v, seqlens=sl)
    a = run_decode(clean)
    b_ = run_decode(dirty)
    assert torch.equal(a, b_)
    ref, _ = oracle_rows(clean, 1.0)
    check_out(to_np(b_), ref, bf16=(dt == torch.bfloat16), what="beyond seqlen",
              output_rounding=True)


def test_decode_clamps_lengths_and_zero_length():
    B, Hq, Hkv, d, S = 4, 2, 1, 64, 50
    g = torch.Generator(device=DEV).manual_seed(5)
    q = torch.randn(B, Hq, d, generator=g, device=DEV)
    rho = torch.randn(B, Hq, d, generator=g, device=DEV) * 0.2
    k = torch.randn(B, S, Hkv, d, generator=g, device=DEV) * 0.3
    v = torch.randn(B, S, Hkv, d, generator=g, device=DEV)
    sl = torch.tensor([0, -5, 500, 1], dtype=torch.int32, device=DEV)
    inp = dict(q=q, rho=rho, k_cache=k, v_cache=v, seqlens=sl)
    out = run_decode(inp, 0.125)
    ref, _ = oracle_rows(inp, 0.125)
    check_out(to_np(out), ref, bf16=False, what="clamped lengths")
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[1]) == 0
    assert torch.allclose(out[3], v[3, 0, 0].expand(Hq, d), atol=1e-6)  # one key: out = v_0


def test_decode_rho_zero_is_softmax():
    """rho = 0: the operator is plain softmax attention (page 3, W_R = 0)."""
    B, Hq, Hkv, d, S = 4, 8, 2, 128, 700
    g = torch.Generator(device=DEV).manual_seed(9)
    q = torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3
    k = torch.randn(B, S, Hkv, d, generator=g, device=DEV) * 0.3
    v = torch.randn(B, S, Hkv, d, generator=g, device=DEV) * 0.3
    sl = torch.tensor([700, 513, 64, 2], dtype=torch.int32, device=DEV)
    out = plx.decode(q, torch.zeros_like(q), k, v, sl, softmax_scale=1.0)
    ref, _ = oracle.decode(q, torch.zeros_like(q), k, v, sl, 1.0)
    check_out(to_np(out), ref, bf16=False, what="rho=0")


@pytest.mark.parametrize("lens", [[200, 1, 300], [97, 1000, 5, 16], [4096, 1, 1, 1]],
                         ids=["short", "mixed", "one_long"])
def test_decode_lengths_far_below_capacity(lens):
    """Lengths far below S_max: fewer key tiles than CTAs, so segments split
    over CTAs with empty tile ranges between their pieces; the pieces must still
    merge into the oracle's result (fp32 through the state path, and bf16)."""
    B, Hq, Hkv, d, S = len(lens), 16, 8, 128, 4096
    g = torch.Generator(device=DEV).manual_seed(sum(lens))
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    rho = (torch.randn(B, Hq, d, generator=g, device=DEV) * 0.3).to(torch.bfloat16)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=DEV) * s).to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = plx.decode(q, rho, k, v, sl, softmax_scale=1.0)
    st = plx.decode_state(q, rho, k, v, sl, softmax_scale=1.0)
    f32 = plx.merge_states(st[None].contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref, _ = oracle.decode(q, rho, k, v, sl, 1.0)
    check_out(to_np(f32), ref, bf16=True, what=f"lengths {lens} (fp32 result)")
    assert torch.equal(out, f32.to(torch.bfloat16))


def test_decode_in_a_cuda_graph_replays_with_new_data():
    """plx_decode captured once in a CUDA graph and replayed after the cache
    changed: every replay must equal an eager call on the new contents (split
    segments' pieces carry the launch's identity, so a replay never merges a
    piece an earlier replay left in the workspace)."""
    shape = W.DecodeShape(B=6, Hq=16, Hkv=8, d=128, S_max=2000, ctx=2000, ragged=True)
    inp = W.make_decode(shape, seed=12, device=DEV)
    other = W.make_decode(shape, seed=13, device=DEV)
    ws = plx.decode_workspace(shape.B, shape.Hq, shape.Hkv, shape.d, shape.S_max, device=DEV)
    out = torch.empty_like(inp["q"])
    args = (inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        plx.decode(*args, softmax_scale=1.0, out=out, workspace=ws)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        plx.decode(*args, softmax_scale=1.0, out=out, workspace=ws)
    for src in (other, inp, other):
        inp["k_cache"].copy_(src["k_cache"])
        inp["v_cache"].copy_(src["v_cache"])
        graph.replay()
        torch.cuda.synchronize()
        eager = plx.decode(*args, softmax_scale=1.0)
        torch.cuda.synchronize()
        assert torch.equal(out, eager)


def test_decode_deterministic():
    shape = W.DecodeShape(B=8, Hq=16, Hkv=8, d=128, S_max=3000, ctx=3000, ragged=True)
    inp = W.make_decode(shape, seed=4, device=DEV)
    a = run_decode(inp)
    b = run_decode(inp)
    assert torch.equal(a, b)


def test_decode_workspace_too_small():
    q = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16, device=DEV)
    sl = torch.ones(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(plx.PlxError) as e:
        plx.decode(q, q, k, k, sl, workspace=ws)
    assert e.value.status == plx.PLX_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("cell", W.sweep_cells(), ids=lambda c: f"B{c.B}_ctx{c.ctx}")
def test_decode_sweep_sampled_rows(cell):
    """Decode sweep (B in 1..2048, context 128..32768 capped at 120 GB of cache,
    ragged lengths): up to 64 seeded (b, h) rows per cell against the oracle."""
    inp = W.make_decode(cell, seed=0, device=DEV)
    out = run_decode(inp, 1.0)
    rows = W.sample_rows_decode(cell.B, cell.Hq, 64, seed=1)
    ref, _ = oracle_rows(inp, 1.0, rows=rows)
    got = to_np(out[torch.as_tensor(rows[:, 0]), torch.as_tensor(rows[:, 1])])
    check_out(got, ref, bf16=True, what=f"sweep B={cell.B} ctx={cell.ctx}")
    del inp, out
    torch.cuda.empty_cache()

"""The probe projection rho = W_R x (page 1 "Parallax: Parameterized Local
Linear Attention Gives Transformers a 'Second Eye'", section 1.3: one extra
projection matrix; page 3 "Parallax keeps softmax, adds covariance correction
branch": rho_i = W_R x_i) on the GPU, through the C ABI, against the fp64
oracle: the projection alone (tensor-core GEMM for bf16, CUDA cores for fp32)
and composed with the decode and prefill operators, whose outputs are checked
against the oracle fed the exact fp64 probes."""
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


def _check_projection(got, x, w, bf16):
    ref = oracle.probe(x, w)
    mag = np.abs(to_np(x).reshape(-1, x.shape[-1])) @ np.abs(to_np(w)).T  # sum |x||w|
    mag = mag.reshape(ref.shape)
    g = to_np(got)
    err = np.abs(g - ref)
    # bf16: the result's own rounding (2^-8 relative) plus fp32 accumulation;
    # fp32: accumulation only
    bound = (2.0 ** -8 * np.abs(ref) if bf16 else 0.0) + 2.0 ** -20 * mag + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, f"projection error {worst:.3f} of its bound"


# On 148 SMs the bf16 shapes reach each schedule: one tile (1x64x64,
# 128x136x64), clusters of CTAs splitting K (5x256x72, 300x2048x2048,
# 1000x384x520 with an uneven split, 32x2048x2048 the decode batch),
# persistent single tiles (2000x1024x256), persistent pairs of tiles with an
# odd last tile and ragged M, N, K (2100x1096x136), SM pairs with ragged M, N,
# K and more 256 x 256 tiles than pairs (4100x1032x200); the smallest N and K
# the tensor cores take (3x8x16, 129x264x8: one partial tile and one partial
# k block).
@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (5, 256, 72), (128, 136, 64), (300, 2048, 2048),
                                   (1000, 384, 520), (32, 2048, 2048), (2000, 1024, 256),
                                   (4100, 1032, 200), (2100, 1096, 136), (3, 8, 16),
                                   (129, 264, 8)],
                         ids=["1x64x64", "5x256x72", "128x136x64", "300x2048x2048", "1000x384x520",
                              "32x2048x2048", "2000x1024x256", "4100x1032x200", "2100x1096x136",
                              "3x8x16", "129x264x8"])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_projection_matches_oracle(M, N, K, dt):
    x, w = W.make_probe_inputs((M,), K, N, seed=M + N + K, device=DEV, dtype=dt)
    rho = plx.probe_projection(x, w)
    torch.cuda.synchronize()
    _check_projection(rho, x, w, dt == torch.bfloat16)


def test_projection_zero_matrix_gives_zero():
    x, w = W.make_probe_inputs((77,), 128, 256, seed=1, device=DEV)
    rho = plx.probe_projection(x, torch.zeros_like(w))
    torch.cuda.synchronize()
    assert torch.count_nonzero(rho) == 0


def test_decode_x_b32_ctx4096():
    """Decode workload B=32, H_q=16, H_kv=8, d=128, context 4096 with rho = x W_R^T
    computed on the device (x ~ N(0,1) of width 2048, W_R ~ N(0, 0.02^2)):
    every (b, h) row against the oracle given the exact fp64 probes."""
    shape = W.WORKLOADS["decode_b32_ctx4096"]
    inp = W.make_decode(shape, seed=0, device=DEV)
    x, w = W.make_probe_inputs((shape.B,), 2048, shape.Hq * shape.d, seed=7, device=DEV)
    out, rho = plx.decode_x(inp["q"], x, w, inp["k_cache"], inp["v_cache"], inp["seqlens"],
                            softmax_scale=1.0)
    torch.cuda.synchronize()
    _check_projection(rho.reshape(shape.B, -1), x, w, True)
    rho_ref = oracle.probe(x, w).reshape(shape.B, shape.Hq, shape.d)
    ref, _ = oracle.decode(inp["q"], rho_ref, inp["k_cache"], inp["v_cache"], inp["seqlens"], 1.0)
    check_out(to_np(out), ref, bf16=True, what="decode_x")
    # the same as plx_decode on the probes it computed
    same = plx.decode(inp["q"], rho, inp["k_cache"], inp["v_cache"], inp["seqlens"],
                      softmax_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(same, out)


def test_prefill_x_b8_l4096_sampled_rows():
    """Prefill workload B=8, L=4096, H_q=16, H_kv=8, d=128 (1% outlier keys) with
    rho = x W_R^T from x [8, 4096, 2048]: 256 seeded rows against the oracle
    given the exact fp64 probes of those rows."""
    shape = W.WORKLOADS["prefill_b8_l4096"]
    inp = W.make_prefill(shape, seed=0, device=DEV)
    x, w = W.make_probe_inputs((shape.B, shape.L), 2048, shape.Hq * shape.d, seed=8,
                               device=DEV, w_std=0.0022)
    out, rho, lse = plx.prefill_x(inp["q"], x, w, inp["k"], inp["v"], causal=True,
                                  softmax_scale=1.0)
    torch.cuda.synchronize()
    rows = W.sample_rows_prefill(shape, 256, seed=2)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    xr = x[torch.as_tensor(b), torch.as_tensor(i)]
    _check_projection(rho[torch.as_tensor(b), torch.as_tensor(i)].reshape(len(rows), -1), xr, w,
                      True)
    rho_ref = np.zeros((shape.B, shape.L, shape.Hq, shape.d))
    rho_ref[b, i] = oracle.probe(xr, w).reshape(len(rows), shape.Hq, shape.d)
    ref, _ = oracle.prefill(inp["q"], rho_ref, inp["k"], inp["v"], True, 1.0, rows=rows)
    check_out(to_np(out[torch.as_tensor(b), torch.as_tensor(i), torch.as_tensor(h)]), ref,
              bf16=True, what="prefill_x rows", output_rounding=True)


def test_prefill_x_fp32_tiny():
    """fp32 throughout (CUDA-core projection and prefill) at the 1e-4 bar."""
    B, L, Hq, Hkv, d, dm = 1, 128, 2, 1, 64, 96
    g = torch.Generator(device=DEV).manual_seed(3)
    s = d ** -0.25
    q = torch.randn(B, L, Hq, d, generator=g, device=DEV) * s
    k = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    v = torch.randn(B, L, Hkv, d, generator=g, device=DEV) * s
    x, w = W.make_probe_inputs((B, L), dm, Hq * d, seed=4, device=DEV, dtype=torch.float32,
                               w_std=0.01)
    out, rho, lse = plx.prefill_x(q, x, w, k, v, causal=True, softmax_scale=1.0)
    torch.cuda.synchronize()
    rho_ref = oracle.probe(x, w).reshape(B, L, Hq, d)
    ref, _ = oracle.prefill(q, rho_ref, k, v, True, 1.0)
    check_out(to_np(out), ref, bf16=False, what="prefill_x fp32")

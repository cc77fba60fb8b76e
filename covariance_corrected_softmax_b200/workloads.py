"""Seeded synthetic inputs shaped like the Parallax pages' workloads.

This module holds no part of the attention arithmetic: it only draws random
tensors with fixed seeds, shapes and value distributions, so that the CUDA path,
the oracle, the tests and the benchmark all see the same bits.  Nothing here
imports the CUDA library or the oracle.

Workload families (the pages give no dataset; these synthetic inputs stand in
for the decode grid quoted on page 3, "Parallax keeps softmax, adds covariance
correction branch": batch 1-2048, context 128-32768, and for causal prefill):

* ``prefill_tiny_fp32``  fp32, B=1, H=1, L=128, d=64, causal; q, k, v ~ N(0,1)
  d^-1/4, rho ~ N(0, 0.1^2).  Run also with rho = 0 (plain softmax attention).
* ``decode_b32_ctx4096`` bf16 KV cache, B=32, H_q=16, H_kv=8, d=128, every
  sequence at context 4096; q, k, v ~ N(0,1) d^-1/4; rho = x W_R^T with
  x ~ N(0,1) of width 2048 and W_R ~ N(0, 0.02^2), reshaped to [B, H_q, d].
* ``decode_sweep``       bf16, H_q=16, H_kv=8, d=128, B in {1, 8, 64, 512, 2048}
  x context in {128, 1024, 8192, 32768}; per-sequence lengths uniform in
  [ceil(ctx/2), ctx]; caches whose allocated bytes would reach 120e9 are capped
  to the largest multiple of 1024 below it.
* ``prefill_b8_l4096``   bf16 causal prefill, B=8, L=4096, H_q=16, H_kv=8, d=128;
  1% of key rows (independent per batch, position and KV head) scaled by 8
  before rounding; rho ~ N(0, 0.1^2).
* ``prefill_b1_l32768``  bf16 causal prefill, B=1, L=32768, H_q=32, H_kv=8,
  d=128, same distributions.

All draws are fp32 from ``torch.Generator(device).manual_seed(seed)`` and are
rounded to the storage dtype with round-to-nearest-even.  The same seed gives
different numbers on CPU and CUDA generators; a check always compares both sides
on one set of tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

KV_CAP_BYTES = 120e9


@dataclass(frozen=True)
class PrefillShape:
    B: int
    L: int
    Hq: int
    Hkv: int
    d: int
    dtype: torch.dtype = torch.bfloat16
    causal: bool = True
    outlier_frac: float = 0.0
    rho_std: float = 0.1

    def flops(self) -> float:
        """Algorithmic flops: 8d per visible (query, key) pair per query head."""
        pairs = self.L * (self.L + 1) / 2 if self.causal else float(self.L) * self.L
        return 8.0 * self.d * pairs * self.B * self.Hq


@dataclass(frozen=True)
class DecodeShape:
    B: int
    Hq: int
    Hkv: int
    d: int
    S_max: int
    ctx: int
    ragged: bool = False
    dtype: torch.dtype = torch.bfloat16
    rho_mode: str = "projection"  # rho = x W_R^T (width H_q*d); or "normal"


WORKLOADS: Dict[str, object] = {
    "prefill_tiny_fp32": PrefillShape(B=1, L=128, Hq=1, Hkv=1, d=64, dtype=torch.float32),
    "decode_b32_ctx4096": DecodeShape(B=32, Hq=16, Hkv=8, d=128, S_max=4096, ctx=4096),
    "prefill_b8_l4096": PrefillShape(B=8, L=4096, Hq=16, Hkv=8, d=128, outlier_frac=0.01),
    "prefill_b1_l32768": PrefillShape(B=1, L=32768, Hq=32, Hkv=8, d=128, outlier_frac=0.01),
}

SWEEP_BATCHES = (1, 8, 64, 512, 2048)
SWEEP_CONTEXTS = (128, 1024, 8192, 32768)


def kv_bytes(B: int, S_max: int, Hkv: int, d: int, elem: int = 2) -> int:
    """Allocated bytes of the K and V caches together."""
    return B * S_max * Hkv * d * elem * 2


def capped_context(B: int, ctx: int, Hkv: int = 8, d: int = 128) -> int:
    """Largest context <= ctx (a multiple of 1024 when capped) under the 120e9 cap."""
    if kv_bytes(B, ctx, Hkv, d) < KV_CAP_BYTES:
        return ctx
    per_pos = kv_bytes(B, 1, Hkv, d)
    c = int(KV_CAP_BYTES // per_pos)
    c -= c % 1024
    while kv_bytes(B, c, Hkv, d) >= KV_CAP_BYTES:
        c -= 1024
    return c


def sweep_cells() -> List[DecodeShape]:
    cells = []
    for B in SWEEP_BATCHES:
        for ctx in SWEEP_CONTEXTS:
            c = capped_context(B, ctx)
            cells.append(DecodeShape(B=B, Hq=16, Hkv=8, d=128, S_max=c, ctx=c, ragged=True))
    return cells


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std: float, g, device, dtype) -> torch.Tensor:
    """fp32 N(0, std^2) draws rounded (RNE) to dtype; chunked along dim 0."""
    out = torch.empty(shape, dtype=dtype, device=device)
    if out.numel() == 0:
        return out
    per = max(1, int(2 ** 28 // max(1, out[0].numel())))  # ~1 GiB fp32 per chunk
    for s in range(0, shape[0], per):
        e = min(shape[0], s + per)
        x = torch.randn((e - s,) + tuple(shape[1:]), generator=g, device=device,
                        dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[s:e].copy_(x)
    return out


def make_prefill(shape: PrefillShape, seed: int = 0, device="cpu",
                 rho_zero: bool = False) -> Dict[str, torch.Tensor]:
    """q, rho [B, L, Hq, d]; k, v [B, L, Hkv, d] in shape.dtype."""
    B, L, Hq, Hkv, d = shape.B, shape.L, shape.Hq, shape.Hkv, shape.d
    g = _gen(device, seed)
    s = d ** -0.25
    q = _normal((B, L, Hq, d), s, g, device, shape.dtype)
    if shape.outlier_frac > 0:
        k32 = torch.randn((B, L, Hkv, d), generator=g, device=device, dtype=torch.float32)
        k32.mul_(s)
        hit = torch.rand((B, L, Hkv, 1), generator=g, device=device) < shape.outlier_frac
        k32 = torch.where(hit, k32 * 8.0, k32)
        k = k32.to(shape.dtype)
        del k32
    else:
        k = _normal((B, L, Hkv, d), s, g, device, shape.dtype)
    v = _normal((B, L, Hkv, d), s, g, device, shape.dtype)
    rho = _normal((B, L, Hq, d), shape.rho_std, g, device, shape.dtype)
    if rho_zero:
        rho.zero_()
    return {"q": q, "rho": rho, "k": k, "v": v}


def make_decode(shape: DecodeShape, seed: int = 0, device="cpu",
                copies: int = 1) -> Dict[str, object]:
    """q, rho [B, Hq, d]; k_cache, v_cache [B, S_max, Hkv, d]; seqlens int32 [B].

    ``copies`` > 1 returns extra independent cache copies under ``"k_caches"``
    and ``"v_caches"`` (lists), for benchmarks that rotate buffers to keep the
    L2 cache cold; every copy holds different random bits.
    """
    B, Hq, Hkv, d, S = shape.B, shape.Hq, shape.Hkv, shape.d, shape.S_max
    g = _gen(device, seed)
    s = d ** -0.25
    q = _normal((B, Hq, d), s, g, device, shape.dtype)
    if shape.rho_mode == "projection":
        width = Hq * d
        x = torch.randn((B, width), generator=g, device=device, dtype=torch.float32)
        w_r = torch.randn((width, width), generator=g, device=device, dtype=torch.float32)
        w_r.mul_(0.02)
        rho = (x @ w_r.t()).reshape(B, Hq, d).to(shape.dtype)
        del x, w_r
    else:
        rho = _normal((B, Hq, d), 0.1, g, device, shape.dtype)
    if shape.ragged:
        lo = math.ceil(0.5 * shape.ctx)
        seqlens = torch.randint(lo, shape.ctx + 1, (B,), generator=g, device=device,
                                dtype=torch.int64).to(torch.int32)
    else:
        seqlens = torch.full((B,), shape.ctx, dtype=torch.int32, device=device)
    ks, vs = [], []
    for _ in range(max(1, copies)):
        ks.append(_normal((B, S, Hkv, d), s, g, device, shape.dtype))
        vs.append(_normal((B, S, Hkv, d), s, g, device, shape.dtype))
    out = {"q": q, "rho": rho, "k_cache": ks[0], "v_cache": vs[0], "seqlens": seqlens}
    if copies > 1:
        out["k_caches"] = ks
        out["v_caches"] = vs
    return out


def make_probe_inputs(lead: Tuple[int, ...], d_model: int, n_out: int, seed: int = 0,
                      device="cpu", dtype=torch.bfloat16, w_std: float = 0.02
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Layer inputs x [*lead, d_model] ~ N(0, 1) and a projection W_R
    [n_out, d_model] ~ N(0, w_std^2) (the decode workload's probe recipe:
    width 2048, std 0.02), rounded to dtype."""
    g = _gen(device, seed)
    x = _normal(tuple(lead) + (d_model,), 1.0, g, device, dtype)
    w = _normal((n_out, d_model), w_std, g, device, dtype)
    return x, w


def sample_rows_prefill(shape: PrefillShape, n: int, seed: int = 1,
                        stratified: bool = True) -> np.ndarray:
    """n seeded (b, h, i) rows; with ``stratified`` row k lies in [kL/n, (k+1)L/n)."""
    rng = np.random.default_rng(seed)
    b = rng.integers(0, shape.B, n)
    h = rng.integers(0, shape.Hq, n)
    if stratified and n <= shape.L:
        edges = (np.arange(n + 1) * shape.L) // n
        i = np.array([rng.integers(edges[k], max(edges[k + 1], edges[k] + 1)) for k in range(n)])
    else:
        i = rng.integers(0, shape.L, n)
    return np.stack([b, h, i], axis=1).astype(np.int64)


def sample_rows_decode(B: int, Hq: int, n: int, seed: int = 1) -> np.ndarray:
    """min(n, B*Hq) distinct seeded (b, h) rows."""
    rng = np.random.default_rng(seed)
    total = B * Hq
    idx = rng.choice(total, size=min(n, total), replace=False)
    return np.stack([idx // Hq, idx % Hq], axis=1).astype(np.int64)

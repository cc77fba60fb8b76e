"""Pins for the oracle's probe projection and prefill gradients: checks against
facts fixed outside the oracle itself.

* probe projection rho = W_R x (page 1 "Parallax: Parameterized Local Linear
  Attention Gives Transformers a 'Second Eye'", section 1.3: one extra
  projection matrix; page 3 "Parallax keeps softmax, adds covariance
  correction branch": rho_i = W_R x_i): brute force in pure-Python loops on
  tiny shapes, the identity and zero matrices, and W_R = 0 composed with the
  operator giving softmax attention (page 3: W_R = 0 recovers softmax).
* gradients of the prefill operator (the pages print none): central finite
  differences of the forward oracle; fp64 torch autograd of the operator
  written from its definition with the explicit covariance matrix; at
  rho = 0, fp64 autograd of torch's scaled dot-product attention.

Each pin takes an ``oracle.Oracle`` handle; the same functions run against the
real oracle (tests/test_oracle_ext.py) and against copies with planted
mistakes (tests/test_oracle_mutants.py).
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F


def _close(a, b, atol, rtol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    tol = atol + rtol * (float(np.max(np.abs(b))) if b.size else 0.0)
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.3e}"


# ------------------------------------------------------------------- projection
def pin_probe_brute_force(O):
    """rho[m][n] = sum_k W_R[n][k] x[m][k], by plain Python loops."""
    rng = np.random.default_rng(41)
    for M, N, K in ((1, 1, 1), (3, 4, 5), (2, 7, 3)):
        x = rng.standard_normal((M, K))
        w = rng.standard_normal((N, K))
        ref = [[sum(w[n][kk] * x[m][kk] for kk in range(K)) for n in range(N)] for m in range(M)]
        _close(O.probe(x, w), ref, atol=1e-12, what=f"probe {M}x{N}x{K}")


def pin_probe_identity_and_zero(O):
    """W_R = I gives rho = x; W_R = 0 gives rho = 0; leading dims of x are kept."""
    rng = np.random.default_rng(42)
    x = rng.standard_normal((2, 3, 6))
    _close(O.probe(x, np.eye(6)), x, atol=0.0, what="identity")
    _close(O.probe(x, np.zeros((4, 6))), np.zeros((2, 3, 4)), atol=0.0, what="zero")
    perm = np.eye(6)[[5, 0, 3, 1, 4, 2]]
    _close(O.probe(x, perm), x[..., [5, 0, 3, 1, 4, 2]], atol=0.0, what="permutation")


def pin_zero_projection_is_softmax(O):
    """rho = W_R x with W_R = 0, through the operator: softmax attention
    (page 3: W_R = 0 recovers softmax).  Library check: torch SDPA in fp64."""
    rng = np.random.default_rng(43)
    B, L, Hq, Hkv, d, dm = 1, 9, 2, 1, 4, 8
    x = rng.standard_normal((B, L, dm))
    rho = O.probe(x, np.zeros((Hq * d, dm))).reshape(B, L, Hq, d)
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    out, _ = O.prefill(q, rho, k, v, True, 0.4)
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.4)
    _close(out, ref.permute(0, 2, 1, 3).numpy(), atol=1e-12, what="W_R = 0")


# -------------------------------------------------------------------- gradients
def _inputs(seed, B=1, L=6, Hq=2, Hkv=1, d=3, rho_std=0.7):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, L, Hq, d))
    rho = rng.standard_normal((B, L, Hq, d)) * rho_std
    k = rng.standard_normal((B, L, Hkv, d))
    v = rng.standard_normal((B, L, Hkv, d))
    g = rng.standard_normal((B, L, Hq, d))
    return q, rho, k, v, g


def pin_bwd_finite_differences(O):
    """Every gradient entry equals the central difference of sum(g * out) from
    the forward oracle (explicit covariance form), causal and not, GQA."""
    for causal in (True, False):
        q, rho, k, v, g = _inputs(44 + causal, B=1, L=5, Hq=2, Hkv=1, d=3)
        scale = 0.6
        grads = O.prefill_bwd(q, rho, k, v, g, causal, scale)
        args = {"q": q, "rho": rho, "k": k, "v": v}
        eps = 1e-5
        for (name, arr), gr in zip(args.items(), grads):
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                vals = []
                for sgn in (1.0, -1.0):
                    a = arr.copy()
                    a[idx] += sgn * eps
                    kw = dict(args, **{name: a})
                    out, _ = O.prefill(kw["q"], kw["rho"], kw["k"], kw["v"], causal, scale)
                    vals.append(float((out * g).sum()))
                num[idx] = (vals[0] - vals[1]) / (2 * eps)
            _close(gr, num, atol=1e-7, rtol=1e-7, what=f"d{name} causal={causal}")


def _explicit_forward_torch(q, rho, k, v, causal, scale):
    """The operator from its definition: per row, the softmax-weighted
    population covariance matrix of keys and values, contracted with rho on the
    key side, subtracted from the softmax output (torch fp64, autograd)."""
    B, L, Hq, d = q.shape
    G = Hq // k.shape[2]
    rows = []
    for b in range(B):
        for i in range(L):
            per_head = []
            for h in range(Hq):
                n = i + 1 if causal else L
                K = k[b, :n, h // G]
                V = v[b, :n, h // G]
                a = torch.softmax(scale * (K @ q[b, i, h]), dim=0)
                mu = a @ K
                o = a @ V
                cov = (a[:, None] * (K - mu)).T @ (V - o)   # d_k x d_v
                per_head.append(o - cov.T @ rho[b, i, h])
            rows.append(torch.stack(per_head))
    return torch.stack(rows).reshape(B, L, Hq, d)


def pin_bwd_autograd_explicit_definition(O):
    """Gradients equal fp64 torch autograd of the operator written from its
    definition (explicit covariance matrix), causal and not, GQA."""
    for causal in (True, False):
        q, rho, k, v, g = _inputs(46 + causal, B=2, L=7, Hq=4, Hkv=2, d=4)
        scale = 0.45
        ts = [torch.tensor(a, requires_grad=True) for a in (q, rho, k, v)]
        out = _explicit_forward_torch(*ts, causal, scale)
        (out * torch.from_numpy(g)).sum().backward()
        grads = O.prefill_bwd(q, rho, k, v, g, causal, scale)
        for name, t, gr in zip(("q", "rho", "k", "v"), ts, grads):
            _close(gr, t.grad.numpy(), atol=1e-11, rtol=1e-11, what=f"d{name} causal={causal}")


def pin_bwd_rho_zero_is_softmax_attention(O):
    """rho = 0: dq, dk, dv equal fp64 autograd of torch's scaled dot-product
    attention (page 3: W_R = 0 recovers softmax)."""
    q, _, k, v, g = _inputs(48, B=1, L=8, Hq=2, Hkv=2, d=5)
    rho = np.zeros_like(q)
    for causal in (True, False):
        qt, kt, vt = (torch.tensor(a, requires_grad=True).permute(0, 2, 1, 3) for a in (q, k, v))
        qt.retain_grad()
        kt.retain_grad()
        vt.retain_grad()
        out = F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=0.3)
        (out * torch.from_numpy(g).permute(0, 2, 1, 3)).sum().backward()
        dq, _, dk, dv = O.prefill_bwd(q, rho, k, v, g, causal, 0.3)
        _close(dq, qt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=1e-12, what="dq")
        _close(dk, kt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=1e-12, what="dk")
        _close(dv, vt.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12, rtol=1e-12, what="dv")


PROBE_PINS = [pin_probe_brute_force, pin_probe_identity_and_zero, pin_zero_projection_is_softmax]
BWD_PINS = [pin_bwd_finite_differences, pin_bwd_autograd_explicit_definition,
            pin_bwd_rho_zero_is_softmax_attention]
ALL_EXT_PINS = PROBE_PINS + BWD_PINS

"""Pins for the oracle: checks against facts fixed outside the oracle itself.

Each pin takes an ``oracle.Oracle`` handle and a form ("explicit" or
"expanded") and raises AssertionError when the oracle disagrees with

* a library routine that computes a special case (torch's scaled dot-product
  attention for rho = 0, numpy's weighted covariance, scipy's logsumexp,
  numpy's weighted least squares for LLA's solved probe),
* a closed form derived by hand (one key, two keys, uniform weights),
* an invariant of the definition (key translation, value shift, linearity in
  rho, key permutation, grouped heads = repeated heads, causal row = prefix).

The same functions run against the real oracle (tests/test_oracle.py) and
against copies of it with planted mistakes (tests/test_oracle_mutants.py), which
must each fail at least one pin.

Sources of the facts: page 1 "Parallax: Parameterized Local Linear Attention
Gives Transformers a 'Second Eye'" (1.1 softmax attention, 1.2 LLA's local
linear hypothesis, 1.3 the operator and the solved probe, 2.1 the taxonomy:
zero probe = softmax, uniform weighting at h -> infinity) and page 3 "Parallax
keeps softmax, adds covariance correction branch" (W_R = 0 recovers softmax).
"""
from __future__ import annotations

import numpy as np
import scipy.special
import torch
import torch.nn.functional as F

ATOL = 1e-10


def _close(a, b, atol=ATOL, rtol=1e-10, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    tol = atol + rtol * (np.max(np.abs(b)) if b.size else 0.0)
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.3e}"


def _rand(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


# ----------------------------------------------------------------------------
def pin_rho_zero_is_softmax(O, form):
    """rho = 0 gives softmax attention exactly (page 3: W_R = 0 recovers
    softmax; page 1 2.1: zero probe + softmax weighting = softmax attention).
    Library check: torch scaled_dot_product_attention in fp64, with GQA heads
    repeated, causal and not."""
    rng = np.random.default_rng(11)
    for causal in (True, False):
        for G in (1, 2, 4):
            B, L, Hkv, dk, dv = 2, 19, 2, 6, 5
            Hq = Hkv * G
            q = _rand(rng, B, L, Hq, dk)
            k = _rand(rng, B, L, Hkv, dk)
            v = _rand(rng, B, L, Hkv, dv)
            rho = np.zeros((B, L, Hq, dk))
            scale = 0.37
            out, lse = O.prefill(q, rho, k, v, causal, scale, form=form)
            qt = torch.from_numpy(q).permute(0, 2, 1, 3)
            kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
            vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
            ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
            _close(out, ref.permute(0, 2, 1, 3).numpy(), what=f"rho=0 causal={causal} G={G}")
            sc = scale * torch.einsum("bhid,bhjd->bhij", qt, kt)
            if causal:
                sc = sc.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), -np.inf)
            _close(lse, torch.logsumexp(sc, dim=-1).numpy(), what="lse")


def pin_weighted_covariance(O, form):
    """Sigma_KV is the softmax-weighted population covariance of keys and
    values (page 1 1.3 "weighted covariance of K and V"; 2.1 "softmax
    weighting"), contracted with rho on the key side.  Library check: numpy.cov
    with aweights and bias=True, weights from scipy.special.softmax."""
    rng = np.random.default_rng(12)
    for dk, dv in ((3, 5), (5, 3), (4, 4)):
        n = 9
        q = _rand(rng, dk)
        rho = _rand(rng, dk)
        K = _rand(rng, n, dk)
        V = _rand(rng, n, dv)
        scale = 0.8
        a = scipy.special.softmax(scale * K @ q)
        joint = np.cov(np.concatenate([K, V], axis=1).T, aweights=a, bias=True)
        sigma_kv = joint[:dk, dk:]
        o = np.average(V, axis=0, weights=a)
        ref = o - sigma_kv.T @ rho
        out, lse = O.rows(q[None], rho[None], K[None], V[None], [0], [n], scale, form)
        _close(out[0], ref, what=f"weighted covariance dk={dk} dv={dv}")
        _close(lse[0], scipy.special.logsumexp(scale * K @ q), what="lse")


def pin_lla_solved_probe(O, form):
    """With LLA's solved probe rho* = Sigma_KK^-1 (mu - q) (page 1 1.3: the
    optimal probe Sigma^-1 mu, measured from the query), the operator equals
    the intercept of the softmax-weighted local linear fit v ~ b + W^T (k - q)
    (page 1 1.2: hypothesis b + W(x - q)).  Library check: numpy.linalg.lstsq on
    sqrt(a)-scaled rows.  This fixes the sign, the centring of both sides, the
    key-side contraction (d_k != d_v) and the population normalisation."""
    rng = np.random.default_rng(13)
    for dk, dv in ((3, 5), (4, 2), (4, 4)):
        n = 14
        q = _rand(rng, dk)
        K = _rand(rng, n, dk)
        V = _rand(rng, n, dv)
        scale = 0.5
        a = scipy.special.softmax(scale * K @ q)
        mu = a @ K
        sigma_kk = np.cov(K.T, aweights=a, bias=True)
        rho = np.linalg.solve(sigma_kk, mu - q)
        X = np.concatenate([np.ones((n, 1)), K - q], axis=1)
        w = np.sqrt(a)[:, None]
        beta = np.linalg.lstsq(w * X, w * V, rcond=None)[0]
        out, _ = O.rows(q[None], rho[None], K[None], V[None], [0], [n], scale, form)
        _close(out[0], beta[0], atol=1e-9, what=f"LLA intercept dk={dk} dv={dv}")


def pin_single_and_two_keys(O, form):
    """One key: out = v_0 (a = 1, the covariance vanishes).  Two keys, by hand:
    Sigma_KV = a0 a1 (k0 - k1)(v0 - v1)^T, so out = o - a0 a1 (t0 - t1)(v0 - v1)
    with t = rho . k."""
    rng = np.random.default_rng(14)
    dk, dv = 4, 3
    q, rho = _rand(rng, dk), _rand(rng, dk)
    K, V = _rand(rng, 2, dk), _rand(rng, 2, dv)
    out, lse = O.rows(q[None], rho[None], K[None], V[None], [0], [1], 0.9, form)
    _close(out[0], V[0], what="single key")
    _close(lse[0], 0.9 * K[0] @ q, what="single key lse")
    scale = 0.9
    s0, s1 = scale * K[0] @ q, scale * K[1] @ q
    a0 = 1.0 / (1.0 + np.exp(s1 - s0))
    a1 = 1.0 - a0
    t0, t1 = rho @ K[0], rho @ K[1]
    o = a0 * V[0] + a1 * V[1]
    ref = o - a0 * a1 * (t0 - t1) * (V[0] - V[1])
    out, _ = O.rows(q[None], rho[None], K[None], V[None], [0], [2], scale, form)
    _close(out[0], ref, what="two keys")


def pin_uniform_weights(O, form):
    """scale = 0 (bandwidth h -> infinity, page 1 2.1: uniform weighting):
    out = mean(v) - cov_pop(t, v) with t = K rho.  Library: numpy.cov(bias)."""
    rng = np.random.default_rng(15)
    n, dk, dv = 11, 5, 3
    q, rho = _rand(rng, dk), _rand(rng, dk)
    K, V = _rand(rng, n, dk), _rand(rng, n, dv)
    t = K @ rho
    c = np.cov(np.concatenate([t[:, None], V], axis=1).T, bias=True)[0, 1:]
    ref = V.mean(axis=0) - c
    out, lse = O.rows(q[None], rho[None], K[None], V[None], [0], [n], 0.0, form)
    _close(out[0], ref, what="uniform weights")
    _close(lse[0], np.log(n), what="uniform lse")


def pin_invariances(O, form):
    """Key translation leaves out unchanged (softmax shift invariance and
    centring); a value shift shifts out by the same vector (the weights
    1 + tbar - t_j sum to one); out - o_SA is linear in rho; a permutation of the
    key/value rows leaves out unchanged."""
    rng = np.random.default_rng(16)
    n, dk, dv = 10, 4, 6
    q, rho = _rand(rng, dk), _rand(rng, dk)
    K, V = _rand(rng, n, dk), _rand(rng, n, dv)
    sc = 0.7
    base, _ = O.rows(q[None], rho[None], K[None], V[None], [0], [n], sc, form)
    ck = _rand(rng, dk)
    tr, _ = O.rows(q[None], rho[None], (K + ck)[None], V[None], [0], [n], sc, form)
    _close(tr, base, atol=1e-9, what="key translation")
    cv = _rand(rng, dv)
    sh, _ = O.rows(q[None], rho[None], K[None], (V + cv)[None], [0], [n], sc, form)
    _close(sh, base + cv, atol=1e-9, what="value shift")
    zero, _ = O.rows(q[None], np.zeros((1, dk)), K[None], V[None], [0], [n], sc, form)
    lam = -2.5
    lin, _ = O.rows(q[None], (lam * rho)[None], K[None], V[None], [0], [n], sc, form)
    _close(lin - zero, lam * (base - zero), atol=1e-9, what="linearity in rho")
    perm = rng.permutation(n)
    pm, _ = O.rows(q[None], rho[None], K[perm][None], V[perm][None], [0], [n], sc, form)
    _close(pm, base, atol=1e-9, what="key permutation")


def pin_layouts(O, form):
    """Grouped-query heads equal multi-head attention with each KV head
    repeated G times; causal row i equals non-causal attention over keys 0..i;
    decode at seqlen i+1 equals prefill row i; seqlen 0 gives 0 and -inf."""
    rng = np.random.default_rng(17)
    B, L, Hkv, G, d = 2, 13, 2, 3, 4
    Hq = Hkv * G
    q, rho = _rand(rng, B, L, Hq, d), _rand(rng, B, L, Hq, d)
    k, v = _rand(rng, B, L, Hkv, d), _rand(rng, B, L, Hkv, d)
    sc = 0.6
    gqa, lse_g = O.prefill(q, rho, k, v, True, sc, form=form)
    mha, lse_m = O.prefill(q, rho, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), True, sc,
                           form=form)
    _close(gqa, mha, what="GQA = repeated MHA")
    _close(lse_g, lse_m, what="GQA lse")
    for i in (0, 5, L - 1):
        pre, _ = O.prefill(q[:, :i + 1], rho[:, :i + 1], k[:, :i + 1], v[:, :i + 1], False, sc,
                           form=form)
        _close(gqa[:, i], pre[:, i], what=f"causal row {i} = prefix")
        seq = np.full(B, i + 1, dtype=np.int32)
        dec, _ = O.decode(q[:, i], rho[:, i], k, v, seq, sc, form=form)
        _close(dec, gqa[:, i], what=f"decode seqlen {i + 1} = prefill row {i}")
    seq = np.array([0, 1], dtype=np.int32)
    dec, lse = O.decode(q[:, 3], rho[:, 3], k, v, seq, sc, form=form)
    _close(dec[0], np.zeros((Hq, d)), what="empty key set")
    assert np.all(np.isneginf(lse[0])), "empty key set lse must be -inf"
    _close(dec[1], np.repeat(v[1, 0], G, axis=0), what="seqlen 1")


def pin_forms_agree(O, form):
    """The explicit covariance form and the expanded streaming form agree
    (o - Sigma_KV^T rho = o - (sum a t v - tbar o), by expanding the product)."""
    rng = np.random.default_rng(18)
    R, P, S, dk, dv = 6, 3, 40, 7, 5
    q, rho = _rand(rng, R, dk), _rand(rng, R, dk)
    K, V = _rand(rng, P, S, dk), _rand(rng, P, S, dv)
    rs = rng.integers(0, P, R)
    rn = rng.integers(1, S + 1, R)
    e, le = O.rows(q, rho, K, V, rs, rn, 0.45, "explicit")
    x, lx = O.rows(q, rho, K, V, rs, rn, 0.45, "expanded")
    _close(e, x, atol=1e-11, what="explicit vs expanded")
    _close(le, lx, what="lse forms")


ALL_PINS = [pin_rho_zero_is_softmax, pin_weighted_covariance, pin_lla_solved_probe,
            pin_single_and_two_keys, pin_uniform_weights, pin_invariances, pin_layouts,
            pin_forms_agree]

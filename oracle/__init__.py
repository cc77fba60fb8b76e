"""Oracle: slow, plain fp64 CPU reference for Parallax attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` may import this package.  The product path
(``covariance_corrected_softmax_b200``) never imports it and shares no code with
it; the only thing both sides share is the seeded input generator module, which
holds none of the method's arithmetic.

The arithmetic lives in ``plx_oracle.c`` (fp64, one query row at a time).  This
module only marshals layouts into the C routine's "key stream" form and applies
the two layout readings the pages leave open:

* GQA head mapping: query head ``h`` reads key/value head ``h // (H_q // H_kv)``
  (consecutive query heads share a KV head).  The pages never mention grouped
  heads; this is the plainest reading of a multi-head operator with fewer KV
  heads than query heads.
* Key sets: causal prefill row ``i`` sees keys ``0..i``; non-causal sees all
  ``L``; decode of batch ``b`` sees cache rows ``0..seqlen_b-1`` with ``seqlen_b``
  clamped to ``[0, S_max]``; an empty set gives ``out = 0`` and ``lse = -inf``.

Operator (page 1 "Parallax: Parameterized Local Linear Attention Gives
Transformers a 'Second Eye'", section 1.3; page 3 "Parallax keeps softmax, adds
covariance correction branch"): ``out_i = o_SA,i - Sigma_KV^(i)^T rho_i`` with
``Sigma_KV^(i) = sum_j a_ij (k_j - mu_i)(v_j - o_SA,i)^T``.

Also here: the probe projection ``rho = W_R x`` (page 1 section 1.3: one extra
projection matrix; page 3: rho_i = W_R x_i), and the gradients of the prefill
operator (the pages print none; the derivation is written out in
``plx_oracle.c``), pinned by central finite differences of the forward and by
fp64 autograd of the explicit-covariance definition; ``prefill_bwd_sampled``
evaluates selected entries of the same gradients in numpy, row by row, and is
pinned against the C routine.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "plx_oracle.c")
_LIB = os.path.join(_HERE, "libplx_oracle.so")

FORM_EXPLICIT = 0  # forms the d_k x d_v covariance matrix (the definition)
FORM_EXPANDED = 1  # o - (sum a t v - (sum a t) o): the one-pass rewrite
_FORMS = {"explicit": FORM_EXPLICIT, "expanded": FORM_EXPANDED}


def build(src: str = _SRC, out: str = _LIB, extra_flags: Sequence[str] = ()) -> str:
    """Compile the C oracle with gcc into a shared library; returns its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", *extra_flags,
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class Oracle:
    """Handle on one compiled copy of the C oracle (tests may load mutants)."""

    def __init__(self, lib_path: str = _LIB):
        if lib_path == _LIB and (not os.path.exists(_LIB)
                                 or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
            build()
        self.path = lib_path
        self._lib = ctypes.CDLL(lib_path)
        f = self._lib.plxo_rows
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        f.argtypes = [dp, dp, dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                      ctypes.c_int, ip, ip, ctypes.c_int64, ctypes.c_double,
                      ctypes.c_int, dp, dp, ctypes.c_int]
        f.restype = ctypes.c_int
        self._rows = f
        i64 = ctypes.c_int64
        f = self._lib.plxo_probe
        f.argtypes = [dp, dp, dp, i64, i64, i64]
        f.restype = ctypes.c_int
        self._probe = f
        f = self._lib.plxo_prefill_bwd
        f.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64, ctypes.c_int,
                      ctypes.c_double, dp, dp, dp, dp, ctypes.c_int]
        f.restype = ctypes.c_int
        self._bwd = f

    # ------------------------------------------------------------------ core
    def rows(self, q, rho, k, v, row_stream, row_nkeys, scale: float,
             form: str = "explicit", threads: Optional[int] = None
             ) -> Tuple[np.ndarray, np.ndarray]:
        """Evaluate query rows against key/value streams.

        q, rho: [R, dk]; k: [P, S, dk]; v: [P, S, dv]; row_stream, row_nkeys: [R].
        Returns (out [R, dv], lse [R]) in float64.
        """
        q = _f64(q)
        rho = _f64(rho)
        k = _f64(k)
        v = _f64(v)
        R, dk = q.shape
        P, S, dk2 = k.shape
        dv = v.shape[2]
        assert rho.shape == (R, dk) and dk2 == dk and v.shape[:2] == (P, S)
        rs = np.ascontiguousarray(np.asarray(row_stream, dtype=np.int64).reshape(R))
        rn = np.ascontiguousarray(np.asarray(row_nkeys, dtype=np.int64).reshape(R))
        out = np.zeros((R, dv), dtype=np.float64)
        lse = np.zeros((R,), dtype=np.float64)
        if R == 0:
            return out, lse
        if P == 0:  # no streams: every row must be empty
            assert np.all(rn == 0)
            k = np.zeros((1, max(S, 1), dk))
            v = np.zeros((1, max(S, 1), dv))
            P, S = 1, max(S, 1)
            rs = np.zeros_like(rs)
        rc = self._rows(_p(q), _p(rho), _p(k), _p(v), P, S, dk, dv,
                        rs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                        rn.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
                        float(scale), _FORMS[form], _p(out), _p(lse),
                        int(threads or default_threads()))
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return out, lse

    # --------------------------------------------------------------- layouts
    def prefill(self, q, rho, k, v, causal: bool, scale: float, rows=None,
                form: str = "explicit", threads: Optional[int] = None):
        """Prefill rows.  q, rho: [B, L, Hq, dk]; k: [B, L, Hkv, dk]; v: [B, L, Hkv, dv].

        rows: None (all rows; returns out [B, L, Hq, dv], lse [B, Hq, L]) or an
        int array [R, 3] of (b, h, i) (returns out [R, dv], lse [R]).
        """
        B, L, Hq, dk = q.shape
        Hkv = k.shape[2]
        assert Hq % Hkv == 0, "H_q must be a multiple of H_kv"
        G = Hq // Hkv
        full = rows is None
        if full:
            bb, ii, hh = np.meshgrid(np.arange(B), np.arange(L), np.arange(Hq), indexing="ij")
            rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
        hk = h // G
        nkeys = (i + 1) if causal else np.full_like(i, L)
        sid, ks, vs = _streams(k, v, b, hk, int(nkeys.max()) if len(nkeys) else 0)
        out, lse = self.rows(_take(q, (b, i, h)), _take(rho, (b, i, h)), ks, vs, sid, nkeys,
                             scale, form, threads)
        if full:
            out = out.reshape(B, L, Hq, -1)
            lse = lse.reshape(B, L, Hq).transpose(0, 2, 1).copy()
        return out, lse

    def decode(self, q, rho, k_cache, v_cache, seqlens, scale: float, rows=None,
               form: str = "explicit", threads: Optional[int] = None):
        """Single-token decode.  q, rho: [B, Hq, dk]; caches: [B, S_max, Hkv, d].

        rows: None (all; returns out [B, Hq, dv], lse [B, Hq]) or an int array
        [R, 2] of (b, h) (returns out [R, dv], lse [R]).
        """
        B, Hq, dk = q.shape
        S_max, Hkv = k_cache.shape[1], k_cache.shape[2]
        assert Hq % Hkv == 0, "H_q must be a multiple of H_kv"
        G = Hq // Hkv
        sl = np.clip(np.asarray(_np(seqlens)).astype(np.int64).reshape(B), 0, S_max)
        full = rows is None
        if full:
            bb, hh = np.meshgrid(np.arange(B), np.arange(Hq), indexing="ij")
            rows = np.stack([bb.ravel(), hh.ravel()], axis=1)
        rows = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        b, h = rows[:, 0], rows[:, 1]
        nkeys = sl[b]
        sid, ks, vs = _streams(k_cache, v_cache, b, h // G, int(nkeys.max()) if len(nkeys) else 0)
        out, lse = self.rows(_take(q, (b, h)), _take(rho, (b, h)), ks, vs, sid, nkeys,
                             scale, form, threads)
        if full:
            out = out.reshape(B, Hq, -1)
            lse = lse.reshape(B, Hq)
        return out, lse


def _probe(self, x, w):
    """rho = x W_R^T: x [..., K], w [N, K] -> [..., N] (fp64)."""
    x = _f64(x)
    w = _f64(w)
    lead, K = x.shape[:-1], x.shape[-1]
    N = w.shape[0]
    assert w.shape == (N, K), "W_R must be [N, K] with K the width of x"
    xm = np.ascontiguousarray(x.reshape(-1, K))
    out = np.zeros((xm.shape[0], N), dtype=np.float64)
    if self._probe(_p(xm), _p(w), _p(out), xm.shape[0], N, K) != 0:
        raise ValueError("oracle rejected its arguments")
    return out.reshape(*lead, N)


def _prefill_bwd(self, q, rho, k, v, dout, causal: bool, scale: float,
                 threads: Optional[int] = None):
    """Gradients of sum(dout * out) for the prefill operator.

    q, rho, dout [B, L, Hq, d]; k, v [B, L, Hkv, d].  Returns (dq, drho, dk,
    dv) in float64, shaped like q, rho, k, v.
    """
    q, rho, k, v, g = (_f64(t) for t in (q, rho, k, v, dout))
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    assert rho.shape == q.shape and g.shape == q.shape and k.shape == (B, L, Hkv, d)
    assert v.shape == k.shape and Hq % Hkv == 0
    dq, dr = np.zeros_like(q), np.zeros_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(k)
    rc = self._bwd(_p(q), _p(rho), _p(k), _p(v), _p(g), B, L, Hq, Hkv, d, int(bool(causal)),
                   float(scale), _p(dq), _p(dr), _p(dk), _p(dv),
                   int(threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return dq, dr, dk, dv


Oracle.probe = _probe
Oracle.prefill_bwd = _prefill_bwd


def _np(x):
    """numpy view of a numpy array or a (CPU or device) torch tensor, exact values."""
    if isinstance(x, np.ndarray):
        return x
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu")
            if x.dtype in (torch.bfloat16, torch.float16):
                x = x.to(torch.float32)  # exact
            return x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(_np(x), dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _take(x, idx):
    """x[idx] for integer index arrays, gathered before any host copy."""
    if isinstance(x, np.ndarray):
        return x[idx]
    import torch
    tidx = tuple(torch.as_tensor(np.asarray(a), dtype=torch.long, device=x.device) for a in idx)
    return _np(x[tidx])


def _streams(k, v, b, hk, n: int):
    """Gather the distinct (batch, kv-head) key/value streams the rows need.

    Only the first ``n`` rows of each needed stream are copied to the host, so
    sampled rows of a large device-resident cache stay cheap.
    """
    pairs = np.stack([b, hk], axis=1)
    uniq, inv = np.unique(pairs, axis=0, return_inverse=True)
    n = max(n, 1)
    ks = np.stack([_f64(k[int(pb), :n, int(ph), :]) for pb, ph in uniq]) if len(uniq) else \
        np.zeros((0, n, k.shape[-1]))
    vs = np.stack([_f64(v[int(pb), :n, int(ph), :]) for pb, ph in uniq]) if len(uniq) else \
        np.zeros((0, n, v.shape[-1]))
    return inv.reshape(-1), ks, vs


def prefill_bwd_sampled(q, rho, k, v, g, causal: bool, scale: float, rows=None, keys=None):
    """Selected entries of the prefill gradients, fp64, in plain numpy one row
    at a time (for large shapes, where the full routine would take too long):
    dq, drho at the query rows ``rows`` [R, 3] of (b, h, i), and dk, dv at the
    key rows ``keys`` [S, 3] of (b, hk, j).  The operator and its gradients are
    those of ``plxo_prefill_bwd`` (derivation in ``plx_oracle.c``): for row i
    with visible keys j, a = softmax(scale q.k), t = rho.k, gv = g.v,
    tbar = sum a t, go = sum a gv, c = 1 + tbar - t, out = sum a c v,
    D = g.out + tbar go, ds = a (c gv + t go - D), dt = a (go - gv);
    dq = scale sum ds k, drho = sum dt k; dk_j = sum over the rows that see key
    j of scale ds q + dt rho; dv_j = sum a c g.  Returns (dq [R, d], drho [R, d],
    dk [S, d], dv [S, d])."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    streams = {}

    def stream(b, hk):
        if (b, hk) not in streams:
            streams[(b, hk)] = (_f64(k[b, :, hk, :]), _f64(v[b, :, hk, :]))
        return streams[(b, hk)]

    cache = {}

    def row(b, h, i):
        if (b, h, i) not in cache:
            K, V = stream(b, h // G)
            n = i + 1 if causal else L
            K, V = K[:n], V[:n]
            qi, ri, gi = _f64(q[b, i, h, :]), _f64(rho[b, i, h, :]), _f64(g[b, i, h, :])
            s = scale * (K @ qi)
            a = np.exp(s - s.max())
            a /= a.sum()
            t = K @ ri
            gv = V @ gi
            tbar = float(a @ t)
            go = float(a @ gv)
            c = 1.0 + tbar - t
            out = (a * c) @ V
            D = float(gi @ out) + tbar * go
            ds = a * (c * gv + t * go - D)
            dt = a * (go - gv)
            cache[(b, h, i)] = (K, qi, ri, gi, a, c, ds, dt)
        return cache[(b, h, i)]

    rows = np.zeros((0, 3), dtype=np.int64) if rows is None else \
        np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    keys = np.zeros((0, 3), dtype=np.int64) if keys is None else \
        np.asarray(keys, dtype=np.int64).reshape(-1, 3)
    dq = np.zeros((len(rows), d))
    drho = np.zeros((len(rows), d))
    for r, (b, h, i) in enumerate(rows):
        K, _, _, _, _, _, ds, dt = row(int(b), int(h), int(i))
        dq[r] = scale * (ds @ K)
        drho[r] = dt @ K
    dk = np.zeros((len(keys), d))
    dv = np.zeros((len(keys), d))
    for r, (b, hk, j) in enumerate(keys):
        b, hk, j = int(b), int(hk), int(j)
        for h in range(hk * G, (hk + 1) * G):
            for i in range(j if causal else 0, L):
                _, qi, ri, gi, a, c, ds, dt = row(b, h, i)
                dk[r] += scale * ds[j] * qi + dt[j] * ri
                dv[r] += a[j] * c[j] * gi
    return dq, drho, dk, dv


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from ``plx_oracle.c`` (compiled on first use if needed)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def prefill(*args, **kw):
    return get().prefill(*args, **kw)


def decode(*args, **kw):
    return get().decode(*args, **kw)


def rows(*args, **kw):
    return get().rows(*args, **kw)


def probe(*args, **kw):
    return get().probe(*args, **kw)


def prefill_bwd(*args, **kw):
    return get().prefill_bwd(*args, **kw)

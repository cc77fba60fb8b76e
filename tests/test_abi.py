"""The C ABI library: it loads, exports what include/plx.h declares, and its
host-side argument checks reject bad calls before touching a GPU."""
import ctypes
import os
import re

import pytest

from covariance_corrected_softmax_b200 import plx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "plx.h")

FAKE = 0x10000  # never dereferenced: every case below fails validation first


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"PLX_API\s+[\w\s\*]+?\b(plx_\w+)\s*\(", text)


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("plx_prefill_fwd", "plx_decode", "plx_decode_workspace_bytes",
              "plx_status_string", "plx_last_cuda_error", "plx_device_error", "plx_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(plx.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(lib, n), f"{n} declared in plx.h but not exported"


def test_status_strings():
    assert plx.status_string(0) == "PLX_OK"
    assert plx.status_string(3) == "PLX_ERR_WORKSPACE_TOO_SMALL"
    assert plx.lib().plx_version() >= 100


def _decode(**kw):
    a = dict(q=FAKE, rho=FAKE, k=FAKE, v=FAKE, sl=FAKE, out=FAKE, B=2, Hq=4, Hkv=2, d=128,
             S=64, dtype=plx.PLX_BF16, scale=1.0, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return plx.lib().plx_decode(a["q"], a["rho"], a["k"], a["v"], a["sl"], a["out"], a["B"],
                                a["Hq"], a["Hkv"], a["d"], a["S"], a["dtype"], a["scale"],
                                a["ws"], a["wsb"], None)


def _prefill(**kw):
    """plx_prefill_fwd, or plx_prefill_fwd_ex when out_dtype is given."""
    a = dict(q=FAKE, rho=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, causal=1, B=1, L=16, Hq=2,
             Hkv=1, d=64, dtype=plx.PLX_F32, out_dtype=None, scale=0.125)
    a.update(kw)
    head = (a["q"], a["rho"], a["k"], a["v"], a["out"], a["lse"], a["causal"], a["B"], a["L"],
            a["Hq"], a["Hkv"], a["d"], a["dtype"])
    if a["out_dtype"] is None:
        return plx.lib().plx_prefill_fwd(*head, a["scale"], None)
    return plx.lib().plx_prefill_fwd_ex(*head, a["out_dtype"], a["scale"], None)


def _prototype(name):
    """Parameter list of a declaration in plx.h, whitespace-normalised."""
    with open(HEADER) as f:
        text = f.read()
    m = re.search(r"PLX_API\s+plx_status\s+" + name + r"\s*\(([^;]*)\)\s*;", text)
    assert m, name
    return [" ".join(p.split()) for p in m.group(1).split(",")]


def test_prefill_fwd_prototype_is_the_specified_one():
    """plx_prefill_fwd(q, rho, k, v, out, lse, causal, B, L, H_q, H_kv, d, dtype,
    softmax_scale, stream): one dtype for q, rho, k, v and out."""
    assert _prototype("plx_prefill_fwd") == [
        "const void* q", "const void* rho", "const void* k", "const void* v", "void* out",
        "float* lse", "int causal", "int B", "int L", "int H_q", "int H_kv", "int d",
        "plx_dtype dtype", "float softmax_scale", "void* stream"]
    ex = _prototype("plx_prefill_fwd_ex")
    assert ex[:13] == _prototype("plx_prefill_fwd")[:13]
    assert ex[13:] == ["plx_dtype out_dtype", "float softmax_scale", "void* stream"]
    assert _prototype("plx_decode") == [
        "const void* q", "const void* rho", "const void* k_cache", "const void* v_cache",
        "const int32_t* seqlens", "void* out", "int B", "int H_q", "int H_kv", "int d",
        "int S_max", "plx_dtype dtype", "float softmax_scale", "void* workspace",
        "size_t workspace_bytes", "void* stream"]


INV = plx.PLX_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("kw", [
    dict(d=96), dict(d=0), dict(Hq=3, Hkv=2), dict(Hq=0), dict(Hkv=0), dict(B=-1), dict(S=0),
    dict(dtype=7), dict(scale=float("nan")), dict(scale=float("inf")), dict(q=None),
    dict(k=None), dict(sl=None), dict(ws=None), dict(out=None), dict(q=FAKE + 8),
    dict(v=FAKE + 4), dict(ws=FAKE + 8), dict(sl=FAKE + 2),
])
def test_decode_rejects(kw):
    assert _decode(**kw) == INV


def test_decode_empty_batch_is_noop():
    assert _decode(B=0, q=None, k=None) == plx.PLX_OK


def _decode_append(**kw):
    a = dict(q=FAKE, rho=FAKE, kn=FAKE, vn=FAKE, k=FAKE, v=FAKE, sl=FAKE, out=FAKE, B=2, Hq=4,
             Hkv=2, d=128, S=64, dtype=plx.PLX_BF16, scale=1.0, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return plx.lib().plx_decode_append(a["q"], a["rho"], a["kn"], a["vn"], a["k"], a["v"],
                                       a["sl"], a["out"], a["B"], a["Hq"], a["Hkv"], a["d"],
                                       a["S"], a["dtype"], a["scale"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(kn=None), dict(vn=None), dict(kn=FAKE + 8), dict(vn=FAKE + 4), dict(d=96),
    dict(Hq=3, Hkv=2), dict(S=0), dict(k=None), dict(sl=FAKE + 2), dict(scale=float("nan")),
])
def test_decode_append_rejects(kw):
    # argument checks come before any device work, so nothing is written
    assert _decode_append(**kw) == INV


def _decode_paged(**kw):
    a = dict(q=FAKE, rho=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, out=FAKE, B=2, Hq=4, Hkv=2,
             d=128, npages=8, ps=16, maxp=4, dtype=plx.PLX_BF16, scale=1.0, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return plx.lib().plx_decode_paged(a["q"], a["rho"], a["kp"], a["vp"], a["bt"], a["sl"],
                                      a["out"], a["B"], a["Hq"], a["Hkv"], a["d"], a["npages"],
                                      a["ps"], a["maxp"], a["dtype"], a["scale"], a["ws"],
                                      a["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(ps=0), dict(ps=8), dict(ps=24), dict(npages=0), dict(maxp=0), dict(bt=None),
    dict(bt=FAKE + 2), dict(kp=None), dict(vp=FAKE + 8), dict(d=96), dict(Hq=3, Hkv=2),
    dict(scale=float("nan")), dict(sl=None),
])
def test_decode_paged_rejects(kw):
    assert _decode_paged(**kw) == INV


def test_decode_paged_too_large_pool_unsupported():
    assert _decode_paged(npages=1 << 27, ps=32) == plx.PLX_ERR_UNSUPPORTED


def test_decode_paged_empty_batch_is_noop():
    assert _decode_paged(B=0, q=None, bt=None) == plx.PLX_OK


def test_decode_append_empty_batch_is_noop():
    assert _decode_append(B=0, q=None, kn=None, vn=None) == plx.PLX_OK


@pytest.mark.parametrize("kw", [
    dict(d=32), dict(Hq=2, Hkv=3), dict(causal=2), dict(L=-1), dict(dtype=3),
    dict(scale=float("nan")), dict(q=None), dict(rho=None), dict(out=None), dict(k=FAKE + 8),
    dict(lse=FAKE + 2), dict(out_dtype=plx.PLX_BF16), dict(out_dtype=5),
    dict(dtype=plx.PLX_BF16, scale=float("inf")), dict(dtype=plx.PLX_BF16, out_dtype=7),
])
def test_prefill_rejects(kw):
    assert _prefill(**kw) == INV


def _prefill_varlen(**kw):
    a = dict(q=FAKE, rho=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, cu=FAKE, n=3, T=300, maxs=128,
             causal=1, Hq=4, Hkv=2, d=128, dtype=plx.PLX_BF16, out_dtype=None, scale=0.1)
    a.update(kw)
    od = a["dtype"] if a["out_dtype"] is None else a["out_dtype"]
    return plx.lib().plx_prefill_varlen(a["q"], a["rho"], a["k"], a["v"], a["out"], a["lse"],
                                        a["cu"], a["n"], a["T"], a["maxs"], a["causal"], a["Hq"],
                                        a["Hkv"], a["d"], a["dtype"], od, a["scale"], None)


@pytest.mark.parametrize("kw", [
    dict(n=-1), dict(T=-1), dict(maxs=-1), dict(d=80), dict(Hq=3, Hkv=2), dict(causal=3),
    dict(cu=None), dict(cu=FAKE + 2), dict(q=None), dict(k=FAKE + 8), dict(lse=FAKE + 1),
    dict(scale=float("nan")), dict(out_dtype=5),
])
def test_prefill_varlen_rejects(kw):
    assert _prefill_varlen(**kw) == INV


def test_prefill_varlen_fp32_unsupported_and_empty_noop():
    assert _prefill_varlen(dtype=plx.PLX_F32) == plx.PLX_ERR_UNSUPPORTED
    assert _prefill_varlen(n=0, q=None) == plx.PLX_OK
    assert _prefill_varlen(T=0, q=None) == plx.PLX_OK


def test_decode_state_and_merge_reject_bad_arguments():
    L = plx.lib()
    # plx_decode_state: no state buffer, misaligned state
    assert L.plx_decode_state(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 4, 2, 128, 64,
                              plx.PLX_BF16, 1.0, FAKE, 1 << 20, None) == INV
    assert L.plx_decode_state(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, 2, 4, 2, 128, 64,
                              plx.PLX_BF16, 1.0, FAKE, 1 << 20, None) == INV
    # plx_merge_states: R < 1, bad d, bad dtype, null pointers; B = 0 is a no-op
    assert L.plx_merge_states(FAKE, 0, FAKE, 2, 4, 128, plx.PLX_BF16, None) == INV
    assert L.plx_merge_states(FAKE, 2, FAKE, 2, 4, 96, plx.PLX_BF16, None) == INV
    assert L.plx_merge_states(FAKE, 2, FAKE, 2, 4, 128, 9, None) == INV
    assert L.plx_merge_states(None, 2, FAKE, 2, 4, 128, plx.PLX_F32, None) == INV
    assert L.plx_merge_states(FAKE, 2, FAKE + 4, 2, 4, 128, plx.PLX_F32, None) == INV
    assert L.plx_merge_states(None, 2, None, 0, 4, 128, plx.PLX_F32, None) == plx.PLX_OK


def test_prefill_empty_is_noop():
    assert _prefill(B=0, q=None) == plx.PLX_OK
    assert _prefill(L=0, q=None) == plx.PLX_OK
    assert _prefill(B=0, q=None, dtype=plx.PLX_BF16, out_dtype=plx.PLX_F32) == plx.PLX_OK


def test_workspace_query_rejects_bad_shapes():
    L = plx.lib()
    assert L.plx_decode_workspace_bytes(1, 3, 2, 128, 64) == 0
    assert L.plx_decode_workspace_bytes(1, 2, 2, 80, 64) == 0
    assert L.plx_decode_workspace_bytes(1, 2, 2, 64, 0) == 0


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "covariance_corrected_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "plx_oracle" not in src and "plxo_" not in src, fn


def test_wait_limit_rejects_out_of_range_values():
    # checked before any device call
    L = plx.lib()
    assert L.plx_set_wait_limit_ns(999) == INV
    assert L.plx_set_wait_limit_ns(61 * 10 ** 9) == INV


def test_probe_projection_rejects():
    L = plx.lib()
    f = L.plx_probe_projection
    assert f(FAKE, FAKE, FAKE, 4, 16, 8, 7, None) == INV             # dtype
    assert f(FAKE, FAKE, FAKE, -1, 16, 8, plx.PLX_BF16, None) == INV  # M
    assert f(FAKE, FAKE, FAKE, 4, 16, 0, plx.PLX_BF16, None) == INV   # K
    assert f(None, FAKE, FAKE, 4, 16, 8, plx.PLX_BF16, None) == INV
    assert f(FAKE, FAKE + 8, FAKE, 4, 16, 8, plx.PLX_BF16, None) == INV
    assert f(FAKE, FAKE, FAKE, 4, 16, 12, plx.PLX_BF16, None) == plx.PLX_ERR_UNSUPPORTED  # K % 8
    assert f(FAKE, FAKE, FAKE, 4, 20, 8, plx.PLX_BF16, None) == plx.PLX_ERR_UNSUPPORTED  # N % 8
    big = 2 ** 31 - 504  # tile row coordinates would pass 2^31
    assert f(FAKE, FAKE, FAKE, big, 16, 8, plx.PLX_BF16, None) == plx.PLX_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 4, big, 8, plx.PLX_BF16, None) == plx.PLX_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 4, 65535 * 16 + 1, 8, plx.PLX_F32, None) == plx.PLX_ERR_UNSUPPORTED
    assert f(None, None, None, 0, 16, 8, plx.PLX_BF16, None) == plx.PLX_OK  # M = 0: no-op


def test_prefill_x_and_decode_x_check_both_steps_first():
    L = plx.lib()
    # bad attention argument (d = 96) with a valid projection: nothing launched
    assert L.plx_prefill_fwd_x(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 2, 1,
                               96, 64, plx.PLX_BF16, 1.0, None) == INV
    # bad projection (x misaligned) with valid attention arguments
    assert L.plx_prefill_fwd_x(FAKE, FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 2,
                               1, 64, 64, plx.PLX_BF16, 1.0, None) == INV
    assert L.plx_prefill_fwd_x(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 2, 1,
                               64, 0, plx.PLX_BF16, 1.0, None) == INV  # d_model
    assert L.plx_decode_x(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, 2, 4, 2, 128, 64,
                          256, plx.PLX_BF16, 1.0, FAKE, 1 << 20, None) == INV  # seqlens
    assert L.plx_decode_x(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 128, 64,
                          255, plx.PLX_BF16, 1.0, FAKE, 1 << 20, None) == plx.PLX_ERR_UNSUPPORTED
    assert L.plx_decode_x(None, None, None, None, None, None, None, None, 0, 4, 2, 128, 64,
                          256, plx.PLX_BF16, 1.0, None, 0, None) == plx.PLX_OK


def _bwd(**kw):
    a = dict(q=FAKE, rho=FAKE, k=FAKE, v=FAKE, g=FAKE, dq=FAKE, dr=FAKE, dk=FAKE,
             dv=FAKE, causal=1, B=1, L=16, Hq=2, Hkv=1, d=64, dtype=plx.PLX_BF16, scale=0.1,
             ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return plx.lib().plx_prefill_bwd(a["q"], a["rho"], a["k"], a["v"], a["g"], a["dq"],
                                     a["dr"], a["dk"], a["dv"], a["causal"], a["B"], a["L"],
                                     a["Hq"], a["Hkv"], a["d"], a["dtype"], a["scale"], a["ws"],
                                     a["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(d=96), dict(Hq=3, Hkv=2), dict(causal=2), dict(L=-1), dict(dtype=5),
    dict(scale=float("nan")), dict(q=None), dict(g=None), dict(dk=None), dict(ws=None),
    dict(dv=FAKE + 8), dict(g=FAKE + 4),
])
def test_prefill_bwd_rejects(kw):
    assert _bwd(**kw) == INV


def test_prefill_bwd_workspace():
    L = plx.lib()
    assert L.plx_prefill_bwd_workspace_bytes(2, 100, 4) == 2 * 100 * 4 * 16
    assert _bwd(wsb=16 * 2 * 16 - 1) == plx.PLX_ERR_WORKSPACE_TOO_SMALL
    assert _bwd(B=0, q=None) == plx.PLX_OK

"""Thin ctypes binding of libplx (the C ABI in include/plx.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory (outputs, decode
workspace) and the current CUDA stream.  There is no fallback: if the library
is missing or a call fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libplx.so")

PLX_OK, PLX_ERR_INVALID_ARGUMENT, PLX_ERR_UNSUPPORTED, PLX_ERR_WORKSPACE_TOO_SMALL, \
    PLX_ERR_CUDA = range(5)
PLX_F32, PLX_BF16 = 0, 1
_DTYPES = {torch.float32: PLX_F32, torch.bfloat16: PLX_BF16}

_lib: Optional[ctypes.CDLL] = None


class PlxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)}"
        if status == PLX_ERR_CUDA:
            msg += f" (cudaError {lib().plx_last_cuda_error()})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded libplx.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m covariance_corrected_softmax_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.plx_prefill_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp]
        L.plx_prefill_fwd.restype = i
        L.plx_prefill_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp]
        L.plx_prefill_fwd_ex.restype = i
        L.plx_decode_workspace_bytes.argtypes = [i, i, i, i, i]
        L.plx_decode_workspace_bytes.restype = sz
        L.plx_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, sz, vp]
        L.plx_decode.restype = i
        L.plx_decode_append.argtypes = [vp] * 8 + [i] * 6 + [f, vp, sz, vp]
        L.plx_decode_append.restype = i
        L.plx_decode_paged.argtypes = [vp] * 7 + [i] * 8 + [f, vp, sz, vp]
        L.plx_decode_paged.restype = i
        L.plx_prefill_varlen.argtypes = [vp] * 7 + [i] * 9 + [f, vp]
        L.plx_prefill_varlen.restype = i
        L.plx_decode_state.argtypes = [vp] * 6 + [i] * 6 + [f, vp, sz, vp]
        L.plx_decode_state.restype = i
        L.plx_merge_states.argtypes = [vp, i, vp, i, i, i, i, vp]
        L.plx_merge_states.restype = i
        L.plx_status_string.argtypes = [i]
        L.plx_status_string.restype = ctypes.c_char_p
        L.plx_last_cuda_error.argtypes = []
        L.plx_last_cuda_error.restype = i
        L.plx_device_error.argtypes = [ctypes.POINTER(i), i]
        L.plx_device_error.restype = i
        L.plx_probe_projection.argtypes = [vp, vp, vp, i, i, i, i, vp]
        L.plx_probe_projection.restype = i
        L.plx_prefill_fwd_x.argtypes = [vp] * 8 + [i] * 8 + [f, vp]
        L.plx_prefill_fwd_x.restype = i
        L.plx_decode_x.argtypes = [vp] * 8 + [i] * 7 + [f, vp, sz, vp]
        L.plx_decode_x.restype = i
        L.plx_prefill_bwd_workspace_bytes.argtypes = [i, i, i]
        L.plx_prefill_bwd_workspace_bytes.restype = sz
        L.plx_prefill_bwd.argtypes = [vp] * 9 + [i] * 7 + [f, vp, sz, vp]
        L.plx_prefill_bwd.restype = i
        L.plx_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.plx_set_wait_limit_ns.restype = i
        L.plx_selftest_wait.argtypes = [vp]
        L.plx_selftest_wait.restype = i
        L.plx_version.argtypes = []
        L.plx_version.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().plx_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != PLX_OK:
        raise PlxError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")
    return _DTYPES[t.dtype]


def _same(ref: torch.Tensor, *ts: torch.Tensor) -> None:
    for t in ts:
        if t.dtype != ref.dtype or t.device != ref.device:
            raise TypeError("q, rho, k and v must share dtype and device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def prefill(q: torch.Tensor, rho: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
            causal: bool = True, softmax_scale: Optional[float] = None,
            return_lse: bool = True, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None, stream=None,
            out_dtype: Optional[torch.dtype] = None
            ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Parallax attention forward: q, rho [B, L, Hq, d]; k, v [B, L, Hkv, d].

    Returns (out [B, L, Hq, d], lse [B, Hq, L] fp32 or None).  softmax_scale
    defaults to 1/sqrt(d); out_dtype defaults to the input dtype (torch.float32
    is also accepted for bf16 inputs).
    """
    _same(q, rho, k, v)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if rho.shape != q.shape or k.shape != (B, L, Hkv, d) or v.shape != k.shape:
        raise ValueError("shape mismatch among q, rho, k, v")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    args = (_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None,
            int(bool(causal)), B, L, Hq, Hkv, d, _dtype_code(q))
    if out.dtype == q.dtype:
        st, name = lib().plx_prefill_fwd(*args, scale, _stream(stream)), "plx_prefill_fwd"
    else:
        st = lib().plx_prefill_fwd_ex(*args, _dtype_code(out), scale, _stream(stream))
        name = "plx_prefill_fwd_ex"
    _check(st, name)
    return out, (lse if return_lse else None)


def prefill_varlen(q: torch.Tensor, rho: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   cu_seqlens: torch.Tensor, max_seqlen: int, causal: bool = True,
                   softmax_scale: Optional[float] = None, return_lse: bool = True,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   stream=None, out_dtype: Optional[torch.dtype] = None
                   ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Packed variable-length forward: q, rho [T, Hq, d]; k, v [T, Hkv, d];
    cu_seqlens int32 [num_seqs + 1] on the device; max_seqlen >= every length.
    Returns (out [T, Hq, d], lse [Hq, T] fp32 or None)."""
    _same(q, rho, k, v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if rho.shape != q.shape or k.shape != (T, Hkv, d) or v.shape != k.shape:
        raise ValueError("shape mismatch among q, rho, k, v")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != q.device or \
            cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 [num_seqs + 1] device tensor")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device)
    st = lib().plx_prefill_varlen(_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(out),
                                  _ptr(lse) if return_lse else None, _ptr(cu_seqlens),
                                  cu_seqlens.numel() - 1, T, int(max_seqlen), int(bool(causal)),
                                  Hq, Hkv, d, _dtype_code(q), _dtype_code(out), scale,
                                  _stream(stream))
    _check(st, "plx_prefill_varlen")
    return out, (lse if return_lse else None)


def probe_projection(x: torch.Tensor, w_r: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """rho = x W_R^T: x [..., K], w_r [N, K] -> [..., N] in x's dtype."""
    _same(x, w_r)
    K = x.shape[-1]
    N = w_r.shape[0]
    if w_r.dim() != 2 or w_r.shape[1] != K:
        raise ValueError("w_r must be [N, K] with K the last dimension of x")
    M = x.numel() // K if K else 0
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=x.dtype, device=x.device)
    st = lib().plx_probe_projection(_ptr(x), _ptr(w_r), _ptr(out), M, N, K, _dtype_code(x),
                                    _stream(stream))
    _check(st, "plx_probe_projection")
    return out


def prefill_x(q: torch.Tensor, x: torch.Tensor, w_r: torch.Tensor, k: torch.Tensor,
              v: torch.Tensor, causal: bool = True, softmax_scale: Optional[float] = None,
              return_lse: bool = True, stream=None
              ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """Forward with rho = x W_R^T computed on the device: q [B, L, Hq, d];
    x [B, L, d_model]; w_r [Hq d, d_model]; k, v [B, L, Hkv, d].  Returns
    (out, rho, lse)."""
    _same(q, x, w_r, k, v)
    B, L, Hq, d = q.shape
    Hkv, dm = k.shape[2], x.shape[-1]
    if x.shape != (B, L, dm) or w_r.shape != (Hq * d, dm) or k.shape != (B, L, Hkv, d) or \
            v.shape != k.shape:
        raise ValueError("shape mismatch among q, x, w_r, k, v")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    rho = torch.empty_like(q)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device) if return_lse else None
    st = lib().plx_prefill_fwd_x(_ptr(q), _ptr(x), _ptr(w_r), _ptr(k), _ptr(v), _ptr(rho),
                                 _ptr(out), _ptr(lse), int(bool(causal)), B, L, Hq, Hkv, d, dm,
                                 _dtype_code(q), scale, _stream(stream))
    _check(st, "plx_prefill_fwd_x")
    return out, rho, lse


def decode_x(q: torch.Tensor, x: torch.Tensor, w_r: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor, seqlens: torch.Tensor, softmax_scale: Optional[float] = None,
             workspace: Optional[torch.Tensor] = None, stream=None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode with rho = x W_R^T computed on the device: q [B, Hq, d];
    x [B, d_model]; w_r [Hq d, d_model].  Returns (out, rho)."""
    _same(q, x, w_r, k_cache, v_cache)
    B, Hq, d = q.shape
    S_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    dm = x.shape[-1]
    if x.shape != (B, dm) or w_r.shape != (Hq * d, dm) or \
            k_cache.shape != (B, S_max, Hkv, d) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch among q, x, w_r, k_cache, v_cache")
    if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B] on the same device")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    rho = torch.empty_like(q)
    out = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, d, S_max, device=q.device)
    st = lib().plx_decode_x(_ptr(q), _ptr(x), _ptr(w_r), _ptr(k_cache), _ptr(v_cache),
                            _ptr(seqlens), _ptr(rho), _ptr(out), B, Hq, Hkv, d, S_max, dm,
                            _dtype_code(q), scale, _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "plx_decode_x")
    return out, rho


def prefill_bwd_workspace_bytes(B: int, L: int, Hq: int) -> int:
    return int(lib().plx_prefill_bwd_workspace_bytes(B, L, Hq))


def prefill_bwd(q: torch.Tensor, rho: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                dout: torch.Tensor, causal: bool = True, softmax_scale: Optional[float] = None,
                grads=None, workspace: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq, drho, dk, dv), fp32, of sum(dout * out) for the forward
    plx.prefill(q, rho, k, v, causal, softmax_scale).  `grads` (four fp32
    tensors shaped like q, rho, k, v) and `workspace` may be passed in to be
    reused across calls."""
    _same(q, rho, k, v, dout)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if rho.shape != q.shape or dout.shape != q.shape or k.shape != (B, L, Hkv, d) or \
            v.shape != k.shape:
        raise ValueError("shape mismatch among q, rho, k, v, dout")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        dq, drho = torch.empty(q.shape, **f32), torch.empty(q.shape, **f32)
        dk, dv = torch.empty(k.shape, **f32), torch.empty(k.shape, **f32)
    else:
        dq, drho, dk, dv = grads
        for t_, ref in ((dq, q), (drho, q), (dk, k), (dv, k)):
            if t_.dtype != torch.float32 or t_.shape != ref.shape or not t_.is_contiguous() or \
                    t_.device != q.device:
                raise ValueError("grads must be contiguous fp32 tensors shaped like q, rho, k, v")
    nws = prefill_bwd_workspace_bytes(B, L, Hq)
    ws = workspace if workspace is not None else \
        torch.empty(max(nws, 16), dtype=torch.uint8, device=q.device)
    st = lib().plx_prefill_bwd(_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(dout),
                               _ptr(dq), _ptr(drho), _ptr(dk), _ptr(dv), int(bool(causal)), B, L,
                               Hq, Hkv, d, _dtype_code(q), scale, _ptr(ws), ws.numel(),
                               _stream(stream))
    _check(st, "plx_prefill_bwd")
    return dq, drho, dk, dv


def decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, S_max: int) -> int:
    return int(lib().plx_decode_workspace_bytes(B, Hq, Hkv, d, S_max))


def decode_workspace(B: int, Hq: int, Hkv: int, d: int, S_max: int,
                     device=None) -> torch.Tensor:
    """A device buffer sized for plx_decode on the current device."""
    n = decode_workspace_bytes(B, Hq, Hkv, d, S_max)
    if n == 0:
        raise ValueError("invalid decode shape")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def decode(q: torch.Tensor, rho: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           seqlens: torch.Tensor, softmax_scale: Optional[float] = None,
           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """Single-token decode: q, rho [B, Hq, d]; caches [B, S_max, Hkv, d];
    seqlens int32 [B] on the device.  Returns out [B, Hq, d]."""
    _same(q, rho, k_cache, v_cache)
    B, Hq, d = q.shape
    S_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    if rho.shape != q.shape or k_cache.shape != (B, S_max, Hkv, d) or \
            v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch among q, rho, k_cache, v_cache")
    if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B] on the same device")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, d, S_max, device=q.device)
    st = lib().plx_decode(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                          _ptr(out), B, Hq, Hkv, d, S_max, _dtype_code(q), scale,
                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check(st, "plx_decode")
    return out


def decode_state(q: torch.Tensor, rho: torch.Tensor, k_cache: torch.Tensor,
                 v_cache: torch.Tensor, seqlens: torch.Tensor,
                 softmax_scale: Optional[float] = None, state: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """decode() over this cache, returning each row's softmax state
    [B, Hq, 2d + 4] fp32 (m, l, z, 0, o, u) instead of the output."""
    _same(q, rho, k_cache, v_cache)
    B, Hq, d = q.shape
    S_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    if rho.shape != q.shape or k_cache.shape != (B, S_max, Hkv, d) or \
            v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch among q, rho, k_cache, v_cache")
    if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B] on the same device")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if state is None:
        state = torch.empty((B, Hq, 2 * d + 4), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, d, S_max, device=q.device)
    st = lib().plx_decode_state(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                _ptr(state), B, Hq, Hkv, d, S_max, _dtype_code(q), scale,
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(st, "plx_decode_state")
    return state


def merge_states(states: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out [B, Hq, d] from states [R, B, Hq, 2d + 4] (decode_state layout)."""
    if states.dtype != torch.float32 or states.dim() != 4 or not states.is_contiguous():
        raise ValueError("states must be a contiguous fp32 [R, B, Hq, 2d + 4] tensor")
    R, B, Hq, w = states.shape
    d = (w - 4) // 2
    if out is None:
        out = torch.empty((B, Hq, d), dtype=out_dtype, device=states.device)
    st = lib().plx_merge_states(_ptr(states), R, _ptr(out), B, Hq, d, _dtype_code(out),
                                _stream(stream))
    _check(st, "plx_merge_states")
    return out


def context_parallel_decode(q: torch.Tensor, rho: torch.Tensor, k_local: torch.Tensor,
                            v_local: torch.Tensor, seqlens_local: torch.Tensor,
                            softmax_scale: Optional[float] = None, group=None,
                            out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """Decode with the context split over the ranks of a torch.distributed group:
    each rank holds a contiguous slice of every sequence's cache (seqlens_local =
    the slice's filled length); the ranks' states are all-gathered (the one
    exchange) and merged.  Every rank returns the full output (out_dtype, by
    default q's).  NCCL groups gather device tensors; other backends (gloo)
    gather through host memory."""
    import torch.distributed as dist
    state = decode_state(q, rho, k_local, v_local, seqlens_local, softmax_scale)
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        states = torch.empty((world,) + tuple(state.shape), dtype=state.dtype,
                             device=state.device)
        dist.all_gather_into_tensor(states, state, group=group)
    else:
        host = state.cpu()
        parts = [torch.empty_like(host) for _ in range(world)]
        dist.all_gather(parts, host, group=group)
        states = torch.stack(parts).to(state.device)
    return merge_states(states, out_dtype=out_dtype or q.dtype)


def decode_paged(q: torch.Tensor, rho: torch.Tensor, k_pages: torch.Tensor,
                 v_pages: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                 softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode over a paged cache: k_pages, v_pages [num_pages, page_size, Hkv, d];
    block_table int32 [B, max_pages] (device); seqlens int32 [B] (device)."""
    _same(q, rho, k_pages, v_pages)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if rho.shape != q.shape or k_pages.shape != (num_pages, page_size, Hkv, d) or \
            v_pages.shape != k_pages.shape:
        raise ValueError("shape mismatch among q, rho, k_pages, v_pages")
    if block_table.dtype != torch.int32 or block_table.device != q.device or \
            block_table.dim() != 2 or block_table.shape[0] != B or \
            not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 [B, max_pages] device tensor")
    if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B] on the same device")
    max_pages = block_table.shape[1]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, d, max_pages * page_size, device=q.device)
    st = lib().plx_decode_paged(_ptr(q), _ptr(rho), _ptr(k_pages), _ptr(v_pages),
                                _ptr(block_table), _ptr(seqlens), _ptr(out), B, Hq, Hkv, d,
                                num_pages, page_size, max_pages, _dtype_code(q), scale,
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(st, "plx_decode_paged")
    return out


def decode_append(q: torch.Tensor, rho: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                  k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor,
                  softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One serving step: k_new, v_new [B, Hkv, d] are written to cache row
    seqlens[b] - 1 (the lengths count the new token), then decode as decode()."""
    _same(q, rho, k_new, v_new, k_cache, v_cache)
    B, Hq, d = q.shape
    S_max, Hkv = k_cache.shape[1], k_cache.shape[2]
    if rho.shape != q.shape or k_cache.shape != (B, S_max, Hkv, d) or \
            v_cache.shape != k_cache.shape or k_new.shape != (B, Hkv, d) or \
            v_new.shape != k_new.shape:
        raise ValueError("shape mismatch among q, rho, k_new, v_new, k_cache, v_cache")
    if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B] on the same device")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = decode_workspace(B, Hq, Hkv, d, S_max, device=q.device)
    st = lib().plx_decode_append(_ptr(q), _ptr(rho), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(seqlens), _ptr(out), B, Hq, Hkv, d, S_max,
                                 _dtype_code(q), scale, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "plx_decode_append")
    return out


def device_error(clear: bool = True) -> int:
    """The kernels' device-side error word (0 = none); synchronises."""
    code = ctypes.c_int(0)
    _check(lib().plx_device_error(ctypes.byref(code), int(clear)), "plx_device_error")
    return code.value


def set_wait_limit_ns(ns: int = 0) -> None:
    """Diagnostic: the limit of every bounded wait in the kernels on the current
    device (0 restores the default, 2 s); synchronises."""
    _check(lib().plx_set_wait_limit_ns(int(ns)), "plx_set_wait_limit_ns")


def selftest_wait(stream=None) -> None:
    """Diagnostic: enqueue a kernel whose one bounded wait can only run out."""
    _check(lib().plx_selftest_wait(_stream(stream)), "plx_selftest_wait")

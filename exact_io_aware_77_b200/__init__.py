"""Exact, IO-aware attention for B200 (sm_100a).

``forward`` and ``backward`` take contiguous bf16 CUDA tensors of shape
[B, H, N, d] (K and V may have fewer heads, H_kv, with H a multiple of H_kv:
multi-query / grouped-query attention) and run the hand-written kernels of
libfa_b200.so on the current torch stream.  torch supplies device memory and
streams only.
"""

from __future__ import annotations

import ctypes
import math

from . import _lib
from ._lib import FAError, STATUS, STATUS_NAMES, load

__all__ = ["forward", "forward_fp8", "backward", "decode", "decode_fp8kv", "decode_workspace_size", "bwd_workspace_size", "check_status", "FAError", "STATUS", "STATUS_NAMES", "load", "default_scale"]


def default_scale(d: int) -> float:
    """1/sqrt(d_k): the scale of the attention formula."""
    return 1.0 / math.sqrt(d)


def _stream_handle(device) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(q, k, v, *rest):
    """q (and o, dO in rest): [B, H, N, d]; k, v: [B, H_kv, N, d] with H a multiple of H_kv.
    Any strides with a contiguous last dimension (the library checks their alignment)."""
    import torch
    for t in (q, k, v) + rest:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.stride(-1) == 1):
            raise ValueError("expected bf16 CUDA tensors of shape [B, H, N, d] with contiguous d")
        if t.device != q.device:
            raise ValueError("device mismatch")
    if any(t.shape != q.shape for t in rest) or k.shape != v.shape:
        raise ValueError("shape mismatch")
    B, H, N, d = q.shape
    if k.shape[0] != B or k.shape[2:] != (N, d) or k.shape[1] < 1 or H % k.shape[1]:
        raise ValueError("k and v must be [B, H_kv, N, d] with H a multiple of H_kv")
    return int(k.shape[1])


def _check_like(t, ref, what: str) -> None:
    """t must be a bf16 tensor shaped like ref, on ref's device, with contiguous d."""
    import torch
    if not (t.dtype == torch.bfloat16 and t.shape == ref.shape and t.dim() == 4 and t.stride(-1) == 1
            and t.device == ref.device):
        raise ValueError(f"{what} must be a bf16 tensor shaped like {tuple(ref.shape)} on {ref.device} "
                         "with contiguous d")


def _check_lse(lse, ref, rows: int) -> None:
    import torch
    if not (lse.dtype == torch.float32 and lse.is_contiguous() and lse.numel() == rows and lse.device == ref.device):
        raise ValueError(f"lse must be a contiguous fp32 tensor of {rows} elements on {ref.device}")


def _check_workspace(ws, ref) -> None:
    """Caller scratch must be a contiguous tensor on ref's device; its size and alignment are
    the library's to check (FA_ERR_WORKSPACE, FA_ERR_ALIGN)."""
    if not (ws.device == ref.device and ws.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous tensor on {ref.device}")


def _raise(name, st):
    if st != _lib.FA_OK:
        raise FAError(name, st)


def forward(q, k, v, scale: float | None = None, causal: bool = False, window: int = 0,
            out=None, lse=None):
    """O, L = attention(Q, K, V); O bf16 [B,H,N,d], L fp32 [B,H,N] (natural-log logsumexp).

    d is 64, 128 or 256."""
    import torch
    H_kv = _check_qkv(q, k, v)
    B, H, N, d = q.shape
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_like(out, q, "out")
    _check_lse(lse, q, B * H * N)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr())
    mask = (scale, int(bool(causal)), int(window), _stream_handle(q.device))
    if not all(t.is_contiguous() for t in (q, k, v, out)):
        st = _lib.strides_array((q, k, v, out))
        _raise("fa_fwd_strided", _lib.fa_fwd_strided(*ptrs, B, H, H_kv, N, d, ctypes.addressof(st), *mask))
    elif H_kv == H:
        _raise("fa_fwd", _lib.fa_fwd(*ptrs, B, H, N, d, *mask))
    else:
        _raise("fa_fwd_gqa", _lib.fa_fwd_gqa(*ptrs, B, H, H_kv, N, d, *mask))
    return out, lse


def forward_fp8(q8, k8, vt8, q_scale: float, k_scale: float, v_scale: float, scale: float | None = None,
                causal: bool = False, window: int = 0, out=None, lse=None):
    """O, L of attention on E4M3 inputs: Q = q_scale E4M3(q8), K = k_scale E4M3(k8),
    V = v_scale E4M3(vt8)^T.

    q8 [B, H, N, 128], k8 [B, H_kv, N, 128], vt8 [B, H_kv, 128, N]: contiguous CUDA tensors of
    torch.uint8 or torch.float8_e4m3fn codes; N a multiple of 16.  Returns O bf16 [B, H, N, 128] and
    L fp32 [B, H, N].
    """
    import torch
    q8, k8, vt8 = (x.view(torch.uint8) if x.dtype == torch.float8_e4m3fn else x for x in (q8, k8, vt8))
    for t in (q8, k8, vt8):
        if not (t.is_cuda and t.dtype == torch.uint8 and t.dim() == 4 and t.is_contiguous() and t.device == q8.device):
            raise ValueError("q8, k8, vt8 must be contiguous E4M3 code tensors on one CUDA device")
    B, H, N, d = q8.shape
    H_kv = int(k8.shape[1])
    if k8.shape != (B, H_kv, N, d) or vt8.shape != (B, H_kv, d, N):
        raise ValueError("k8 must be [B, H_kv, N, d] and vt8 [B, H_kv, d, N]")
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    if not (out.shape == (B, H, N, d) and out.dtype == torch.bfloat16 and out.is_contiguous() and out.device == q8.device):
        raise ValueError("out must be a contiguous bf16 tensor [B, H, N, d] on q8's device")
    _check_lse(lse, q8, B * H * N)
    _raise("fa_fwd_fp8", _lib.fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(), float(q_scale), float(k_scale),
                                         float(v_scale), out.data_ptr(), lse.data_ptr(), B, H, H_kv, N, d, scale,
                                         int(bool(causal)), int(window), _stream_handle(q8.device)))
    return out, lse


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    """Bytes of scratch device memory backward() needs (O(N*d))."""
    n = _lib.fa_bwd_workspace_size(B, H, N, d)
    if n == 0:
        raise ValueError("invalid shape")
    return n


def backward(q, k, v, o, lse, do, scale: float | None = None, causal: bool = False, window: int = 0,
             grads=None, workspace=None, phases: int = 7):
    """dQ (like q), dK, dV (like k) of sum(O o dO), recomputing P from the forward's L.

    ``phases`` selects the steps of the backward (1 preprocess, 2 recompute kernel, 4 dQ
    finalise); running 1, 2, 4 in turn with the same workspace equals the default 7.
    """
    import torch
    H_kv = _check_qkv(q, k, v, o, do)
    B, H, N, d = q.shape
    _check_lse(lse, q, B * H * N)
    scale = default_scale(d) if scale is None else float(scale)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    for g, t, name in zip(grads, (q, k, v), ("dq", "dk", "dv")):
        _check_like(g, t, name)
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, q)
    dq, dk, dv = grads
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    rest = (d, scale, int(bool(causal)), int(window), workspace.data_ptr(),
            workspace.numel() * workspace.element_size())
    if not all(t.is_contiguous() for t in (q, k, v, o, do, dq, dk, dv)):
        st = _lib.strides_array((q, k, v, o, do, dq, dk, dv))
        _raise("fa_bwd_strided", _lib.fa_bwd_strided(*ptrs, B, H, H_kv, N, d, ctypes.addressof(st), scale,
                                                     int(bool(causal)), int(window), workspace.data_ptr(),
                                                     workspace.numel() * workspace.element_size(), int(phases),
                                                     _stream_handle(q.device)))
        return dq, dk, dv
    if H_kv != H:
        _raise("fa_bwd_gqa", _lib.fa_bwd_gqa(*ptrs, B, H, H_kv, N, *rest, int(phases), _stream_handle(q.device)))
        return dq, dk, dv
    args = ptrs + (B, H, N) + rest
    if phases == 7:
        _raise("fa_bwd", _lib.fa_bwd(*args, _stream_handle(q.device)))
    else:
        _raise("fa_bwd_phases", _lib.fa_bwd_phases(*args, int(phases), _stream_handle(q.device)))
    return dq, dk, dv


def decode_workspace_size(B: int, H: int, H_kv: int, N_q: int, N_k: int, d: int, causal: bool = False,
                          window: int = 0) -> int:
    """Bytes of scratch device memory decode() needs (0 when the keys fit one split)."""
    if not (1 <= N_q <= N_k and B >= 1 and H_kv >= 1 and H % H_kv == 0 and d in (64, 128, 256) and window >= 0):
        raise ValueError("invalid shape")
    return _lib.fa_decode_workspace_size(B, H, H_kv, N_q, N_k, d, int(bool(causal)), int(window))


def decode(q, k, v, scale: float | None = None, causal: bool = False, window: int = 0,
           out=None, lse=None, workspace=None):
    """O, L for N_q new query rows over N_k >= N_q keys (a generation step over a K/V cache).

    q: bf16 [B, H, N_q, d]; k, v: bf16 [B, H_kv, N_k, d]; query row i stands at key position
    N_k - N_q + i, where the causal and window masks apply.  Returns O bf16 [B, H, N_q, d] and
    L fp32 [B, H, N_q].  Any strides with a contiguous last dimension.
    """
    import torch
    for t in (q, k, v):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.stride(-1) == 1):
            raise ValueError("expected bf16 CUDA tensors of shape [B, heads, N, d] with contiguous d")
        if t.device != q.device:
            raise ValueError("device mismatch")
    B, H, N_q, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, H_kv, N_k, d]")
    H_kv, N_k = int(k.shape[1]), int(k.shape[2])
    scale = default_scale(d) if scale is None else float(scale)
    need = decode_workspace_size(B, H, H_kv, N_q, N_k, d, causal, window)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    _check_like(out, q, "out")
    _check_lse(lse, q, B * H * N_q)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _check_workspace(workspace, q)
    ws_ptr = workspace.data_ptr() if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = None
    if not all(t.is_contiguous() for t in (q, k, v, out)):
        st = _lib.strides_array((q, k, v, out))
    _raise("fa_fwd_decode", _lib.fa_fwd_decode(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, H_kv, N_q, N_k, d,
        ctypes.addressof(st) if st is not None else 0, scale, int(bool(causal)), int(window), ws_ptr, ws_bytes,
        _stream_handle(q.device)))
    return out, lse


def decode_fp8kv(q, k8, v8, k_scale: float, v_scale: float, scale: float | None = None, causal: bool = False,
                 window: int = 0, out=None, lse=None, workspace=None):
    """decode() over an FP8 key/value cache: K = k_scale * E4M3(k8), V = v_scale * E4M3(v8).

    k8, v8: [B, H_kv, N_k, d] E4M3 codes (torch.uint8 or torch.float8_e4m3fn), strides in
    multiples of 16 elements; q bf16 [B, H, N_q, d].  Returns O bf16 and L fp32 as decode().
    """
    import torch
    k8, v8 = (x.view(torch.uint8) if x.dtype == torch.float8_e4m3fn else x for x in (k8, v8))
    if not (q.is_cuda and q.dtype == torch.bfloat16 and q.dim() == 4 and q.stride(-1) == 1):
        raise ValueError("q must be a bf16 CUDA tensor [B, H, N_q, d] with contiguous d")
    for t in (k8, v8):
        if not (t.dtype == torch.uint8 and t.dim() == 4 and t.stride(-1) == 1 and t.device == q.device):
            raise ValueError("k8 and v8 must be E4M3 code tensors [B, H_kv, N_k, d] on q's device, d contiguous")
    B, H, N_q, d = q.shape
    if k8.shape != v8.shape or k8.shape[0] != B or k8.shape[3] != d:
        raise ValueError("k8 and v8 must be [B, H_kv, N_k, d]")
    H_kv, N_k = int(k8.shape[1]), int(k8.shape[2])
    scale = default_scale(d) if scale is None else float(scale)
    need = decode_workspace_size(B, H, H_kv, N_q, N_k, d, causal, window)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    _check_like(out, q, "out")
    _check_lse(lse, q, B * H * N_q)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _check_workspace(workspace, q)
    ws_ptr = workspace.data_ptr() if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = None
    if not all(t.is_contiguous() for t in (q, k8, v8, out)):
        st = _lib.strides_array((q, k8, v8, out))
    _raise("fa_fwd_decode_fp8kv", _lib.fa_fwd_decode_fp8kv(
        q.data_ptr(), k8.data_ptr(), v8.data_ptr(), float(k_scale), float(v_scale), out.data_ptr(), lse.data_ptr(),
        B, H, H_kv, N_q, N_k, d, ctypes.addressof(st) if st is not None else 0, scale, int(bool(causal)),
        int(window), ws_ptr, ws_bytes, _stream_handle(q.device)))
    return out, lse


def check_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status code."""
    return _lib.fa_check_status(_stream_handle(device))

"""Exact, IO-aware attention for B200 (sm_100a).

``forward`` and ``backward`` take contiguous bf16 CUDA tensors of shape
[B, H, N, d] and run the hand-written kernels of libfa_b200.so on the current
torch stream.  torch supplies device memory and streams only.
"""

from __future__ import annotations

import math

from . import _lib
from ._lib import FAError, STATUS, STATUS_NAMES, load

__all__ = ["forward", "check_status", "FAError", "STATUS", "STATUS_NAMES", "load", "default_scale"]


def default_scale(d: int) -> float:
    """1/sqrt(d_k): the scale of the attention formula."""
    return 1.0 / math.sqrt(d)


def _stream_handle(device) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(*ts):
    import torch
    t0 = ts[0]
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError("expected contiguous bf16 CUDA tensors of shape [B, H, N, d]")
        if t.shape != t0.shape or t.device != t0.device:
            raise ValueError("shape/device mismatch")


def _raise(name, st):
    if st != _lib.FA_OK:
        raise FAError(name, st)


def forward(q, k, v, scale: float | None = None, causal: bool = False, window: int = 0,
            out=None, lse=None):
    """O, L = attention(Q, K, V); O bf16 [B,H,N,d], L fp32 [B,H,N] (natural-log logsumexp)."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = _lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     B, H, N, d, scale, int(bool(causal)), int(window), _stream_handle(q.device))
    _raise("fa_fwd", st)
    return out, lse


def check_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status code."""
    return _lib.fa_check_status(_stream_handle(device))

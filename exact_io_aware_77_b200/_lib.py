"""ctypes binding of libfa_b200.so: the C-ABI entry points under the same names.

Argument marshalling only -- every step of the attention path runs in the CUDA
kernels behind these calls.  Loading fails loudly when the library has not been
built; there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fa.h")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_NULL", 2: "FA_ERR_SHAPE", 3: "FA_ERR_HEADDIM", 4: "FA_ERR_ALIGN",
    5: "FA_ERR_MASK", 6: "FA_ERR_WORKSPACE", 7: "FA_ERR_CUDA", 8: "FA_ERR_DEVICE",
    9: "FA_ERR_TIMEOUT", 10: "FA_ERR_SCALE", 11: "FA_ERR_NOALLOC_LIMIT",
    12: "FA_ERR_INTERNAL", 13: "FA_ERR_PHASES",
}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

_c_int, _c_float, _c_void_p, _c_size_t = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_c_ull = ctypes.c_ulonglong

# name -> (restype, argtypes); mirrors include/fa.h
SIGNATURES = {
    "fa_fwd": (_c_int, [_c_void_p] * 5 + [_c_int] * 4 + [_c_float, _c_int, _c_int, _c_void_p]),
    "fa_bwd_workspace_size": (_c_size_t, [_c_int] * 4),
    "fa_bwd": (_c_int, [_c_void_p] * 9 + [_c_int] * 4 + [_c_float, _c_int, _c_int, _c_void_p, _c_size_t,
                                                         _c_void_p]),
    "fa_bwd_phases": (_c_int, [_c_void_p] * 9 + [_c_int] * 4 + [_c_float, _c_int, _c_int, _c_void_p, _c_size_t,
                                                                _c_int, _c_void_p]),
    "fa_bwd_noalloc": (_c_int, [_c_void_p] * 9 + [_c_int] * 4 + [_c_float, _c_int, _c_int, _c_void_p]),
    "fa_fwd_gqa": (_c_int, [_c_void_p] * 5 + [_c_int] * 5 + [_c_float, _c_int, _c_int, _c_void_p]),
    "fa_fwd_strided": (_c_int, [_c_void_p] * 5 + [_c_int] * 5 + [_c_void_p, _c_float, _c_int, _c_int, _c_void_p]),
    "fa_bwd_strided": (_c_int, [_c_void_p] * 9 + [_c_int] * 5 + [_c_void_p, _c_float, _c_int, _c_int, _c_void_p,
                                                                 _c_size_t, _c_int, _c_void_p]),
    "fa_bwd_gqa": (_c_int, [_c_void_p] * 9 + [_c_int] * 5 + [_c_float, _c_int, _c_int, _c_void_p, _c_size_t,
                                                             _c_int, _c_void_p]),
    "fa_decode_workspace_size": (_c_size_t, [_c_int] * 8),
    "fa_fwd_decode": (_c_int, [_c_void_p] * 5 + [_c_int] * 6 + [_c_void_p, _c_float, _c_int, _c_int, _c_void_p,
                                                                _c_size_t, _c_void_p]),
    "fa_fwd_decode_fp8kv": (_c_int, [_c_void_p] * 3 + [_c_float, _c_float] + [_c_void_p] * 2 + [_c_int] * 6 +
                            [_c_void_p, _c_float, _c_int, _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "fa_fwd_fp8": (_c_int, [_c_void_p] * 3 + [_c_float] * 3 + [_c_void_p] * 2 + [_c_int] * 5 +
                   [_c_float, _c_int, _c_int, _c_void_p]),
    "fa_status_string": (ctypes.c_char_p, [_c_int]),
    "fa_check_status": (_c_int, [_c_void_p]),
    "fa_set_wait_limit_ns": (None, [_c_ull]),
    "fa_selftest_timeout": (_c_int, [_c_ull, _c_void_p]),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


_lib = None


def load() -> ctypes.CDLL:
    """Load the built library (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m exact_io_aware_77_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def header_symbols() -> list[str]:
    """Every function include/fa.h declares (FA_EXPORT lines)."""
    text = open(HEADER).read()
    return re.findall(r"FA_EXPORT\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def _call(name, *args) -> int:
    return getattr(load(), name)(*args)


def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, window, stream) -> int:
    return _call("fa_fwd", q, k, v, o, lse, B, H, N, d, scale, causal, window, stream)


def fa_bwd_workspace_size(B, H, N, d) -> int:
    return _call("fa_bwd_workspace_size", B, H, N, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window, workspace,
           workspace_bytes, stream) -> int:
    return _call("fa_bwd", q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window,
                 workspace, workspace_bytes, stream)


def fa_bwd_phases(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window, workspace,
                  workspace_bytes, phases, stream) -> int:
    return _call("fa_bwd_phases", q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window,
                 workspace, workspace_bytes, phases, stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window, stream) -> int:
    """fa_bwd with the library's built-in 64 MiB scratch instead of a caller workspace."""
    return _call("fa_bwd_noalloc", q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, window,
                 stream)


def fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, window, stream) -> int:
    """fa_fwd with H_kv K/V heads shared by contiguous groups of the H query heads."""
    return _call("fa_fwd_gqa", q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, window, stream)


def fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, causal, window, workspace,
               workspace_bytes, phases, stream) -> int:
    """fa_bwd_phases with H_kv shared K/V heads; dk, dv are [B, H_kv, N, d]."""
    return _call("fa_bwd_gqa", q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, causal, window,
                 workspace, workspace_bytes, phases, stream)


class FaStrides(ctypes.Structure):
    """fa_strides: element strides (b, h, n) of a [B, heads, N, d] array with contiguous d."""
    _fields_ = [("b", ctypes.c_longlong), ("h", ctypes.c_longlong), ("n", ctypes.c_longlong)]


def strides_array(tensors):
    """A ctypes array of FaStrides for [B, heads, N, d] tensors (kept alive by the caller)."""
    arr = (FaStrides * len(tensors))()
    for i, t in enumerate(tensors):
        sb, sh, sn, _ = t.stride()
        arr[i] = FaStrides(sb, sh, sn)
    return arr


def fa_fwd_strided(q, k, v, o, lse, B, H, H_kv, N, d, strides, scale, causal, window, stream) -> int:
    """fa_fwd_gqa with per-array strides (``strides``: address of 4 fa_strides, or 0)."""
    return _call("fa_fwd_strided", q, k, v, o, lse, B, H, H_kv, N, d, strides, scale, causal, window, stream)


def fa_bwd_strided(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, strides, scale, causal, window, workspace,
                   workspace_bytes, phases, stream) -> int:
    """fa_bwd_gqa with per-array strides (``strides``: address of 8 fa_strides)."""
    return _call("fa_bwd_strided", q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, strides, scale, causal,
                 window, workspace, workspace_bytes, phases, stream)


def fa_decode_workspace_size(B, H, H_kv, N_q, N_k, d, causal, window) -> int:
    return _call("fa_decode_workspace_size", B, H, H_kv, N_q, N_k, d, causal, window)


def fa_fwd_decode(q, k, v, o, lse, B, H, H_kv, N_q, N_k, d, strides, scale, causal, window, workspace,
                  workspace_bytes, stream) -> int:
    """Forward of N_q new query rows (the last N_q key positions) over N_k keys."""
    return _call("fa_fwd_decode", q, k, v, o, lse, B, H, H_kv, N_q, N_k, d, strides, scale, causal, window,
                 workspace, workspace_bytes, stream)


def fa_fwd_decode_fp8kv(q, k8, v8, k_scale, v_scale, o, lse, B, H, H_kv, N_q, N_k, d, strides, scale, causal,
                        window, workspace, workspace_bytes, stream) -> int:
    """fa_fwd_decode over E4M3 K/V codes with per-tensor scales."""
    return _call("fa_fwd_decode_fp8kv", q, k8, v8, k_scale, v_scale, o, lse, B, H, H_kv, N_q, N_k, d, strides, scale,
                 causal, window, workspace, workspace_bytes, stream)


def fa_fwd_fp8(q8, k8, vt8, q_scale, k_scale, v_scale, o, lse, B, H, H_kv, N, d, scale, causal, window,
               stream) -> int:
    """The forward on E4M3 Q, K and transposed V with per-tensor scales."""
    return _call("fa_fwd_fp8", q8, k8, vt8, q_scale, k_scale, v_scale, o, lse, B, H, H_kv, N, d, scale, causal,
                 window, stream)


def fa_status_string(status: int) -> str:
    return status_string(status)


def fa_check_status(stream) -> int:
    return _call("fa_check_status", stream)


def fa_set_wait_limit_ns(limit_ns: int) -> None:
    _call("fa_set_wait_limit_ns", limit_ns)


def fa_selftest_timeout(limit_ns: int, stream) -> int:
    return _call("fa_selftest_timeout", limit_ns, stream)

"""Shared helpers of the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (fixed for this method): bf16 O max-abs <= 2e-2 and mean-abs <= 2e-3;
fp32 logsumexp max-abs <= 1e-3; gradients relative L2 <= 1e-2.  The GPU result is
widened to fp64 and compared with the unrounded fp64 oracle.
"""

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
L_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def forward_errors(o_gpu, l_gpu, o_ref, l_ref) -> dict:
    o_gpu, l_gpu = to64(o_gpu), to64(l_gpu)
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(l_gpu)), "non-finite output"
    e = np.abs(o_gpu - o_ref)
    return {"o_max": float(e.max()), "o_mean": float(e.mean()),
            "l_max": float(np.abs(l_gpu - l_ref).max())}


def assert_forward_close(o_gpu, l_gpu, o_ref, l_ref, what=""):
    err = forward_errors(o_gpu, l_gpu, o_ref, l_ref)
    assert err["o_max"] <= O_MAX_ABS, (what, err)
    assert err["o_mean"] <= O_MEAN_ABS, (what, err)
    assert err["l_max"] <= L_MAX_ABS, (what, err)
    return err


GRAD_RMS_FLOOR = 1e-3


def rel_l2(a, ref) -> float:
    """||a - ref|| / max(||ref||, 1e-3 * sqrt(n)).

    The floor matters only for gradients that are zero by the mathematics (a window of 1
    makes dS, hence dQ and dK, exactly 0); there the relative error has no meaning and the
    check becomes an absolute RMS error of at most 1e-5 per element.
    """
    a = to64(a) if isinstance(a, torch.Tensor) else a
    floor = GRAD_RMS_FLOOR * np.sqrt(ref.size)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), floor))


def assert_grads_close(grads_gpu, grads_ref, what=""):
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), grads_gpu, grads_ref):
        gg = to64(g)
        assert np.all(np.isfinite(gg)), (what, name, "non-finite")
        errs[name] = rel_l2(gg, r)
        assert errs[name] <= GRAD_REL_L2, (what, errs)
    return errs


def fp8_o_bound(q, k, v, scale, causal, window, o_ref):
    """Per-element bound on |O - O_ref| for the FP8 forward, derived from its arithmetic: P is
    rounded to E4M3 before P V (relative error <= 2^-4 for normal values, absolute <= 2^-10 below
    E4M3's normal range) while l sums the exact P, so with w_j = exp(s_j - max s) over the allowed
    keys, |dO_c| <= sum_j max(2^-4 w_j, 2^-10) |V_jc| / sum_j w_j; plus the bf16 rounding of O
    (2^-8 |O|) and 1e-3 for the fp32 exponentials and sums.  q [B, H, N, d], k and v [B, H_kv, N, d]
    (dequantised, fp64)."""
    from oracle import attention as orc
    B, H, N, _ = q.shape
    g = H // k.shape[1]
    ok = orc.allowed_mask(N, N, causal, window)
    bound = np.empty_like(o_ref)
    for b in range(B):
        for h in range(H):
            sc = np.where(ok, scale * (q[b, h] @ k[b, h // g].T), -np.inf)
            w = np.exp(sc - sc.max(axis=1, keepdims=True))
            per = np.where(ok, np.maximum(2.0 ** -4 * w, 2.0 ** -10), 0.0)
            bound[b, h] = (per @ np.abs(v[b, h // g])) / w.sum(axis=1, keepdims=True)
    return bound + 2.0 ** -8 * np.abs(o_ref) + 1e-3

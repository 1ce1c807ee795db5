"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

If a mutant survived every pin, the pins would not be tying the oracle to the
definition of attention tightly enough; this file is the evidence that they do.
"""

import numpy as np
import pytest

from oracle import attention as orc
from tests.oracle_pins import PINS


def _scores_transposed(q, k, scale, ok):
    return np.where(ok, scale * (k @ q.T), -np.inf)


def _scores_no_scale(q, k, scale, ok):
    return np.where(ok, q @ k.T, -np.inf)


def _rows_mask_causal_strict(r, n_k, causal, window):
    i = r[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((r.size, n_k), dtype=bool)
    if causal:
        ok &= j < i
    if window > 0:
        ok &= j >= i - window + 1
    return ok


def _rows_mask_window_wide(r, n_k, causal, window):
    i = r[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((r.size, n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window
    return ok


def _rows_mask_two_sided_wide(r, n_k, causal, window):
    i = r[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((r.size, n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window + 1
        if not causal:
            ok &= j <= i + window
    return ok


def _rows_mask_one_sided_only(r, n_k, causal, window):
    i = r[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((r.size, n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window + 1
    return ok


def _softmax_no_shift(s):
    e = np.exp(s)
    denom = np.sum(e, axis=1, keepdims=True)
    return e / denom, np.log(denom)[:, 0]


def _softmax_log2(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    denom = np.sum(e, axis=1, keepdims=True)
    return e / denom, (m + np.log2(denom))[:, 0]


def _softmax_lse_no_max(s):
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    denom = np.sum(e, axis=1, keepdims=True)
    return e / denom, np.log(denom)[:, 0]


def _make_bwd(variant):
    def bwd(q, k, v, do, scale, causal, window):
        o, lse, p = orc._head_forward(q, k, v, scale, causal, window)
        dv = p.T @ do
        dp = do @ v.T
        d_row = np.sum(p * dp, axis=1, keepdims=True)
        if variant == "dv_untransposed":
            dv = p @ do
        if variant == "dp_swapped":
            dp = (v @ do.T).T if dp.shape[0] == dp.shape[1] else do @ v.T * 1.01
        if variant == "delta_wrong_axis":
            d_row = np.sum(p * dp, axis=0, keepdims=True)
        if variant == "delta_missing":
            d_row = 0.0
        ds = p * (dp - d_row)
        dq = scale * (ds @ k)
        dk = scale * (ds.T @ q)
        if variant == "dq_no_scale":
            dq = ds @ k
        if variant == "dk_untransposed":
            dk = scale * (ds @ q)
        return dq, dk, dv
    return bwd


def _head_forward_pv_transposed(q, k, v, scale, causal, window, row_start=0):
    ok = orc.allowed_mask(q.shape[0], k.shape[0], causal, window, row_start)
    p, lse = orc._softmax_rows(orc._scores(q, k, scale, ok))
    return p.T @ v, lse, p


def _kv_head_interleaved(n_heads, n_kv_heads):
    return np.arange(n_heads) % n_kv_heads


def _backward_shared_kv_first_only(q, k, v, do, scale, causal=False, window=0):
    q, k, v, do = orc._as64(q), orc._as64(k), orc._as64(v), orc._as64(do)
    idx = orc.kv_head_of(q.shape[-3], k.shape[-3])
    dq, dk, dv = orc.attention_backward(q, k[..., idx, :, :], v[..., idx, :, :], do, scale, causal, window)
    g = q.shape[-3] // k.shape[-3]
    return dq, dk[..., ::g, :, :], dv[..., ::g, :, :]


def _e4m3_bias_8(codes):
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return sign * np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)


def _e4m3_no_subnormals(codes):
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    return sign * np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)


def _fp8kv_v_scale_dropped(q, k8, v8, k_scale, v_scale, scale, causal=False, window=0):
    return orc.attention_forward_decode(q, k_scale * orc.e4m3_to_float(k8), orc.e4m3_to_float(v8), scale, causal,
                                        window)


def _fp8_v_not_transposed(q8, k8, vt8, q_scale, k_scale, v_scale, scale, causal=False, window=0):
    q = q_scale * orc.e4m3_to_float(q8)
    k = k_scale * orc.e4m3_to_float(k8)
    v = v_scale * orc.e4m3_to_float(vt8).reshape(k.shape)   # the codes read as [N, d], not transposed
    return orc.attention_forward_shared_kv(q, k, v, scale, causal, window)


MUTANTS = {
    "fp8_v_not_transposed": ("attention_forward_fp8", _fp8_v_not_transposed),
    "e4m3_bias_8": ("e4m3_to_float", _e4m3_bias_8),
    "e4m3_no_subnormals": ("e4m3_to_float", _e4m3_no_subnormals),
    "fp8kv_v_scale_dropped": ("attention_forward_decode_fp8kv", _fp8kv_v_scale_dropped),
    "decode_rows_first": ("_decode_row_start", lambda n_q, n_k: 0),
    "decode_rows_one_early": ("_decode_row_start", lambda n_q, n_k: max(0, n_k - n_q - 1)),
    "scores_transposed": ("_scores", _scores_transposed),
    "scale_dropped": ("_scores", _scores_no_scale),
    "causal_excludes_diagonal": ("_rows_mask", _rows_mask_causal_strict),
    "window_one_too_wide": ("_rows_mask", _rows_mask_window_wide),
    "negative_window_accepted": ("_check_mask_args", lambda causal, window: None),
    "two_sided_window_one_too_wide": ("_rows_mask", _rows_mask_two_sided_wide),
    "two_sided_window_upper_edge_missing": ("_rows_mask", _rows_mask_one_sided_only),
    "no_max_shift": ("_softmax_rows", _softmax_no_shift),
    "lse_in_log2": ("_softmax_rows", _softmax_log2),
    "lse_missing_max": ("_softmax_rows", _softmax_lse_no_max),
    "probabilities_transposed": ("_head_forward", _head_forward_pv_transposed),
    "dv_untransposed": ("_head_backward", _make_bwd("dv_untransposed")),
    "delta_wrong_axis": ("_head_backward", _make_bwd("delta_wrong_axis")),
    "delta_missing": ("_head_backward", _make_bwd("delta_missing")),
    "dq_no_scale": ("_head_backward", _make_bwd("dq_no_scale")),
    "dk_untransposed": ("_head_backward", _make_bwd("dk_untransposed")),
    "kv_heads_interleaved": ("kv_head_of", _kv_head_interleaved),
    "shared_kv_grad_not_summed": ("attention_backward_shared_kv", _backward_shared_kv_first_only),
}


def _first_failing_pin():
    import warnings
    for name in sorted(PINS):
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                PINS[name](orc)
        except Exception:  # an assertion, or a shape/overflow error the slip causes
            return name
    return None


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(orc, attr, fn)
    caught_by = _first_failing_pin()
    assert caught_by is not None, f"mutant {mutant} survived every pin"

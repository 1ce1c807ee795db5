"""Checks that pin the fp64 oracle to facts other than itself.

Each check takes the oracle module and raises AssertionError when the oracle
disagrees with a closed form, an invariant of exact attention, a hand-derived
example (tests/golden/), central finite differences, or an independent library
routine (torch's scaled_dot_product_attention and autograd, in float64).  The
checks are written so that a plausible slip anywhere in the oracle (a dropped
scale, a swapped operand, an off-by-one mask edge, a missing max shift, a
transposed gradient) fails at least one of them; tests/test_oracle_mutants.py
plants such slips and confirms it.
"""

from __future__ import annotations

import json
import math
import pathlib

import numpy as np

GOLDEN = pathlib.Path(__file__).parent / "golden"
MASKS = [(False, 0), (True, 0), (True, 1), (True, 3), (True, 7), (False, 1), (False, 3), (False, 7)]


def _rng(seed):
    return np.random.default_rng(seed)


def _qkv(seed, n=13, d=5, lead=(2,), std=1.0):
    r = _rng(seed)
    return [std * r.standard_normal(lead + (n, d)) for _ in range(3)]


def _band(i, n, causal, window):
    """[lo, hi] of the keys row i may attend (closed interval), written from the mask readings."""
    lo = max(0, i - window + 1) if window > 0 else 0
    if causal:
        hi = i
    elif window > 0:
        hi = min(n - 1, i + window - 1)
    else:
        hi = n - 1
    return lo, hi


def _n_allowed(i, n, causal, window):
    lo, hi = _band(i, n, causal, window)
    return hi - lo + 1


# --- forward pins -------------------------------------------------------------------------

def rows_sum_to_one(orc):
    """Every softmax row is a probability vector over the allowed keys only."""
    q, k, _ = _qkv(1)
    for causal, window in MASKS:
        p = orc.attention_probabilities(q, k, 0.7, causal, window)
        assert np.all(p >= 0)
        assert np.max(np.abs(p.sum(-1) - 1.0)) < 1e-12
        n = q.shape[-2]
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        masked = np.zeros((n, n), bool)
        if causal:
            masked |= j > i
        if window:
            masked |= j < i - window + 1
            if not causal:
                masked |= j > i + window - 1
        assert np.all(p[..., masked] == 0.0)
        assert np.all(p[..., ~masked] > 0.0)


def constant_v(orc):
    """V with every row equal to c gives O rows equal to c for every mask."""
    q, k, _ = _qkv(2)
    c = np.array([0.5, -2.0, 3.25, 0.0, 1.0])
    v = np.broadcast_to(c, q.shape).copy()
    for causal, window in MASKS:
        o, _ = orc.attention_forward(q, k, v, 0.9, causal, window)
        assert np.max(np.abs(o - c)) < 1e-12


def causal_row0(orc):
    """Causal row 0 sees only key 0: O_0 = v_0 and L_0 = scale q_0 . k_0."""
    q, k, v = _qkv(3)
    o, lse = orc.attention_forward(q, k, v, 0.37, True, 0)
    assert np.max(np.abs(o[..., 0, :] - v[..., 0, :])) < 1e-12
    l0 = 0.37 * np.sum(q[..., 0, :] * k[..., 0, :], -1)
    assert np.max(np.abs(lse[..., 0] - l0)) < 1e-12


def causal_future_independence(orc):
    """Changing keys/values after row i leaves causal rows <= i unchanged, and changes row i+1."""
    q, k, v = _qkv(4)
    o, lse = orc.attention_forward(q, k, v, 0.5, True, 0)
    i = 6
    k2, v2 = k.copy(), v.copy()
    k2[..., i + 1:, :] += 3.0
    v2[..., i + 1:, :] -= 5.0
    o2, l2 = orc.attention_forward(q, k2, v2, 0.5, True, 0)
    assert np.max(np.abs(o2[..., :i + 1, :] - o[..., :i + 1, :])) < 1e-12
    assert np.max(np.abs(l2[..., :i + 1] - lse[..., :i + 1])) < 1e-12
    assert np.max(np.abs(o2[..., i + 1, :] - o[..., i + 1, :])) > 1e-3


def window_one(orc):
    """A window of 1 keeps only the diagonal: O_i = v_i, L_i = scale q_i . k_i."""
    q, k, v = _qkv(5)
    o, lse = orc.attention_forward(q, k, v, 0.8, True, 1)
    assert np.max(np.abs(o - v)) < 1e-12
    assert np.max(np.abs(lse - 0.8 * np.sum(q * k, -1))) < 1e-12


def window_covering_is_causal(orc):
    """A window of N or more equals plain causal attention."""
    q, k, v = _qkv(6)
    n = q.shape[-2]
    o, lse = orc.attention_forward(q, k, v, 0.6, True, 0)
    for w in (n, n + 5):
        o2, l2 = orc.attention_forward(q, k, v, 0.6, True, w)
        assert np.max(np.abs(o2 - o)) < 1e-12 and np.max(np.abs(l2 - lse)) < 1e-12


def window_edge(orc):
    """Row i with window W ignores key i-W and depends on key i-W+1."""
    q, k, v = _qkv(7)
    w, i = 4, 9
    o, _ = orc.attention_forward(q, k, v, 0.6, True, w)
    for j, should_change in ((i - w, False), (i - w + 1, True)):
        k2, v2 = k.copy(), v.copy()
        k2[..., j, :] += 2.0
        v2[..., j, :] += 7.0
        o2, _ = orc.attention_forward(q, k2, v2, 0.6, True, w)
        diff = np.max(np.abs(o2[..., i, :] - o[..., i, :]))
        assert (diff > 1e-3) if should_change else (diff < 1e-12)


def scale_zero(orc):
    """scale = 0 gives uniform weights: L_i = ln(#allowed keys), O_i = mean of the allowed v_j."""
    q, k, v = _qkv(8)
    n = q.shape[-2]
    for causal, window in MASKS:
        o, lse = orc.attention_forward(q, k, v, 0.0, causal, window)
        for i in range(n):
            cnt = _n_allowed(i, n, causal, window)
            lo, hi = _band(i, n, causal, window)
            assert abs(lse[..., i] - math.log(cnt)).max() < 1e-12
            assert np.max(np.abs(o[..., i, :] - v[..., lo:hi + 1, :].mean(-2))) < 1e-12


def key_shift(orc):
    """K_j <- K_j + c for every j leaves O unchanged and shifts L_i by scale q_i . c."""
    q, k, v = _qkv(9)
    c = np.array([0.3, -1.1, 0.7, 2.0, -0.4])
    for causal, window in MASKS:
        o, lse = orc.attention_forward(q, k, v, 0.45, causal, window)
        o2, l2 = orc.attention_forward(q, k + c, v, 0.45, causal, window)
        assert np.max(np.abs(o2 - o)) < 1e-11
        assert np.max(np.abs(l2 - lse - 0.45 * (q @ c))) < 1e-11


def key_permutation(orc):
    """Without a mask, permuting keys and values together leaves O and L unchanged."""
    q, k, v = _qkv(10)
    perm = _rng(10).permutation(q.shape[-2])
    o, lse = orc.attention_forward(q, k, v, 0.5, False, 0)
    o2, l2 = orc.attention_forward(q, k[..., perm, :], v[..., perm, :], 0.5, False, 0)
    assert np.max(np.abs(o2 - o)) < 1e-12 and np.max(np.abs(l2 - lse)) < 1e-12


def large_scores(orc):
    """Scores of 1e3 (exp overflows fp64) must still give the exact softmax: the top key,
    ahead of the runner-up by 200, takes all the weight."""
    n, d = 6, 3
    q = np.zeros((n, d))
    q[:, 0] = 200.0
    k = np.zeros((n, d))
    k[:, 0] = np.arange(n, dtype=float)        # scores 200 * j, up to 1000
    v = _rng(11).standard_normal((n, d))
    o, lse = orc.attention_forward(q, k, v, 1.0, False, 0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(o - v[n - 1])) < 1e-12          # e^-200 relative weight of the runner-up
    assert np.max(np.abs(lse - 200.0 * (n - 1))) < 1e-12


def golden_examples(orc):
    """Hand-derived examples (tests/golden/*.json) reproduce to 1e-12."""
    for path in sorted(GOLDEN.glob("*.json")):
        g = json.loads(path.read_text())
        q, k, v = (np.array(g[x]) for x in ("q", "k", "v"))
        for case in g["cases"]:
            o, lse = orc.attention_forward(q, k, v, g["scale"], case["causal"], case["window"])
            assert np.max(np.abs(o - np.array(case["O"]))) < 1e-12, path.name
            assert np.max(np.abs(lse - np.array(case["L"]))) < 1e-12, path.name
        if "backward_single_row" in g:
            b = g["backward_single_row"]
            dq, dk, dv = orc.attention_backward(np.array(b["q"]), k, v, np.array(b["dO"]), g["scale"])
            assert np.max(np.abs(dq - np.array(b["dQ"]))) < 1e-12
            assert np.max(np.abs(dk - np.array(b["dK"]))) < 1e-12
            assert np.max(np.abs(dv - np.array(b["dV"]))) < 1e-12


def golden_decode_examples(orc):
    """Hand-derived decode examples (tests/golden/decode/*.json): new rows at the last key
    positions, every mask kind, reproduce to 1e-12."""
    for path in sorted((GOLDEN / "decode").glob("*.json")):
        g = json.loads(path.read_text())
        k, v = np.array(g["k"])[None, None], np.array(g["v"])[None, None]
        for case in g["cases"]:
            q = np.ones((1, 1, case["n_q"], 1))
            o, lse = orc.attention_forward_decode(q, k, v, g["scale"], case["causal"], case["window"])
            assert np.max(np.abs(o[0, 0] - np.array(case["O"]))) < 1e-12, (path.name, case)
            assert np.max(np.abs(lse[0, 0] - np.array(case["L"]))) < 1e-12, (path.name, case)


def _torch_reference(q, k, v, scale, causal, window):
    import torch
    import torch.nn.functional as F
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    n = q.shape[-2]
    i = torch.arange(n)[:, None]
    j = torch.arange(n)[None, :]
    ok = torch.ones(n, n, dtype=torch.bool)
    if causal:
        ok &= j <= i
    if window:
        ok &= (j - i).abs() <= window - 1 if not causal else j >= i - window + 1
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=ok, scale=scale)
    return (tq, tk, tv), o


def library_forward(orc):
    """torch scaled_dot_product_attention (float64, boolean mask, explicit scale) agrees to 1e-12."""
    q, k, v = _qkv(12, n=37, d=16, lead=(2, 3))
    for causal, window in MASKS:
        _, o_ref = _torch_reference(q, k, v, 0.25, causal, window)
        o, _ = orc.attention_forward(q, k, v, 0.25, causal, window)
        assert np.max(np.abs(o - o_ref.detach().numpy())) < 1e-12


def library_backward(orc):
    """torch autograd of sum(O o dO) through scaled_dot_product_attention agrees to 1e-11."""
    import torch
    q, k, v = _qkv(13, n=23, d=8, lead=(2,))
    do = _rng(14).standard_normal(q.shape)
    for causal, window in MASKS:
        (tq, tk, tv), o_ref = _torch_reference(q, k, v, 0.4, causal, window)
        (o_ref * torch.tensor(do)).sum().backward()
        dq, dk, dv = orc.attention_backward(q, k, v, do, 0.4, causal, window)
        for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.max(np.abs(mine - ref.numpy())) < 1e-11


def finite_differences(orc):
    """Central differences (h = 1e-6) of sum(O o dO) match dQ, dK, dV on tiny inputs."""
    n, d, h, scale = 7, 3, 1e-6, 0.6
    q, k, v = _qkv(15, n=n, d=d, lead=())
    do = _rng(16).standard_normal((n, d))
    for causal, window in MASKS:
        grads = orc.attention_backward(q, k, v, do, scale, causal, window)

        def f(qq, kk, vv):
            return float(np.sum(orc.attention_forward(qq, kk, vv, scale, causal, window)[0] * do))

        for which, g in enumerate(grads):
            fd = np.zeros((n, d))
            for a in range(n):
                for b in range(d):
                    args_p = [q.copy(), k.copy(), v.copy()]
                    args_m = [q.copy(), k.copy(), v.copy()]
                    args_p[which][a, b] += h
                    args_m[which][a, b] -= h
                    fd[a, b] = (f(*args_p) - f(*args_m)) / (2 * h)
            err = np.linalg.norm(fd - g) / max(np.linalg.norm(fd), 1e-30)
            assert err < 1e-6, (which, causal, window, err)


def delta_identity(orc):
    """sum_j P_ij dP_ij equals rowsum(dO o O): the D term a fused backward uses."""
    q, k, v = _qkv(17, n=19, d=6, lead=())
    do = _rng(18).standard_normal(q.shape)
    for causal, window in MASKS:
        p = orc.attention_probabilities(q, k, 0.5, causal, window)
        o, _ = orc.attention_forward(q, k, v, 0.5, causal, window)
        lhs = np.sum(p * (do @ v.T), -1)
        rhs = np.sum(do * o, -1)
        assert np.max(np.abs(lhs - rhs)) < 1e-12


def row_blocks_match(orc):
    """The row-block forward/backward equal the full-matrix ones (blocks smaller than N)."""
    q, k, v = _qkv(19, n=41, d=8, lead=())
    do = _rng(20).standard_normal(q.shape)
    rows = np.array([0, 3, 17, 40])
    for causal, window in MASKS:
        o, lse = orc.attention_forward(q, k, v, 0.3, causal, window)
        o_r, l_r = orc.attention_forward_rows(q, k, v, 0.3, causal, window, rows=rows, block=3)
        assert np.max(np.abs(o_r - o[rows])) < 1e-12 and np.max(np.abs(l_r - lse[rows])) < 1e-12
        dq, dk, dv = orc.attention_backward(q, k, v, do, 0.3, causal, window)
        dq_r, dk_r, dv_r = orc.attention_backward_rows(q, k, v, do, 0.3, causal, window,
                                                       key_rows=rows, block=5)
        assert np.max(np.abs(dq_r - dq)) < 1e-12
        assert np.max(np.abs(dk_r - dk[rows])) < 1e-12 and np.max(np.abs(dv_r - dv[rows])) < 1e-12
        # disjoint query-row subsets: their dQ rows, and dK/dV contributions summing to the whole
        parts = [np.arange(0, 20), np.arange(20, 41)]
        acc_k, acc_v = 0.0, 0.0
        for qr in parts:
            dq_p, dk_p, dv_p = orc.attention_backward_rows(q, k, v, do, 0.3, causal, window,
                                                           block=7, query_rows=qr)
            assert np.max(np.abs(dq_p - dq[qr])) < 1e-12
            acc_k, acc_v = acc_k + dk_p, acc_v + dv_p
        assert np.max(np.abs(acc_k - dk)) < 1e-12 and np.max(np.abs(acc_v - dv)) < 1e-12


def pair_count(orc):
    """allowed_pairs matches the closed forms N^2, N(N+1)/2 and the banded counts: one-sided
    W(W+1)/2 + (N-W)W, two-sided N(2W-1) - W(W-1) (each edge loses 1 + 2 + ... + (W-1))."""
    for n in (1, 5, 16, 33):
        assert orc.allowed_pairs(n, False, 0) == n * n
        assert orc.allowed_pairs(n, True, 0) == n * (n + 1) // 2
        for w in (1, 4, 40):
            ww = min(w, n)
            assert orc.allowed_pairs(n, True, w) == ww * (ww + 1) // 2 + (n - ww) * ww
            two = n * n if w >= n else n * (2 * w - 1) - w * (w - 1)
            assert orc.allowed_pairs(n, False, w) == two


def two_sided_window(orc):
    """Without causal, a window W keeps |i - j| <= W - 1: W = 1 gives O_i = v_i and
    L_i = scale q_i . k_i; W >= N equals unmasked attention; row i ignores keys i - W and
    i + W and depends on keys i - W + 1 and i + W - 1."""
    q, k, v = _qkv(22)
    n = q.shape[-2]
    o, lse = orc.attention_forward(q, k, v, 0.8, False, 1)
    assert np.max(np.abs(o - v)) < 1e-12
    assert np.max(np.abs(lse - 0.8 * np.sum(q * k, -1))) < 1e-12
    o, lse = orc.attention_forward(q, k, v, 0.6, False, 0)
    for w in (n, n + 3):
        o2, l2 = orc.attention_forward(q, k, v, 0.6, False, w)
        assert np.max(np.abs(o2 - o)) < 1e-12 and np.max(np.abs(l2 - lse)) < 1e-12
    w, i = 4, 6
    o, _ = orc.attention_forward(q, k, v, 0.6, False, w)
    for j, should_change in ((i - w, False), (i + w, False), (i - w + 1, True), (i + w - 1, True)):
        k2, v2 = k.copy(), v.copy()
        k2[..., j, :] += 2.0
        v2[..., j, :] += 7.0
        o2, _ = orc.attention_forward(q, k2, v2, 0.6, False, w)
        diff = np.max(np.abs(o2[..., i, :] - o[..., i, :]))
        assert (diff > 1e-3) if should_change else (diff < 1e-12), (j, diff)


def shared_kv_library(orc):
    """Shared K/V heads (MQA: 1 K/V head; GQA: 2 for 4 query heads) agree with torch
    scaled_dot_product_attention(enable_gqa=True) and its autograd in float64, for every mask."""
    import torch
    import torch.nn.functional as F
    r = _rng(23)
    for h_kv in (1, 2, 4):
        q = r.standard_normal((2, 4, 11, 5))
        k, v = (r.standard_normal((2, h_kv, 11, 5)) for _ in range(2))
        do = r.standard_normal(q.shape)
        n = q.shape[-2]
        i = torch.arange(n)[:, None]
        j = torch.arange(n)[None, :]
        for causal, window in MASKS:
            ok = torch.ones(n, n, dtype=torch.bool)
            if causal:
                ok &= j <= i
            if window:
                ok &= (j - i).abs() <= window - 1 if not causal else j >= i - window + 1
            tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
            o_ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=ok, scale=0.35, enable_gqa=True)
            (o_ref * torch.tensor(do)).sum().backward()
            o, _ = orc.attention_forward_shared_kv(q, k, v, 0.35, causal, window)
            assert np.max(np.abs(o - o_ref.detach().numpy())) < 1e-12, (h_kv, causal, window)
            grads = orc.attention_backward_shared_kv(q, k, v, do, 0.35, causal, window)
            for mine, ref in zip(grads, (tq.grad, tk.grad, tv.grad)):
                assert mine.shape == ref.shape
                assert np.max(np.abs(mine - ref.numpy())) < 1e-11, (h_kv, causal, window)


def shared_kv_finite_differences(orc):
    """Central differences of sum(O o dO) with respect to a shared K/V head match dK and dV."""
    r = _rng(24)
    q = r.standard_normal((3, 6, 3))
    k, v = (r.standard_normal((1, 6, 3)) for _ in range(2))
    do = r.standard_normal(q.shape)
    h = 1e-6
    for causal, window in ((True, 0), (False, 2)):
        _, dk, dv = orc.attention_backward_shared_kv(q, k, v, do, 0.7, causal, window)

        def f(kk, vv):
            return float(np.sum(orc.attention_forward_shared_kv(q, kk, vv, 0.7, causal, window)[0] * do))

        for which, g in ((0, dk), (1, dv)):
            fd = np.zeros_like(g)
            for idx in np.ndindex(g.shape):
                plus, minus = [k.copy(), v.copy()], [k.copy(), v.copy()]
                plus[which][idx] += h
                minus[which][idx] -= h
                fd[idx] = (f(*plus) - f(*minus)) / (2 * h)
            assert np.linalg.norm(fd - g) / np.linalg.norm(fd) < 1e-6, (which, causal, window)


def _decode_torch_mask(n_q, n_k, causal, window):
    """Boolean [n_q, n_k] mask of the generation-step reading: row i sits at key position
    n_k - n_q + i (written here with torch ops, apart from the oracle's mask code)."""
    import torch
    pos = torch.arange(n_k - n_q, n_k)[:, None]
    j = torch.arange(n_k)[None, :]
    ok = torch.ones(n_q, n_k, dtype=torch.bool)
    if causal:
        ok &= j <= pos
    if window:
        ok &= (j - pos).abs() <= window - 1 if not causal else j >= pos - window + 1
    return ok


def decode_library(orc):
    """Few new rows over more keys: O agrees with torch scaled_dot_product_attention
    (float64, enable_gqa, boolean mask) and L with torch.logsumexp of the masked scores, to
    1e-12, for every mask, with 1, 2 or 4 K/V heads for 4 query heads."""
    import torch
    import torch.nn.functional as F
    r = _rng(31)
    for n_q, n_k in ((1, 9), (3, 9), (7, 12), (12, 12)):
        for h_kv in (1, 2, 4):
            q = r.standard_normal((2, 4, n_q, 6))
            k, v = (r.standard_normal((2, h_kv, n_k, 6)) for _ in range(2))
            for causal, window in MASKS:
                ok = _decode_torch_mask(n_q, n_k, causal, window)
                tq, tk, tv = (torch.tensor(x, dtype=torch.float64) for x in (q, k, v))
                o_ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=ok, scale=0.45, enable_gqa=True)
                rep = tk.repeat_interleave(4 // h_kv, dim=1)
                s = torch.where(ok, 0.45 * tq @ rep.transpose(-1, -2), torch.tensor(-math.inf, dtype=torch.float64))
                l_ref = torch.logsumexp(s, dim=-1)
                o, lse = orc.attention_forward_decode(q, k, v, 0.45, causal, window)
                assert o.shape == q.shape and lse.shape == q.shape[:-1]
                assert np.max(np.abs(o - o_ref.numpy())) < 1e-12, (n_q, n_k, h_kv, causal, window)
                assert np.max(np.abs(lse - l_ref.numpy())) < 1e-12, (n_q, n_k, h_kv, causal, window)


def decode_scale_zero(orc):
    """scale = 0 over N_k keys: L_i = ln(#keys allowed at position N_k - N_q + i) and O_i the
    mean of those v_j, for every mask."""
    r = _rng(32)
    n_q, n_k = 4, 11
    q = r.standard_normal((1, n_q, 3))
    k, v = (r.standard_normal((1, n_k, 3)) for _ in range(2))
    for causal, window in MASKS:
        o, lse = orc.attention_forward_decode(q, k, v, 0.0, causal, window)
        for i in range(n_q):
            lo, hi = _band(n_k - n_q + i, n_k, causal, window)
            assert abs(lse[0, i] - math.log(hi - lo + 1)) < 1e-12, (causal, window, i)
            assert np.max(np.abs(o[0, i] - v[0, lo:hi + 1].mean(axis=0))) < 1e-12


def decode_last_rows_of_self_attention(orc):
    """The N_q new rows equal the last N_q rows of the self-attention over all N_k positions."""
    r = _rng(33)
    q_full, k, v = (r.standard_normal((2, 10, 4)) for _ in range(3))
    for n_q in (1, 4, 10):
        for causal, window in MASKS:
            o_full, l_full = orc.attention_forward(q_full, k, v, 0.6, causal, window)
            o, lse = orc.attention_forward_decode(q_full[:, None, -n_q:], k[:, None], v[:, None], 0.6, causal, window)
            assert np.max(np.abs(o[:, 0] - o_full[:, -n_q:])) < 1e-12
            assert np.max(np.abs(lse[:, 0] - l_full[:, -n_q:])) < 1e-12


def e4m3_decoding(orc):
    """Every one of the 256 E4M3 codes decodes as torch's float8_e4m3fn does, and hand-worked
    codes give their values: 0x38 = 1, 0x3C = 1.5, 0xB8 = -1, 0x7E = 448 (largest), 0x08 = 2^-6
    (smallest normal), 0x07 = 7 * 2^-9, 0x01 = 2^-9 (smallest subnormal), 0x80 = -0, 0x7F NaN."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    worked = {0x38: 1.0, 0x3C: 1.5, 0xB8: -1.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x07: 7 * 2.0 ** -9,
              0x01: 2.0 ** -9, 0x00: 0.0}
    for code, val in worked.items():
        assert orc.e4m3_to_float(np.array([code], dtype=np.uint8))[0] == val, hex(code)
    neg0 = orc.e4m3_to_float(np.array([0x80], dtype=np.uint8))[0]
    assert neg0 == 0.0 and math.copysign(1.0, neg0) < 0
    assert np.isnan(orc.e4m3_to_float(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def fp8kv_decode(orc):
    """The FP8 K/V forward equals the plain decode forward on K and V dequantised by torch
    (float8_e4m3fn times the scale); doubling s_k while halving the softmax scale changes
    nothing; O is linear in s_v and L does not depend on it."""
    import torch
    r = _rng(34)
    q = r.standard_normal((2, 4, 3, 8))
    k8, v8 = (r.integers(0, 256, size=(2, 2, 20, 8)).astype(np.uint8) for _ in range(2))
    for a in (k8, v8):   # no NaN codes in the cache
        a[(a & 0x7F) == 0x7F] = 0x38
    dq = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for causal, window in MASKS:
        o, lse = orc.attention_forward_decode_fp8kv(q, k8, v8, 0.05, 0.7, 0.3, causal, window)
        o_ref, l_ref = orc.attention_forward_decode(q, 0.05 * dq(k8), 0.7 * dq(v8), 0.3, causal, window)
        assert np.max(np.abs(o - o_ref)) < 1e-12 and np.max(np.abs(lse - l_ref)) < 1e-12
        o2, l2 = orc.attention_forward_decode_fp8kv(q, k8, v8, 0.1, 0.7, 0.15, causal, window)
        assert np.max(np.abs(o2 - o)) < 1e-12 and np.max(np.abs(l2 - lse)) < 1e-12
        o3, l3 = orc.attention_forward_decode_fp8kv(q, k8, v8, 0.05, 1.4, 0.3, causal, window)
        assert np.max(np.abs(o3 - 2 * o)) < 1e-12 and np.max(np.abs(l3 - lse)) < 1e-12


def fp8_forward(orc):
    """The FP8 forward (V given transposed) equals the plain forward on torch-dequantised Q, K and
    V^T transposed back; doubling s_q while halving s_k changes nothing; O is linear in s_v."""
    import torch
    r = _rng(35)
    dq = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    q8 = r.integers(0, 256, size=(1, 4, 9, 6)).astype(np.uint8)
    k8 = r.integers(0, 256, size=(1, 2, 9, 6)).astype(np.uint8)
    vt8 = r.integers(0, 256, size=(1, 2, 6, 9)).astype(np.uint8)
    for a in (q8, k8, vt8):
        a[(a & 0x7F) == 0x7F] = 0x38
    for causal, window in MASKS:
        o, lse = orc.attention_forward_fp8(q8, k8, vt8, 0.02, 0.05, 0.7, 0.3, causal, window)
        ref = orc.attention_forward_shared_kv(0.02 * dq(q8), 0.05 * dq(k8), 0.7 * np.swapaxes(dq(vt8), -1, -2), 0.3,
                                              causal, window)
        assert o.shape == q8.shape
        assert np.max(np.abs(o - ref[0])) < 1e-12 and np.max(np.abs(lse - ref[1])) < 1e-12
        o2, l2 = orc.attention_forward_fp8(q8, k8, vt8, 0.04, 0.025, 0.7, 0.3, causal, window)
        assert np.max(np.abs(o2 - o)) < 1e-12 and np.max(np.abs(l2 - lse)) < 1e-12
        o3, l3 = orc.attention_forward_fp8(q8, k8, vt8, 0.02, 0.05, 1.4, 0.3, causal, window)
        assert np.max(np.abs(o3 - 2 * o)) < 1e-12 and np.max(np.abs(l3 - lse)) < 1e-12


def rejects_bad_masks(orc):
    """A negative window is rejected, with or without causal."""
    q, k, v = _qkv(21, n=4, d=2, lead=())
    for causal, window in ((True, -1), (False, -1)):
        try:
            orc.attention_forward(q, k, v, 1.0, causal, window)
        except ValueError:
            continue
        raise AssertionError("bad mask accepted")


PINS = {f.__name__: f for f in (
    rows_sum_to_one, constant_v, causal_row0, causal_future_independence, window_one,
    window_covering_is_causal, window_edge, scale_zero, key_shift, key_permutation,
    large_scores, golden_examples, library_forward, library_backward, finite_differences,
    delta_identity, row_blocks_match, pair_count, two_sided_window, shared_kv_library,
    shared_kv_finite_differences, decode_library, decode_scale_zero, decode_last_rows_of_self_attention,
    e4m3_decoding, fp8kv_decode, fp8_forward, golden_decode_examples, rejects_bad_masks,
)}

"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path (``exact_io_aware_77_b200``) and imports nothing from it.

What it computes, and where that is defined:

* Forward.  ``Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V`` is the one
  formula the pages print (FlashAttention (NL), section "Problemen met standaard
  attention"; the same formula, garbled, in FlashAttention (CS)).  The scale is
  an explicit argument (the formula's 1/sqrt(d_k) is the default the workloads
  use), and masking is part of the fused computation (FlashAttention (NL),
  "Samensmelting van bewerkingen in een CUDA-kernel": QK^T, masking, softmax,
  times V).  The method is exact, not an approximation (FlashAttention (NL)
  introduction; memory-optimized flash attention page, "How it compares"), so
  the oracle is the plain definition written out: it materialises the whole
  N x N score matrix S, which is exactly what the fused kernel avoids.
* Per-row logsumexp L_i = ln sum_j exp(S_ij), the only O(N) state the
  backward pass keeps.  The pages do not print it; it is the natural-log
  normaliser of the softmax above.
* Backward.  The pages say only that intermediates are recomputed instead of
  stored (memory-optimized flash attention page, "How it works").  The
  gradients are the chain rule of the forward definition:
  dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij, dS = P o (dP - D),
  dQ = scale dS K, dK = scale dS^T Q.  D is formed from P and dP here, not from
  the identity D_i = rowsum(dO o O) that a fused backward uses, so the two
  sides check each other.

Mask readings (the pages name masking and sliding-window attention, a purely
local window, but fix no convention; sparse-attention glossary, "Abgrenzung &
Vergleiche"):
  causal:   key j is allowed for query i iff j <= i (square self-attention);
  window W: additionally j >= i - W + 1 (the window counts the diagonal, so
            W = 1 keeps only key i);
  window W without causal: the local window on both sides, |i - j| <= W - 1
            (the same count convention: W = 1 keeps only key i);
  W = 0:    no band.
Every row keeps its diagonal, so no row is ever fully masked.

Shared K/V heads.  The pages list Multi-Query Attention among what FlashAttention-2
supports (FlashAttention (NL), "Evolutie en verdere ontwikkelingen",
FlashAttention-2): several query heads read one K/V head.  Reading, generalised to
H_kv K/V heads for H query heads (H a multiple of H_kv; H_kv = 1 is MQA): query head
h reads K/V head h // (H / H_kv), so each K/V head serves a contiguous group of query
heads, and its gradient is the sum over that group.

Few new rows over many keys (a generation step).  The pages name attention engines
for LLM inference that work on the key/value cache during streaming generation
(FlashAttention (NL), "Gespecialiseerde oplossingen": FlashInfer; its reference
list adds FlashDecoding++).  Reading: N_q query rows attend N_k >= N_q keys, and
query row i stands at position N_k - N_q + i of the key sequence (the new rows are
the last N_q positions, after the cached ones), so the causal and window masks
above apply to that position.  With N_q = N_k this is the self-attention above.

FP8 keys and values.  The pages say that FlashAttention-3 supports FP8 (FlashAttention (NL),
"Evolutie en verdere ontwikkelingen", FlashAttention-3), without a format.  Reading: the
E4M3 format of that paper's FP8 path -- 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits, exponent field 0 for subnormals, no infinities, S.1111.111 the only NaN -- with one
scale per tensor: K = s_k * E4M3(K8), V = s_v * E4M3(V8).  The attention is then the
definition above on those dequantised values, in fp64.

Arithmetic is numpy float64 with ``@`` (BLAS DGEMM) as the only library step.
Parity of every function here is pinned by tests/test_oracle.py.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "allowed_mask",
    "attention_forward",
    "attention_probabilities",
    "attention_backward",
    "attention_forward_rows",
    "attention_backward_rows",
    "allowed_pairs",
    "kv_head_of",
    "attention_forward_shared_kv",
    "attention_backward_shared_kv",
    "attention_forward_decode",
    "e4m3_to_float",
    "attention_forward_decode_fp8kv",
    "attention_forward_fp8",
]


def _check_mask_args(causal: bool, window: int) -> None:
    if window < 0:
        raise ValueError("window must be >= 0")


def allowed_mask(n_q: int, n_k: int, causal: bool, window: int, row_start: int = 0) -> np.ndarray:
    """Boolean [n_q, n_k]: True where key j may be attended by query row_start + i."""
    return _rows_mask(np.arange(row_start, row_start + n_q), n_k, causal, window)


def _scores(q: np.ndarray, k: np.ndarray, scale: float, ok: np.ndarray) -> np.ndarray:
    """S = scale * Q K^T with disallowed entries set to -inf (additive 0/-inf mask)."""
    s = scale * (q @ k.T)
    return np.where(ok, s, -np.inf)


def _softmax_rows(s: np.ndarray):
    """Row softmax of S together with the row logsumexp.

    m_i = max_j S_ij is subtracted before exponentiating so that exp never
    overflows; the result is the same softmax (the shift cancels).
    """
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    denom = np.sum(e, axis=1, keepdims=True)
    p = e / denom
    lse = (m + np.log(denom))[:, 0]
    return p, lse


def _head_forward(q, k, v, scale, causal, window, row_start=0):
    ok = allowed_mask(q.shape[0], k.shape[0], causal, window, row_start)
    p, lse = _softmax_rows(_scores(q, k, scale, ok))
    return p @ v, lse, p


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor
        x = x.detach().to("cpu")
        import torch  # local: only needed to widen bf16, which numpy lacks
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _per_head(fn, *arrays):
    """Apply fn to every [N, d] head slice of [..., N, d] arrays."""
    lead = arrays[0].shape[:-2]
    flat = [a.reshape((-1,) + a.shape[-2:]) for a in arrays]
    outs = [fn(*[f[h] for f in flat]) for h in range(flat[0].shape[0])]
    res = []
    for idx in range(len(outs[0])):
        stacked = np.stack([o[idx] for o in outs])
        res.append(stacked.reshape(lead + stacked.shape[1:]))
    return tuple(res)


def attention_forward(q, k, v, scale: float, causal: bool = False, window: int = 0):
    """O = softmax(scale Q K^T + mask) V and L = row logsumexp, in fp64.

    q, k, v: [..., N, d] (any float dtype, widened to fp64).
    Returns (O [..., N, d], L [..., N]).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    o, lse = _per_head(lambda a, b, c: _head_forward(a, b, c, scale, causal, window)[:2], q, k, v)
    return o, lse


def attention_probabilities(q, k, scale: float, causal: bool = False, window: int = 0):
    """P = softmax(scale Q K^T + mask), [..., N, N] (for tests on small N)."""
    q, k = _as64(q), _as64(k)

    def one(a, b):
        ok = allowed_mask(a.shape[0], b.shape[0], causal, window)
        return (_softmax_rows(_scores(a, b, scale, ok))[0],)

    return _per_head(one, q, k)[0]


def _head_backward(q, k, v, do, scale, causal, window):
    o, lse, p = _head_forward(q, k, v, scale, causal, window)
    dv = p.T @ do
    dp = do @ v.T
    d_row = np.sum(p * dp, axis=1, keepdims=True)
    ds = p * (dp - d_row)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def attention_backward(q, k, v, do, scale: float, causal: bool = False, window: int = 0):
    """Gradients of sum(O o dO) with respect to Q, K and V, in fp64.

    Returns (dQ, dK, dV), each [..., N, d].
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    return _per_head(lambda a, b, c, e: _head_backward(a, b, c, e, scale, causal, window), q, k, v, do)


def attention_forward_rows(q, k, v, scale: float, causal: bool = False, window: int = 0,
                           rows=None, block: int = 512):
    """Forward of ONE head ([N, d] inputs) for selected query rows.

    Materialises full-width row blocks of S (block x N) instead of the whole
    N x N matrix, so N = 32768 fits in host memory; each row is still the plain
    softmax over all N keys.  Returns (O [len(rows), d], L [len(rows)]).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    n = q.shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.size, v.shape[1]))
    lse = np.empty(rows.size)
    for b0 in range(0, rows.size, block):
        r = rows[b0:b0 + block]
        ok = _rows_mask(r, k.shape[0], causal, window)
        p, l_blk = _softmax_rows(_scores(q[r], k, scale, ok))
        o[b0:b0 + r.size] = p @ v
        lse[b0:b0 + r.size] = l_blk
    return o, lse


def _rows_mask(r: np.ndarray, n_k: int, causal: bool, window: int) -> np.ndarray:
    _check_mask_args(causal, window)
    i = r[:, None]
    j = np.arange(n_k)[None, :]
    ok = np.ones((r.size, n_k), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window + 1
        if not causal:
            ok &= j <= i + window - 1
    return ok


def attention_backward_rows(q, k, v, do, scale: float, causal: bool = False, window: int = 0,
                            key_rows=None, block: int = 512, query_rows=None):
    """Backward of ONE head for a subset of outputs, without an N x N buffer.

    dQ is returned for the query rows processed (all rows unless ``query_rows``
    is given); dK and dV for ``key_rows`` (all if None).  It is the same chain
    rule as ``attention_backward`` evaluated over full-width row blocks: each
    block of query rows contributes its part of dK and dV (dS^T Q and P^T dO).
    With ``query_rows`` the dK/dV returned are those rows' contributions only.
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    n = q.shape[0]
    key_rows = np.arange(n) if key_rows is None else np.asarray(key_rows, dtype=np.int64)
    qrows = np.arange(n) if query_rows is None else np.asarray(query_rows, dtype=np.int64)
    dq = np.empty((qrows.size, q.shape[1]))
    dk = np.zeros((key_rows.size, q.shape[1]))
    dv = np.zeros((key_rows.size, q.shape[1]))
    for b0 in range(0, qrows.size, block):
        sel = slice(b0, min(qrows.size, b0 + block))
        r = qrows[sel]
        ok = _rows_mask(r, n, causal, window)
        p, _ = _softmax_rows(_scores(q[r], k, scale, ok))
        dp = do[r] @ v.T
        d_row = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - d_row)
        dq[sel] = scale * (ds @ k)
        dk += scale * (ds[:, key_rows].T @ q[r])
        dv += p[:, key_rows].T @ do[r]
    return dq, dk, dv


def kv_head_of(n_heads: int, n_kv_heads: int) -> np.ndarray:
    """K/V head read by each of n_heads query heads (contiguous groups)."""
    if n_kv_heads < 1 or n_heads % n_kv_heads:
        raise ValueError("the query heads must be a whole multiple of the K/V heads")
    return np.arange(n_heads) // (n_heads // n_kv_heads)


def attention_forward_shared_kv(q, k, v, scale: float, causal: bool = False, window: int = 0):
    """Forward with shared K/V heads: q [..., H, N, d]; k, v [..., H_kv, N, d]."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    idx = kv_head_of(q.shape[-3], k.shape[-3])
    return attention_forward(q, k[..., idx, :, :], v[..., idx, :, :], scale, causal, window)


def attention_backward_shared_kv(q, k, v, do, scale: float, causal: bool = False, window: int = 0):
    """Gradients with shared K/V heads: dQ [..., H, N, d]; dK, dV [..., H_kv, N, d], each K/V
    head's gradient summed over the query heads that read it."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    h, h_kv = q.shape[-3], k.shape[-3]
    idx = kv_head_of(h, h_kv)
    dq, dk, dv = attention_backward(q, k[..., idx, :, :], v[..., idx, :, :], do, scale, causal, window)
    group = (h_kv, h // h_kv)
    dk = dk.reshape(dk.shape[:-3] + group + dk.shape[-2:]).sum(axis=-3)
    dv = dv.reshape(dv.shape[:-3] + group + dv.shape[-2:]).sum(axis=-3)
    return dq, dk, dv


def _decode_row_start(n_q: int, n_k: int) -> int:
    """Position, among the n_k keys, of the first of n_q new query rows: they are the last n_q."""
    return n_k - n_q


def attention_forward_decode(q, k, v, scale: float, causal: bool = False, window: int = 0):
    """Forward of N_q new query rows over N_k >= N_q keys: q [..., H, N_q, d];
    k, v [..., H_kv, N_k, d] (shared K/V heads as above).

    Query row i stands at key position N_k - N_q + i; the masks apply there.
    Returns (O [..., H, N_q, d], L [..., H, N_q]).
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    n_q, n_k = q.shape[-2], k.shape[-2]
    if n_q > n_k:
        raise ValueError("more query rows than keys")
    idx = kv_head_of(q.shape[-3], k.shape[-3])
    start = _decode_row_start(n_q, n_k)
    return _per_head(lambda a, b, c: _head_forward(a, b, c, scale, causal, window, start)[:2],
                     q, k[..., idx, :, :], v[..., idx, :, :])


def e4m3_to_float(codes) -> np.ndarray:
    """fp64 values of FP8 E4M3 codes (uint8): (-1)^s 2^(e-7) (1 + m/8) for exponent fields
    e = 1..15, (-1)^s 2^-6 (m/8) for e = 0, NaN for e = 15 with m = 7."""
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def attention_forward_decode_fp8kv(q, k8, v8, k_scale: float, v_scale: float, scale: float,
                                   causal: bool = False, window: int = 0):
    """attention_forward_decode with K = k_scale E4M3(k8) and V = v_scale E4M3(v8): q [..., H, N_q, d];
    k8, v8 uint8 codes [..., H_kv, N_k, d]."""
    if hasattr(k8, "detach"):
        k8, v8 = (x.detach().cpu().numpy() for x in (k8, v8))
    k = float(k_scale) * e4m3_to_float(k8)
    v = float(v_scale) * e4m3_to_float(v8)
    return attention_forward_decode(q, k, v, scale, causal, window)


def attention_forward_fp8(q8, k8, vt8, q_scale: float, k_scale: float, v_scale: float, scale: float,
                          causal: bool = False, window: int = 0):
    """The forward on E4M3 codes with one scale per tensor: Q = q_scale E4M3(q8) [..., H, N, d],
    K = k_scale E4M3(k8) [..., H_kv, N, d], and V = v_scale E4M3(vt8) given transposed,
    vt8 [..., H_kv, d, N]."""
    q8, k8, vt8 = (x.detach().cpu().numpy() if hasattr(x, "detach") else np.asarray(x) for x in (q8, k8, vt8))
    q = float(q_scale) * e4m3_to_float(q8)
    k = float(k_scale) * e4m3_to_float(k8)
    v = float(v_scale) * np.swapaxes(e4m3_to_float(vt8), -1, -2)
    return attention_forward_shared_kv(q, k, v, scale, causal, window)


def allowed_pairs(n: int, causal: bool, window: int) -> int:
    """Number of (query, key) pairs the mask keeps in an N x N self-attention."""
    _check_mask_args(causal, window)
    total = 0
    for i in range(n):
        lo = 0
        hi = i if causal else n - 1
        if window > 0:
            lo = max(0, i - window + 1)
            if not causal:
                hi = min(n - 1, i + window - 1)
        total += hi - lo + 1
    return total

"""Full-size parity samples of the benchmark arms whose only other parity tests are small
shapes: head dimension 256 (forward and backward), the FP8 (E4M3) forward, and the decode step
over an E4M3 K/V cache.  Each runs the whole workload on the B200 in the launch configuration
the bench times, and the fp64 oracle checks whole heads: seeded ones plus the last head of
every batch entry (the grid runs heads in order, so those are CTAs of the final wave).
"""

import numpy as np
import pytest

from oracle import attention as orc
from synthetic import WORKLOADS, head_subset, make_grad_output, make_inputs, make_inputs_fp8, make_inputs_fp8kv
from tests.parity import assert_forward_close, assert_grads_close, fp8_o_bound, L_MAX_ABS, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_77_b200.build import build
    build()
    import exact_io_aware_77_b200 as fa
    fa.load()
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)
    return fa


def _heads(wl, n_random):
    return sorted(set(head_subset(wl, n_random)) | {(b + 1) * wl.H - 1 for b in range(wl.B)})


def test_d256_workload_head_sample(fa):
    """B2 H16 N4096 d256 causal, forward and backward, 8 whole heads (O, L, dQ, dK, dV)."""
    wl = WORKLOADS["d256"]
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    heads = _heads(wl, 8)
    assert len(heads) >= 8
    sel = lambda x: x.reshape(wl.BH, wl.N, wl.d)[heads]
    o_ref, l_ref = orc.attention_forward(sel(q), sel(k), sel(v), wl.scale, wl.causal, wl.window)
    assert_forward_close(sel(o.cpu()), lse.cpu().reshape(wl.BH, wl.N)[heads], o_ref, l_ref, ("d256", heads))
    refs = orc.attention_backward(sel(q), sel(k), sel(v), sel(do), wl.scale, wl.causal, wl.window)
    assert_grads_close([sel(dq.cpu()), sel(dk.cpu()), sel(dv.cpu())], refs, ("d256", heads))


def test_fp8_workload_head_sample(fa):
    """The causal B2 H32 N4096 d128 shape on E4M3 Q, K, V: 8 whole heads against the oracle on
    the dequantised codes, within the per-element bound derived from the E4M3 rounding of P."""
    wl = WORKLOADS["causal"]
    q8, k8, vt8, s_q, s_k, s_v = make_inputs_fp8(wl)
    o, lse = fa.forward_fp8(q8.cuda(), k8.cuda(), vt8.cuda(), s_q, s_k, s_v, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    o64, l64 = to64(o), to64(lse)
    assert np.isfinite(o64).all()
    heads = _heads(wl, 8)
    assert len(heads) >= 8
    for flat in heads:
        b, h = divmod(flat, wl.H)
        one = (slice(b, b + 1), slice(h, h + 1))
        o_ref, l_ref = orc.attention_forward_fp8(q8[one], k8[one], vt8[one], s_q, s_k, s_v, wl.scale, wl.causal,
                                                 wl.window)
        assert np.abs(l64[one] - l_ref).max() <= L_MAX_ABS, ("fp8", b, h)
        qf = s_q * orc.e4m3_to_float(q8[one].numpy())
        kf = s_k * orc.e4m3_to_float(k8[one].numpy())
        vf = s_v * np.swapaxes(orc.e4m3_to_float(vt8[one].numpy()), -1, -2)
        bound = fp8_o_bound(qf, kf, vf, wl.scale, wl.causal, wl.window, o_ref)
        err = np.abs(o64[one] - o_ref)
        assert np.all(err <= bound), ("fp8", b, h, float((err - bound).max()))


def test_decode_fp8_workload_head_sample(fa):
    """The generation step over an E4M3 K/V cache, full size (B8, 64 query heads on 8 K/V heads,
    one new row over 32768 keys, causal): 24 seeded query heads against the oracle on the
    dequantised cache."""
    wl = WORKLOADS["decode"]
    q, k8, v8, s_k, s_v = make_inputs_fp8kv(wl)
    o, lse = fa.decode_fp8kv(q.cuda(), k8.cuda(), v8.cuda(), s_k, s_v, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    o, lse = o.cpu(), lse.cpu()
    g = wl.H // wl.kv_heads
    for flat in sorted(set(head_subset(wl, 24)) | {wl.BH - 1}):
        b, h = divmod(flat, wl.H)
        kv = h // g
        o_ref, l_ref = orc.attention_forward_decode_fp8kv(q[b:b + 1, h:h + 1], k8[b:b + 1, kv:kv + 1],
                                                          v8[b:b + 1, kv:kv + 1], s_k, s_v, wl.scale, wl.causal,
                                                          wl.window)
        assert_forward_close(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], o_ref, l_ref, ("decode_fp8", b, h))

"""B200 parity of the head-dimension-256 forward and backward, the FP8 (E4M3) forward, the decode
kernels over an E4M3 K/V cache and at d = 256, and the persistent forward and backward, with the
tolerances of the other parity tests (the FP8 forward's derived per-element bound from
tests/parity.py).  The persistent kernels are also held bit for bit to the one-item-per-CTA ones.
"""

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import Workload, make_grad_output, make_inputs, make_inputs_fp8, make_inputs_fp8kv
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


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [
    (1, 2, 2, 300, True, 0), (1, 4, 2, 400, False, 50), (2, 2, 1, 257, True, 3), (1, 2, 2, 128, True, 0)])
def test_d256_forward_and_backward(fa, B, H, H_kv, N, causal, window):
    wl = Workload("d256_pending", B, H, N, 256, causal, window, seed=121 + N, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, causal, window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, causal, window)
    assert fa.check_status() == 0
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, causal, window)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, (B, H, H_kv, N, causal, window))
    refs = orc.attention_backward_shared_kv(q, k, v, do, wl.scale, causal, window)
    assert_grads_close([dq.cpu(), dk.cpu(), dv.cpu()], refs, (B, H, H_kv, N, causal, window))


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,ctas,schedule", [
    (1, 2, 2, 300, 128, True, 0, 1, "balanced"), (1, 2, 2, 300, 128, True, 0, 2, "head_major"),
    (2, 2, 1, 600, 128, False, 0, 3, "balanced"), (1, 4, 2, 520, 128, True, 100, 0, "balanced"),
    (2, 2, 1, 257, 64, True, 3, 2, "head_major"), (1, 3, 3, 1000, 64, False, 0, 0, "balanced"),
    (2, 3, 3, 700, 64, True, 0, 5, "balanced"), (1, 1, 1, 1, 128, True, 0, 0, "balanced"),
    (1, 2, 2, 300, 256, True, 0, 1, "balanced"), (1, 4, 2, 400, 256, False, 50, 0, "balanced"),
    (2, 2, 1, 257, 256, True, 3, 3, "head_major")])
def test_persistent_forward(fa, B, H, H_kv, N, d, causal, window, ctas, schedule):
    """The persistent grid against the oracle, and bit for bit against the one-item-per-CTA
    forward: every tile meets the same arithmetic in the same order."""
    wl = Workload("persist_pending", B, H, N, d, causal, window, seed=141 + N, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = fa.forward(qd, kd, vd, wl.scale, causal, window, persistent=True, ctas=ctas, schedule=schedule)
    o1, lse1 = fa.forward(qd, kd, vd, wl.scale, causal, window)
    assert fa.check_status() == 0
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, causal, window)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, (B, H, H_kv, N, d, causal, window, ctas))
    assert torch.equal(o, o1) and torch.equal(lse, lse1)


def test_persistent_forward_strided(fa):
    """Sequence-major [B, N, H, d] arrays (strided views): the persistent grid equals the
    one-item-per-CTA forward on the same views bit for bit, and the oracle within tolerance."""
    B, H, H_kv, N, d = 2, 4, 2, 333, 128
    wl = Workload("persist_strided", B, H, N, d, True, 0, seed=151, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    qs, ks, vs = (x.transpose(1, 2).contiguous().cuda().transpose(1, 2) for x in (q, k, v))
    out = torch.empty(B, N, H, d, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o, lse = fa.forward(qs, ks, vs, wl.scale, True, 0, out=out, persistent=True, ctas=7)
    o1, lse1 = fa.forward(qs, ks, vs, wl.scale, True, 0)
    assert fa.check_status() == 0
    assert torch.equal(o, o1) and torch.equal(lse, lse1)
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, True, 0)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, "strided persistent")


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,ctas,schedule", [
    (1, 2, 2, 300, 128, True, 0, 1, "balanced"), (1, 4, 2, 400, 128, False, 50, 3, "balanced"),
    (2, 2, 1, 257, 64, True, 3, 2, "head_major"), (2, 2, 2, 520, 64, True, 0, 0, "balanced"),
    (1, 2, 2, 1000, 128, False, 0, 0, "head_major")])
def test_persistent_backward(fa, B, H, H_kv, N, d, causal, window, ctas, schedule):
    """The persistent recompute kernel against the oracle; dK and dV bit for bit against the
    one-item-per-CTA kernel (each is summed inside one CTA), dQ to rounding (its fp32 reductions
    arrive in hardware order in both)."""
    wl = Workload("persist_bwd_pending", B, H, N, d, causal, window, seed=161 + N, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, causal, window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, causal, window, persistent=True, ctas=ctas,
                             schedule=schedule)
    dq1, dk1, dv1 = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, causal, window)
    assert fa.check_status() == 0
    assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
    assert (dq.float() - dq1.float()).abs().max().item() <= 1e-2 * max(dq1.float().abs().max().item(), 1e-3)
    refs = orc.attention_backward_shared_kv(q, k, v, do, wl.scale, causal, window)
    assert_grads_close([dq.cpu(), dk.cpu(), dv.cpu()], refs, (B, H, H_kv, N, d, causal, window, ctas, schedule))


@pytest.mark.parametrize("schedule", ["balanced", "head_major"])
def test_persistent_forward_full_size(fa, schedule):
    """The causal B2 H32 N4096 d128 workload: the persistent grid (one CTA per SM, several
    items each) equals the one-item-per-CTA forward bit for bit; sampled rows against the oracle."""
    from synthetic import WORKLOADS
    wl = WORKLOADS["causal"]
    q, k, v = make_inputs(wl)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window, persistent=True, schedule=schedule)
    o1, lse1 = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    assert torch.equal(o, o1) and torch.equal(lse, lse1)
    b, h = 1, 17
    rows = [0, 127, 128, 2049, wl.N - 1]
    o_ref, l_ref = orc.attention_forward(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], wl.scale,
                                         wl.causal, wl.window)
    got = to64(o[b, h, rows])
    assert np.abs(got - o_ref[0, 0, rows]).max() <= 2e-2
    assert np.abs(to64(lse[b, h, rows]) - l_ref[0, 0, rows]).max() <= L_MAX_ABS


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [
    (1, 2, 2, 256, True, 0), (1, 2, 1, 400, True, 0), (1, 2, 2, 304, False, 0), (1, 4, 2, 512, True, 100)])
def test_fp8_forward(fa, B, H, H_kv, N, causal, window):
    wl = Workload("fp8_pending", B, H, N, 128, causal, window, seed=131 + N, H_kv=H_kv)
    q8, k8, vt8, s_q, s_k, s_v = make_inputs_fp8(wl)
    o, lse = fa.forward_fp8(q8.cuda(), k8.cuda(), vt8.cuda(), s_q, s_k, s_v, wl.scale, causal, window)
    assert fa.check_status() == 0
    o_ref, l_ref = orc.attention_forward_fp8(q8, k8, vt8, s_q, s_k, s_v, wl.scale, causal, window)
    o64, l64 = to64(o), to64(lse)
    assert np.isfinite(o64).all() and np.abs(l64 - l_ref).max() <= L_MAX_ABS
    q = s_q * orc.e4m3_to_float(q8.numpy())
    k = s_k * orc.e4m3_to_float(k8.numpy())
    v = s_v * np.swapaxes(orc.e4m3_to_float(vt8.numpy()), -1, -2)
    bound = fp8_o_bound(q, k, v, wl.scale, causal, window, o_ref)
    assert np.all(np.abs(o64 - o_ref) <= bound), float((np.abs(o64 - o_ref) - bound).max())


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,causal,window,fp8", [
    (2, 8, 2, 3, 1000, 128, True, 0, True), (1, 2, 1, 5, 777, 64, False, 50, True),
    (1, 4, 1, 2, 700, 256, True, 0, False), (1, 2, 2, 9, 100, 256, False, 20, False),
    (1, 4, 1, 2, 700, 256, True, 0, True)])
def test_decode_fp8kv_and_d256(fa, B, H, H_kv, N_q, N_k, d, causal, window, fp8):
    wl = Workload("decode_pending", B, H, N_k, d, causal, window, seed=141 + N_k, H_kv=H_kv, Nq=N_q)
    if fp8:
        q, k8, v8, s_k, s_v = make_inputs_fp8kv(wl)
        o, lse = fa.decode_fp8kv(q.cuda(), k8.cuda(), v8.cuda(), s_k, s_v, wl.scale, causal, window)
        o_ref, l_ref = orc.attention_forward_decode_fp8kv(q, k8, v8, s_k, s_v, wl.scale, causal, window)
    else:
        q, k, v = make_inputs(wl)
        o, lse = fa.decode(q.cuda(), k.cuda(), v.cuda(), wl.scale, causal, window)
        o_ref, l_ref = orc.attention_forward_decode(q, k, v, wl.scale, causal, window)
    assert fa.check_status() == 0
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, (B, H, H_kv, N_q, N_k, d, causal, window, fp8))

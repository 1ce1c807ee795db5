"""B200 parity of the head-dimension-256 forward and backward, the FP8 (E4M3) forward, and the
decode kernels over an E4M3 K/V cache and at d = 256, with the tolerances of the other parity
tests (the FP8 forward's derived per-element bound from tests/parity.py).
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

"""Shared K/V heads (multi-query and grouped-query attention) vs the fp64 oracle.

Query head h reads K/V head h // (H / H_kv); dK and dV sum over each K/V head's query heads.
Forward and backward run through the C ABI (fa_fwd_gqa / fa_bwd_gqa via the binding) on
small shapes compared in full, and on the causal N = 4096 shape with 8 K/V heads compared on
seeded heads, with the tolerances of the other parity tests.
"""

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import WORKLOADS, Workload, make_grad_output, make_inputs
from tests.parity import assert_forward_close, assert_grads_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_77_b200.build import build
    build()
    import exact_io_aware_77_b200 as fa
    fa.load()
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)
    return fa


SHAPES = [
    # B, H, H_kv, N, d, causal, window
    (1, 4, 1, 300, 64, True, 0),       # multi-query
    (2, 8, 2, 1000, 128, False, 0),
    (1, 6, 3, 513, 128, True, 100),
    (1, 4, 2, 777, 64, False, 50),     # two-sided window
    (1, 2, 1, 129, 128, False, 0),
    (1, 8, 4, 640, 128, True, 0),
]


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window", SHAPES)
def test_shared_kv_forward_and_backward(fa, B, H, H_kv, N, d, causal, window):
    wl = Workload("gqa_edge", B, H, N, d, causal, window, seed=41 + N + H_kv, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, causal, window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, causal, window)
    assert fa.check_status() == 0
    assert dk.shape == k.shape and dv.shape == v.shape
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, causal, window)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, (B, H, H_kv, N, d, causal, window))
    refs = orc.attention_backward_shared_kv(q, k, v, do, wl.scale, causal, window)
    assert_grads_close([dq.cpu(), dk.cpu(), dv.cpu()], refs, (B, H, H_kv, N, d, causal, window))


def test_equal_heads_match_plain_entry_points(fa):
    """fa_fwd_gqa with H_kv = H gives exactly what fa_fwd gives."""
    wl = Workload("gqa_eq", 1, 3, 300, 128, True, 0, seed=43)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    o1, l1 = fa.forward(q, k, v, wl.scale, True, 0)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    st = fa._lib.fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), 1, 3, 3, 300,
                            128, wl.scale, 1, 0, torch.cuda.current_stream().cuda_stream)
    assert st == 0 and fa.check_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_workload_head_sample(fa):
    """The causal B2 H32 N4096 d128 shape with 8 K/V heads, full size on the GPU; the oracle
    checks two query heads of one group and the gradient of their K/V head."""
    wl = WORKLOADS["gqa"]
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    g = wl.H // wl.kv_heads
    b, kv = 1, 5                                  # K/V head 5 of batch entry 1 and its query heads
    heads = list(range(kv * g, (kv + 1) * g))
    qs, dos = q[b, heads][None], do[b, heads][None]
    ks, vs = k[b, kv][None, None], v[b, kv][None, None]
    o_ref, l_ref = orc.attention_forward_shared_kv(qs, ks, vs, wl.scale, True, 0)
    assert_forward_close(o[b, heads][None].cpu(), lse[b, heads][None].cpu(), o_ref, l_ref, "gqa")
    refs = orc.attention_backward_shared_kv(qs, ks, vs, dos, wl.scale, True, 0)
    assert_grads_close([dq[b, heads][None].cpu(), dk[b, kv][None, None].cpu(), dv[b, kv][None, None].cpu()],
                       refs, "gqa")

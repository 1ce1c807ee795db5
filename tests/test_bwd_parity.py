"""Backward kernels vs the fp64 oracle's chain rule, through the C ABI.

The GPU backward consumes the GPU forward's O and L (as a user would); the oracle
computes dQ, dK, dV from Q, K, V, dO alone.  Gradients must agree to relative L2
<= 1e-2.  Small shapes are compared in full; the causal N=4096 workload is launched
at full size and compared on seeded heads.
"""

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import WORKLOADS, Workload, head_subset, make_grad_output, make_inputs
from tests.parity import assert_grads_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_77_b200.build import build
    build()
    import exact_io_aware_77_b200 as fa
    fa.load()
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)   # a correct pipeline never waits this long
    return fa


def _gpu_grads(fa, wl, q, k, v, do):
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


EDGE = [
    (1, 1, 1, 64, False, 0), (1, 1, 1, 128, True, 0), (1, 2, 17, 128, True, 0), (1, 2, 63, 64, False, 0),
    (1, 2, 64, 128, True, 0), (1, 2, 65, 64, True, 0), (2, 2, 127, 128, False, 0), (1, 2, 129, 128, True, 0),
    (1, 2, 300, 64, True, 7), (1, 2, 300, 128, True, 1), (1, 2, 640, 128, True, 129),
    (1, 2, 1000, 128, True, 200), (1, 1, 1000, 64, True, 2000), (2, 1, 777, 128, False, 0),
    (1, 2, 1024, 128, True, 0), (1, 1, 1536, 64, False, 0),
    # two-sided local windows (causal = 0)
    (1, 2, 300, 128, False, 1), (1, 2, 300, 64, False, 7), (1, 2, 1000, 128, False, 200),
    (1, 1, 640, 128, False, 129), (2, 1, 777, 64, False, 2000),
]


@pytest.mark.parametrize("B,H,N,d,causal,window", EDGE)
def test_small_shapes(fa, B, H, N, d, causal, window):
    wl = Workload("edge", B, H, N, d, causal, window, seed=31 + N + d + window)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl, seed=77 + N)
    grads = _gpu_grads(fa, wl, q, k, v, do)
    refs = orc.attention_backward(q, k, v, do, wl.scale, causal, window)
    assert_grads_close(grads, refs, (B, H, N, d, causal, window))


def test_workload_bwd_full_size_head_sample(fa):
    wl = WORKLOADS["bwd"]
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    grads = _gpu_grads(fa, wl, q, k, v, do)
    # seeded heads plus the first head of batch entry 1 and the last head (the final wave)
    heads = sorted(set(head_subset(wl, 7)) | {wl.H, wl.BH - 1})
    assert len(heads) >= 8
    sel = lambda x: x.reshape(wl.BH, wl.N, wl.d)[heads]
    refs = orc.attention_backward(sel(q), sel(k), sel(v), sel(do), wl.scale, wl.causal, wl.window)
    assert_grads_close([sel(g) for g in grads], refs, ("bwd", heads))


@pytest.mark.parametrize("name", ["long", "swa"])
def test_long_window_backward_sampled(fa, name):
    """N = 32768 with a 4096 window (one-sided and two-sided long-context shapes, 2 heads): dK/dV
    on sampled key rows and dQ on one row block, against the oracle's row-block backward."""
    wl = WORKLOADS[name].with_(H=2)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl, seed=2005)
    dq, dk, dv = _gpu_grads(fa, wl, q, k, v, do)
    rng = np.random.default_rng(5)
    key_rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(wl.N - 64, wl.N),
                                         rng.choice(wl.N, 128, replace=False)]))
    qrows = np.arange(8192, 8192 + 512)
    h = 1
    qh, kh, vh, doh = (x[0, h] for x in (q, k, v, do))
    # dK/dV need every query row; dQ only its own rows
    _, dk_ref, dv_ref = orc.attention_backward_rows(qh, kh, vh, doh, wl.scale, wl.causal, wl.window,
                                                    key_rows=key_rows)
    dq_ref, _, _ = orc.attention_backward_rows(qh, kh, vh, doh, wl.scale, wl.causal, wl.window,
                                               key_rows=key_rows[:1], query_rows=qrows)
    assert_grads_close([dq[0, h][qrows], dk[0, h][key_rows], dv[0, h][key_rows]],
                       [dq_ref, dk_ref, dv_ref], name)


def test_workspace_and_guard_bands(fa):
    """Grads are written exactly in place; the workspace is O(N*d) and the only extra memory."""
    wl = Workload("guard", 1, 2, 300, 128, True, 0, seed=3)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    do = make_grad_output(wl).cuda()
    o, lse = fa.forward(q, k, v, wl.scale, True, 0)
    n, pad = q.numel(), 4096
    bufs = [torch.full((n + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    grads = tuple(b[pad:pad + n].view_as(q) for b in bufs)
    need = fa.bwd_workspace_size(1, 2, 300, 128)
    assert need == 4 * 2 * 384 * (128 + 2)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    fa.backward(q, k, v, o, lse, do, wl.scale, True, 0, grads=grads, workspace=ws)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == base
    assert fa.check_status() == 0
    for b in bufs:
        assert torch.all(b[:pad] == 7.0) and torch.all(b[-pad:] == 7.0)
    with pytest.raises(fa.FAError) as e:
        fa.backward(q, k, v, o, lse, do, wl.scale, True, 0, grads=grads, workspace=ws[:need - 16])
    assert e.value.status == fa.STATUS["FA_ERR_WORKSPACE"]


def test_repeat_is_deterministic_within_tolerance(fa):
    """Two backward calls on the same inputs agree (fp32 reductions may reorder, bf16 outputs
    differ at most by rounding)."""
    wl = Workload("rep", 1, 2, 512, 128, True, 0, seed=8)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    g1 = _gpu_grads(fa, wl, q, k, v, do)
    g2 = _gpu_grads(fa, wl, q, k, v, do)
    for a, b in zip(g1, g2):
        assert torch.allclose(a.float(), b.float(), rtol=1e-2, atol=1e-3)


def test_phases_in_turn_equal_one_call(fa):
    """Preprocess, recompute and finalise run one by one give fa_bwd's result bit for bit."""
    wl = Workload("phases", 1, 3, 700, 128, True, 300, seed=21)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    do = make_grad_output(wl).cuda()
    o, lse = fa.forward(q, k, v, wl.scale, True, 300)
    ref = fa.backward(q, k, v, o, lse, do, wl.scale, True, 300)
    ws = torch.empty(fa.bwd_workspace_size(1, 3, 700, 128), dtype=torch.uint8, device="cuda")
    grads = tuple(torch.empty_like(q) for _ in range(3))
    for ph in (1, 2, 4):
        fa.backward(q, k, v, o, lse, do, wl.scale, True, 300, grads=grads, workspace=ws, phases=ph)
    assert fa.check_status() == 0
    # dK and dV are written once per key row; dQ sums fp32 reductions whose order may differ
    assert torch.equal(grads[1], ref[1]) and torch.equal(grads[2], ref[2])
    assert torch.allclose(grads[0].float(), ref[0].float(), rtol=1e-2, atol=1e-3)

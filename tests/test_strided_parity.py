"""Arrays with arbitrary strides (fa_fwd_strided / fa_bwd_strided through the binding).

The sequence-major [B, N, H, d] layout, and a row-padded layout, hold the same logical
[B, H, N, d] values as the packed tensors.  The forward and dK, dV must equal the packed path's
bit for bit (the same kernels read the same values); dQ (summed by reductions in a varying
order) and everything must also match the fp64 oracle within the usual tolerances.
"""

import pytest
import torch

from oracle import attention as orc
from synthetic import Workload, make_grad_output, make_inputs
from tests.parity import GRAD_REL_L2, assert_forward_close, assert_grads_close, rel_l2, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_77_b200.build import build
    build()
    import exact_io_aware_77_b200 as fa
    fa.load()
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)
    return fa


def _seq_major(x):
    """The same values as x [B, H, N, d], stored as [B, N, H, d] (a strided view)."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def _row_padded(x, pad=64):
    """The same values with every row followed by `pad` unused elements."""
    B, H, N, d = x.shape
    buf = torch.full((B, H, N, d + pad), float("nan"), dtype=x.dtype, device=x.device)
    buf[..., :d] = x
    return buf[..., :d]


CASES = [
    # B, H, H_kv, N, d, causal, window, layout
    (2, 4, 4, 300, 128, True, 0, "seq"),
    (1, 4, 2, 513, 64, False, 0, "seq"),
    (1, 2, 2, 777, 128, False, 100, "pad"),
    (2, 6, 3, 1000, 128, True, 200, "seq"),
]


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window,layout", CASES)
def test_strided_matches_packed_and_oracle(fa, B, H, H_kv, N, d, causal, window, layout):
    wl = Workload("strided", B, H, N, d, causal, window, seed=51 + N, H_kv=H_kv)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    do = make_grad_output(wl).cuda()
    view = _seq_major if layout == "seq" else _row_padded
    qs, ks, vs, dos = (view(x) for x in (q, k, v, do))
    assert not qs.is_contiguous()
    # packed path
    o, lse = fa.forward(q, k, v, wl.scale, causal, window)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, wl.scale, causal, window)
    # strided path: strided inputs, a strided O and strided gradients
    o_s = view(torch.empty_like(q))
    o_s, lse_s = fa.forward(qs, ks, vs, wl.scale, causal, window, out=o_s)
    grads_s = tuple(view(torch.empty_like(x)) for x in (q, k, v))
    dq_s, dk_s, dv_s = fa.backward(qs, ks, vs, o_s, lse_s, dos, wl.scale, causal, window, grads=grads_s)
    assert fa.check_status() == 0
    assert torch.equal(o_s, o) and torch.equal(lse_s, lse)
    assert torch.equal(dk_s, dk) and torch.equal(dv_s, dv)
    assert rel_l2(to64(dq_s), to64(dq)) <= GRAD_REL_L2 / 10
    qc, kc, vc, doc = (x.cpu() for x in (q, k, v, do))
    o_ref, l_ref = orc.attention_forward_shared_kv(qc, kc, vc, wl.scale, causal, window)
    assert_forward_close(o_s.cpu(), lse_s.cpu(), o_ref, l_ref, (B, H, H_kv, N, d, layout))
    refs = orc.attention_backward_shared_kv(qc, kc, vc, doc, wl.scale, causal, window)
    assert_grads_close([dq_s.cpu(), dk_s.cpu(), dv_s.cpu()], refs, (B, H, H_kv, N, d, layout))

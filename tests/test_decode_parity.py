"""Decode-shaped forward (a few new query rows over a longer key sequence) vs the fp64 oracle.

Query row i stands at key position N_k - N_q + i; the masks apply there.  The split-key
kernels run through the C ABI (fa_fwd_decode via the binding): small shapes compared in
full (one split and many, several row blocks, every mask kind, shared K/V heads, d = 64 and
128, strided arrays), and the 32768-key generation step the benchmark times compared on
seeded heads, with the tolerances of the other parity tests.
"""

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import WORKLOADS, Workload, head_subset, make_inputs
from tests.parity import assert_forward_close

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
    # B, H, H_kv, N_q, N_k, d, causal, window
    (1, 1, 1, 1, 1, 64, True, 0),          # one key
    (1, 2, 2, 1, 1, 128, False, 0),
    (1, 4, 1, 1, 300, 128, True, 0),       # multi-query, two splits
    (2, 8, 2, 3, 1000, 128, True, 0),      # 12 rows per K/V head, seven splits
    (1, 4, 4, 20, 20, 64, True, 0),        # N_q = N_k: self-attention, two row blocks
    (1, 2, 1, 5, 777, 128, False, 0),
    (1, 2, 1, 5, 777, 128, True, 100),     # causal window: the visited keys start at 672
    (1, 2, 1, 5, 777, 64, False, 50),      # two-sided window, cut at the end of the keys
    (1, 2, 2, 37, 37, 128, False, 5),
    (1, 2, 2, 37, 37, 128, True, 3),
    (1, 3, 3, 2, 40, 64, True, 1000),      # window wider than the keys
    (2, 16, 2, 1, 3000, 128, True, 0),     # 21 splits
    (1, 8, 1, 4, 2049, 64, False, 0),      # 32 rows: two row blocks, 15 splits
    (1, 6, 2, 7, 129, 128, True, 17),
    (1, 2, 2, 64, 4096, 128, True, 300),   # splits some rows see no key of
    (1, 2, 1, 64, 4096, 64, False, 200),
    (1, 1, 1, 600, 600, 128, True, 0),     # 38 row blocks; CTAs with no key at all
    (1, 2, 2, 300, 2000, 64, True, 0),
]


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,causal,window", SHAPES)
def test_decode_forward(fa, B, H, H_kv, N_q, N_k, d, causal, window):
    wl = Workload("decode_edge", B, H, N_k, d, causal, window, seed=51 + N_k + N_q, H_kv=H_kv, Nq=N_q)
    q, k, v = make_inputs(wl)
    o, lse = fa.decode(q.cuda(), k.cuda(), v.cuda(), wl.scale, causal, window)
    assert fa.check_status() == 0
    assert o.shape == q.shape and lse.shape == (B, H, N_q)
    o_ref, l_ref = orc.attention_forward_decode(q, k, v, wl.scale, causal, window)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, (B, H, H_kv, N_q, N_k, d, causal, window))


def test_decode_equals_self_attention_rows(fa):
    """N_q = N_k through the decode kernels agrees with the self-attention forward kernel to
    within both results' rounding (they share no code)."""
    wl = Workload("decode_self", 1, 4, 333, 128, True, 0, seed=61, H_kv=2)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    o1, l1 = fa.decode(q, k, v, wl.scale, True, 0)
    o2, l2 = fa.forward(q, k, v, wl.scale, True, 0)
    assert fa.check_status() == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_decode_strided(fa):
    """Sequence-major [B, N, heads, d] storage viewed as [B, heads, N, d] gives the packed result."""
    wl = Workload("decode_strided", 2, 8, 900, 128, True, 0, seed=62, H_kv=2, Nq=3)
    q, k, v = make_inputs(wl)
    qs, ks, vs = (x.transpose(1, 2).contiguous().cuda().transpose(1, 2) for x in (q, k, v))
    out = torch.empty(2, 3, 8, 128, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o, lse = fa.decode(qs, ks, vs, wl.scale, True, 0, out=out)
    o_p, l_p = fa.decode(q.cuda(), k.cuda(), v.cuda(), wl.scale, True, 0)
    assert fa.check_status() == 0
    assert torch.equal(o, o_p) and torch.equal(lse, l_p)


def test_decode_workspace_and_errors(fa):
    """A caller workspace is used as given; a short one and N_q > N_k are refused."""
    wl = Workload("decode_ws", 1, 8, 5000, 64, True, 0, seed=63, H_kv=1, Nq=2)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    need = fa.decode_workspace_size(1, 8, 1, 2, 5000, 64, True, 0)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o1, l1 = fa.decode(q, k, v, wl.scale, True, 0, workspace=ws)
    o2, l2 = fa.decode(q, k, v, wl.scale, True, 0)
    assert fa.check_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    with pytest.raises(fa.FAError):
        fa.decode(q, k, v, wl.scale, True, 0, workspace=ws[: need - 16])
    with pytest.raises(ValueError):
        fa.decode(k[:, :, :3].expand(1, 8, 3, 64).contiguous(), q[:, :1, :1].contiguous(),
                  q[:, :1, :1].contiguous(), wl.scale, True, 0)


def test_decode_workload_head_sample(fa):
    """The benchmark's generation step, full size on the GPU (B8, 64 query heads on 8 K/V heads,
    one new row over 32768 keys, causal); the oracle checks 24 seeded query heads."""
    wl = WORKLOADS["decode"]
    q, k, v = make_inputs(wl)
    o, lse = fa.decode(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    o, lse = o.cpu(), lse.cpu()
    g = wl.H // wl.kv_heads
    for flat in head_subset(wl, 24):
        b, h = divmod(flat, wl.H)
        kv = h // g
        o_ref, l_ref = orc.attention_forward_decode(q[b:b + 1, h:h + 1], k[b:b + 1, kv:kv + 1],
                                                    v[b:b + 1, kv:kv + 1], wl.scale, wl.causal, wl.window)
        assert_forward_close(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], o_ref, l_ref, ("decode", b, h))

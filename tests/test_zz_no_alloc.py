"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers may not call cudaMalloc and have no allocator to ask -- an operator living
inside a host framework that owns all device memory, or a service that forbids allocation
once it is running.  fa_bwd_noalloc serves them with scratch kept inside the library.  This
test calls it through the C ABI twice in a row and checks each result against fa_bwd (which
uses a caller workspace), with the gradient tolerance of the other tests.  It also checks
that a problem too large for the built-in scratch is refused before anything runs.

The file name sorts last so that a run stopping at the first failure has already run every
other test; the test also passes on its own in a fresh process.
"""

import gc

import pytest
import torch

from synthetic import Workload, make_grad_output, make_inputs
from tests.parity import GRAD_REL_L2, rel_l2, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from exact_io_aware_77_b200.build import build
    build()
    import exact_io_aware_77_b200 as fa
    fa.load()
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)
    return fa


def _noalloc(fa, wl, q, k, v, o, lse, do, grads):
    dq, dk, dv = grads
    return fa._lib.fa_bwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), wl.B, wl.H, wl.N, wl.d, wl.scale,
        int(wl.causal), wl.window, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_backward_twice(fa):
    wl = Workload("noalloc", 1, 4, 1000, 128, True, 0, seed=12)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    do = make_grad_output(wl).cuda()
    o, lse = fa.forward(q, k, v, wl.scale, wl.causal, wl.window)
    ref = fa.backward(q, k, v, o, lse, do, wl.scale, wl.causal, wl.window)
    ref = [to64(g) for g in ref]
    assert fa.check_status() == 0

    for call in range(2):
        grads = tuple(torch.full_like(q, float("nan")) for _ in range(3))
        gc.collect()
        torch.cuda.synchronize()
        allocs_before = torch.cuda.memory_stats()["allocation.all.allocated"]
        st = _noalloc(fa, wl, q, k, v, o, lse, do, grads)
        assert st == 0, fa.STATUS_NAMES.get(st, st)
        assert fa.check_status() == 0
        # no device allocation went through torch during the call
        assert torch.cuda.memory_stats()["allocation.all.allocated"] == allocs_before
        for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
            err = rel_l2(g, r)
            assert err <= GRAD_REL_L2, (call, name, err)


def test_noalloc_rejects_problems_beyond_its_scratch(fa):
    # 32 heads of N = 4096, d = 128 need 4*32*4096*130 bytes > 64 MiB
    assert fa.bwd_workspace_size(1, 32, 4096, 128) > 64 << 20
    wl = Workload("big", 1, 32, 4096, 128, True, 0)
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(16, dtype=torch.float32, device="cuda")
    st = _noalloc(fa, wl, t, t, t, t, lse, t, (t, t, t))
    assert fa.STATUS_NAMES[st] == "FA_ERR_NOALLOC_LIMIT"
    assert fa.check_status() == 0

"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers may not call cudaMalloc and have no allocator to ask -- an operator living
inside a host framework that owns all device memory, or a service that forbids allocation
once it is running.  fa_bwd_noalloc serves them with scratch kept inside the library.  This
test calls it through the C ABI twice in a row per shape and checks each result

  * against the fp64 oracle, with the gradient tolerance of the other parity tests;
  * against fa_bwd (which uses a caller workspace and runs the same kernels): dK and dV bit for
    bit, since each is summed inside one CTA in a fixed order; dQ to rounding, since its fp32
    partial sums reach the scratch in hardware order;
  * for allocation: neither torch's allocator counter nor the device's free memory
    (cudaMemGetInfo) may change across the call.

It also checks that a problem too large for the built-in scratch is refused before anything
runs.  The file name sorts last so that a run stopping at the first failure has already run
every other test; the test also passes on its own in a fresh process.
"""

import gc

import numpy as np
import pytest
import torch

from oracle import attention as orc
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


@pytest.mark.parametrize("B,H,N,d,causal,window", [
    (1, 4, 1000, 128, True, 0),     # causal, ragged last tile
    (1, 3, 777, 64, False, 50),     # two-sided window, d = 64
    (2, 2, 500, 64, True, 100),     # causal band
])
def test_noalloc_matches_oracle_and_workspace_backward_twice(fa, B, H, N, d, causal, window):
    wl = Workload("noalloc", B, H, N, d, causal, window, seed=12 + N)
    q_h, k_h, v_h = make_inputs(wl)
    do_h = make_grad_output(wl)
    q, k, v, do = (x.cuda() for x in (q_h, k_h, v_h, do_h))
    o, lse = fa.forward(q, k, v, wl.scale, causal, window)
    ref = fa.backward(q, k, v, o, lse, do, wl.scale, causal, window)
    assert fa.check_status() == 0
    oracle = orc.attention_backward(q_h, k_h, v_h, do_h, wl.scale, causal, window)

    for call in range(2):
        grads = tuple(torch.full_like(q, float("nan")) for _ in range(3))
        gc.collect()
        torch.cuda.synchronize()
        allocs_before = torch.cuda.memory_stats()["allocation.all.allocated"]
        free_before = torch.cuda.mem_get_info()[0]
        st = _noalloc(fa, wl, q, k, v, o, lse, do, grads)
        assert st == 0, fa.STATUS_NAMES.get(st, st)
        assert fa.check_status() == 0
        # no device allocation, through torch or directly through the CUDA runtime
        assert torch.cuda.memory_stats()["allocation.all.allocated"] == allocs_before
        assert torch.cuda.mem_get_info()[0] == free_before
        dq, dk, dv = grads
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2]), call
        dq64, dq_ref = to64(dq), to64(ref[0])
        assert np.abs(dq64 - dq_ref).max() <= 1e-2 * max(np.abs(dq_ref).max(), 1e-3), call
        for name, g, r in zip(("dq", "dk", "dv"), grads, oracle):
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

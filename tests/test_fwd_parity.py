"""Forward kernel vs the fp64 oracle, through the C ABI, on seeded inputs.

Small shapes are compared element by element (several tiles, ragged tails, every mask
kind, d = 64 and 128); the named workloads are launched at full size exactly as the
bench launches them and compared on seeded head (and, for N = 32768, row) samples.
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
    fa._lib.fa_set_wait_limit_ns(1_000_000_000)   # a correct pipeline never waits this long
    return fa


def _run(fa, wl):
    q, k, v = make_inputs(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window)
    assert fa.check_status() == 0
    return (q, k, v), o.cpu(), lse.cpu()


EDGE = [
    # B, H, N, d, causal, window
    (1, 1, 1, 64, False, 0), (1, 1, 1, 128, True, 0), (1, 2, 17, 64, False, 0),
    (1, 2, 17, 128, True, 0), (2, 3, 127, 64, True, 0), (1, 2, 128, 128, False, 0),
    (1, 2, 129, 64, True, 0), (1, 2, 129, 128, False, 0), (2, 2, 300, 128, True, 5),
    (1, 2, 300, 64, True, 1), (1, 3, 1000, 128, True, 128), (1, 2, 1000, 64, True, 200),
    (1, 2, 777, 128, True, 2000), (1, 1, 640, 128, True, 129), (2, 2, 513, 64, False, 0),
    (1, 2, 1024, 128, True, 0), (1, 1, 2048, 64, False, 0), (1, 2, 900, 128, True, 256),
    # two-sided local windows (causal = 0): narrower, equal to and wider than a tile, ragged N
    (1, 2, 300, 128, False, 1), (1, 2, 300, 64, False, 5), (2, 2, 1000, 128, False, 128),
    (1, 2, 777, 64, False, 200), (1, 1, 640, 128, False, 129), (1, 2, 513, 128, False, 2000),
]


@pytest.mark.parametrize("B,H,N,d,causal,window", EDGE)
def test_small_shapes_elementwise(fa, B, H, N, d, causal, window):
    wl = Workload("edge", B, H, N, d, causal, window, seed=7 + N + d + window)
    (q, k, v), o, lse = _run(fa, wl)
    o_ref, l_ref = orc.attention_forward(q, k, v, wl.scale, causal, window)
    assert_forward_close(o, lse, o_ref, l_ref, (B, H, N, d, causal, window))


def test_large_magnitude_scores(fa):
    """Q, K with std 3 give scores of std 9 (peaked rows, |S| up to ~40): the running max
    keeps exp2 in range.  V stays N(0, 1) so |O| stays where the absolute bf16 bound applies."""
    wl = Workload("big", 1, 2, 384, 128, True, 0, std=3.0, seed=99)
    q, k, _ = make_inputs(wl)
    v = make_inputs(wl.with_(std=1.0), seed=100)[2]
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), wl.scale, True, 0)
    assert fa.check_status() == 0
    o_ref, l_ref = orc.attention_forward(q, k, v, wl.scale, True, 0)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, "qk std=3")


def test_tiny_scale(fa):
    """scale -> 0 approaches uniform attention; L -> ln(#keys)."""
    wl = Workload("tiny_scale", 1, 2, 200, 64, True, 0, seed=5)
    q, k, v = make_inputs(wl)
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), 1e-6, True, 0)
    assert fa.check_status() == 0
    o_ref, l_ref = orc.attention_forward(q, k, v, 1e-6, True, 0)
    assert_forward_close(o.cpu(), lse.cpu(), o_ref, l_ref, "scale=1e-6")
    assert np.max(np.abs(lse.cpu().numpy()[0, 0] - np.log(np.arange(1, 201)))) < 1e-3


def test_workload_tiny_full(fa):
    wl = WORKLOADS["tiny"]
    (q, k, v), o, lse = _run(fa, wl)
    o_ref, l_ref = orc.attention_forward(q, k, v, wl.scale, wl.causal, wl.window)
    assert_forward_close(o, lse, o_ref, l_ref, "tiny")


def sampled_heads(wl, n_random):
    """Seeded heads plus the first head of the last batch entry and the last head overall: the
    grid runs heads in order, so the last ones are the CTAs of the final wave."""
    return sorted(set(head_subset(wl, n_random)) | {(wl.B - 1) * wl.H, wl.BH - 1})


@pytest.mark.parametrize("name,n_heads", [("gpt2", 7), ("causal", 7)])
def test_workload_full_size_head_sample(fa, name, n_heads):
    """Whole heads (every query tile, the last included) of the full-size workloads."""
    wl = WORKLOADS[name]
    (q, k, v), o, lse = _run(fa, wl)
    heads = sampled_heads(wl, n_heads)
    assert len(heads) >= 8 or wl.BH < 8
    qf, kf, vf = (x.reshape(wl.BH, wl.N, wl.d)[heads] for x in (q, k, v))
    o_ref, l_ref = orc.attention_forward(qf, kf, vf, wl.scale, wl.causal, wl.window)
    assert_forward_close(o.reshape(wl.BH, wl.N, wl.d)[heads], lse.reshape(wl.BH, wl.N)[heads],
                         o_ref, l_ref, (name, heads))


@pytest.mark.parametrize("name", ["long", "swa"])
def test_workload_long_window_sampled_rows(fa, name):
    wl = WORKLOADS[name]
    (q, k, v), o, lse = _run(fa, wl)
    rng = np.random.default_rng(wl.seed)
    rows = np.unique(np.concatenate([
        np.arange(0, 160), np.arange(4000, 4200), np.arange(wl.N - 160, wl.N),
        rng.choice(wl.N, 400, replace=False)]))
    for h in head_subset(wl, wl.oracle_heads):
        qh, kh, vh = (x.reshape(wl.BH, wl.N, wl.d)[h] for x in (q, k, v))
        o_ref, l_ref = orc.attention_forward_rows(qh, kh, vh, wl.scale, wl.causal, wl.window, rows=rows)
        assert_forward_close(o.reshape(wl.BH, wl.N, wl.d)[h][rows], lse.reshape(wl.BH, wl.N)[h][rows],
                             o_ref, l_ref, (name, h))


def test_guard_bands_untouched(fa):
    """O and L written exactly in place: sentinels around both survive."""
    wl = Workload("guard", 1, 2, 300, 128, True, 0, seed=3)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    n_o, n_l, pad = q.numel(), wl.BH * wl.N, 4096
    ob = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lb = torch.full((n_l + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = ob[pad:pad + n_o].view_as(q)
    l = lb[pad:pad + n_l].view(wl.B, wl.H, wl.N)
    fa.forward(q, k, v, wl.scale, True, 0, out=o, lse=l)
    assert fa.check_status() == 0
    for buf in (ob, lb):
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
    assert torch.all(torch.isfinite(o.float())) and torch.all(torch.isfinite(l))


def test_no_extra_device_memory(fa):
    """The forward allocates nothing: device memory in use is the same before and after."""
    for n in (4096, 8192, 16384, 32768):
        wl = Workload("mem", 1, 2, n, 128, True, 4096, seed=1)
        q, k, v = (x.cuda() for x in make_inputs(wl))
        o = torch.empty_like(q)
        l = torch.empty((1, 2, n), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        fa.forward(q, k, v, wl.scale, True, 4096, out=o, lse=l)
        torch.cuda.synchronize()
        assert torch.cuda.max_memory_allocated() == base
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0
        assert fa.check_status() == 0


def test_bad_alignment_rejected_on_device(fa):
    wl = Workload("al", 1, 1, 64, 64, seed=1)
    q, k, v = (x.cuda() for x in make_inputs(wl))
    flat = torch.empty(q.numel() + 1, dtype=torch.bfloat16, device="cuda")
    q_off = flat[1:].view_as(q)   # 2-byte offset: not 16-byte aligned
    with pytest.raises(fa.FAError) as e:
        fa.forward(q_off, k, v)
    assert e.value.status == fa.STATUS["FA_ERR_ALIGN"]


def test_timeout_selftest_reports_and_recovers(fa):
    """A wait that nothing completes runs out, is reported once, and the context stays usable."""
    from exact_io_aware_77_b200 import _lib
    s = torch.cuda.current_stream().cuda_stream
    assert fa.check_status() == 0
    assert _lib.fa_selftest_timeout(2_000_000, s) == 0        # 2 ms limit
    assert fa.check_status() == fa.STATUS["FA_ERR_TIMEOUT"]
    assert fa.check_status() == 0
    test_workload_tiny_full(fa)

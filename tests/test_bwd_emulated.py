"""The backward kernels' own CUDA source (fa_bwd_prep, fa_bwd_kernel<D> at d = 64/128,
fa_bwd256_kernel at d = 256, fa_bwd_dq_final), run on the CPU under the emulation of
tests/host_emu/, vs the oracle's gradients.

Test infrastructure only (see tests/test_fwd_emulated.py for what the emulation restates).
The one inline-asm helper bwd_kernel.cuh holds itself (the untiled bulk copy) is replaced, in
the emulation's copy of the header only, by the stub's stand-in.  O and L come from the oracle
(O rounded to bf16), so the check covers the backward alone.  Tolerance: relative L2 <= 1e-2
per gradient, with the RMS floor of tests/parity.py where a gradient is exactly zero.
"""

import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import Workload, make_grad_output, make_inputs
from tests.parity import GRAD_REL_L2, rel_l2


@pytest.fixture(scope="module")
def emu_bwd(tmp_path_factory):
    from tests.host_emu.build_emu import build_many
    d = str(tmp_path_factory.mktemp("host_emu_bwd"))
    try:
        return build_many(d, {
            64: ("bwd_kernel.cuh", "emu_bwd_main.cpp", "emu_bwd_64", ("EMU_D=64",)),
            128: ("bwd_kernel.cuh", "emu_bwd_main.cpp", "emu_bwd_128", ("EMU_D=128",)),
            256: (["bwd256_kernel.cuh", "bwd_kernel.cuh"], "emu_bwd_main.cpp", "emu_bwd_256", ("EMU_BWD256",)),
            "128_eager": ("bwd_kernel.cuh", "emu_bwd_main.cpp", "emu_bwd_128_eager", ("EMU_D=128", "EMU_EAGER_COPIES")),
            "128_eager_mma": ("bwd_kernel.cuh", "emu_bwd_main.cpp", "emu_bwd_128_eager_mma",
                              ("EMU_D=128", "EMU_EAGER_MMA")),
            "256_eager_mma": (["bwd256_kernel.cuh", "bwd_kernel.cuh"], "emu_bwd_main.cpp", "emu_bwd_256_eager_mma",
                              ("EMU_BWD256", "EMU_EAGER_MMA")),
            "256_eager": (["bwd256_kernel.cuh", "bwd_kernel.cuh"], "emu_bwd_main.cpp", "emu_bwd_256_eager",
                          ("EMU_BWD256", "EMU_EAGER_COPIES")),
        })
    except FileNotFoundError:
        pytest.skip("g++ not available")


CASES = [
    # B, H, H_kv, N, d, causal, window
    (1, 2, 2, 300, 128, True, 0),      # ragged: three key tiles, query tiles past the diagonal
    (1, 4, 2, 400, 128, False, 50),    # two-sided window, two query heads per K/V head
    (2, 2, 1, 257, 64, True, 3),       # multi-query, narrow causal window
    (1, 1, 1, 600, 64, True, 1),       # window 1: dQ = dK = 0, dV = dO
    # head dimension 256 (fa_bwd256_kernel: one CTA per 64-key tile)
    (1, 1, 1, 128, 256, True, 0),
    (1, 1, 1, 300, 256, True, 1),
    (1, 2, 2, 300, 256, False, 0),
]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy()


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window", CASES)
def test_bwd_kernels_emulated(emu_bwd, B, H, H_kv, N, d, causal, window):
    _check_bwd_emulated(emu_bwd[d], [], B, H, H_kv, N, d, causal, window)


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [(1, 2, 2, 300, True, 0), (1, 4, 2, 200, False, 50)])
def test_bwd_kernel_emulated_eager_copies(emu_bwd, B, H, H_kv, N, causal, window):
    """fa_bwd_kernel with copies that land as soon as they are issued: a Q, dO (or L, D) load
    before the MMAs released the buffer would overwrite operands still to be read."""
    _check_bwd_emulated(emu_bwd["128_eager"], [], B, H, H_kv, N, 128, causal, window)


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [(1, 2, 2, 300, True, 0), (1, 4, 2, 200, False, 50)])
def test_bwd_kernel_emulated_eager_mma(emu_bwd, B, H, H_kv, N, causal, window):
    """fa_bwd_kernel with MMAs that run as soon as they are issued: a dV, dK or dQ product issued
    before P^T or dS^T is in place reads it too early."""
    _check_bwd_emulated(emu_bwd["128_eager_mma"], [], B, H, H_kv, N, 128, causal, window)


@pytest.mark.parametrize("kind", ["256_eager_mma", "256_eager"])
@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [(1, 2, 2, 300, True, 0), (1, 4, 2, 200, False, 50)])
def test_bwd256_kernel_emulated_eager(emu_bwd, kind, B, H, H_kv, N, causal, window):
    """fa_bwd256_kernel with MMAs that run at issue (the second dQ half must wait for the first
    half's readout, since both use the same TMEM columns) and with copies that land at issue (a
    Q or dO load before the MMAs of the previous query tile released the stage)."""
    _check_bwd_emulated(emu_bwd[kind], [], B, H, H_kv, N, 256, causal, window)


def _check_bwd_emulated(exe, extra, B, H, H_kv, N, d, causal, window):
    wl = Workload("bwd_emu", B, H, N, d, causal, window, seed=95 + N + H_kv, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    do = make_grad_output(wl)
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, causal, window)
    with tempfile.TemporaryDirectory() as tmp:
        pre = os.path.join(tmp, "x")
        for name, t in (("q", q), ("k", k), ("v", v), ("o", torch.from_numpy(o_ref).to(torch.bfloat16)), ("do", do)):
            _bits(t).tofile(pre + "." + name)
        l_ref.astype(np.float32).tofile(pre + ".lse")
        r = subprocess.run([exe, str(B), str(H), str(H_kv), str(N), str(int(causal)), str(window),
                            repr(wl.scale), pre] + extra, capture_output=True, text=True, timeout=1800)
        assert r.returncode == 0, r.stdout[-1000:] + r.stderr[-4000:]
        outs = [torch.from_numpy(np.fromfile(pre + "." + n, dtype=np.int16)).view(torch.bfloat16).double().numpy()
                for n in ("dq", "dk", "dv")]
    refs = orc.attention_backward_shared_kv(q, k, v, do, wl.scale, causal, window)
    for name, g, ref in zip(("dq", "dk", "dv"), outs, refs):
        g = g.reshape(ref.shape)
        assert np.isfinite(g).all(), f"{name} not written"
        assert rel_l2(g, ref) <= GRAD_REL_L2, (name, rel_l2(g, ref))

"""The tcgen05 forward kernels' own CUDA source (fa_fwd_kernel at d = 64 and 128,
fa_fwd256_kernel at d = 256), run on the CPU under an emulation of their primitives, vs the
oracle.

Test infrastructure only.  tests/host_emu/sm100_stub.cuh restates the documented behaviour of
the sm_100a primitives fwd_kernel.cuh uses -- mbarrier phases and transaction counts, 4-D TMA
tile loads with the 128-byte swizzle and zero fill, TMEM (128 lanes x 512 columns, one lane
quadrant per warp), and kind::f16 MMAs that read their operands through the shared-memory
descriptors (K-major and MN-major 128-byte-swizzled layouts) or from TMEM -- with one host
thread per CUDA thread.  The pure helpers (descriptor encoders, the FMA-pipe exponential) are
cut from the real sm100.cuh, not restated.  Compiled with AddressSanitizer and
UndefinedBehaviorSanitizer: an access outside shared memory, TMEM or a tensor aborts the run,
as does an mbarrier misuse or a TMEM access outside the warp's lane quadrant.  Outputs start as
NaN.  What this cannot show is timing and the hardware's own reading of the descriptors; the
GPU parity tests (tests/test_fwd_parity.py) are the check of those.
"""

import os
import tempfile

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import Workload, make_inputs, make_inputs_fp8
from tests.parity import L_MAX_ABS, O_MAX_ABS, O_MEAN_ABS, fp8_o_bound


@pytest.fixture(scope="module")
def emu_fwd(tmp_path_factory):
    from tests.host_emu.build_emu import build_many
    d = str(tmp_path_factory.mktemp("host_emu_fwd"))
    try:
        return build_many(d, {
            64: ("fwd_kernel.cuh", "emu_fwd_main.cpp", "emu_fwd_64", ("EMU_D=64",)),
            128: ("fwd_kernel.cuh", "emu_fwd_main.cpp", "emu_fwd_128", ("EMU_D=128",)),
            256: (["fwd256_kernel.cuh", "fwd_kernel.cuh"], "emu_fwd_main.cpp", "emu_fwd_256", ("EMU_FWD256",)),
            "fp8": (["fwd_fp8_kernel.cuh", "fwd_kernel.cuh"], "emu_fwd_main.cpp", "emu_fwd_fp8", ("EMU_FWD_FP8",)),
            "128_eager": ("fwd_kernel.cuh", "emu_fwd_main.cpp", "emu_fwd_128_eager", ("EMU_D=128", "EMU_EAGER_COPIES")),
            "128_eager_mma": ("fwd_kernel.cuh", "emu_fwd_main.cpp", "emu_fwd_128_eager_mma",
                              ("EMU_D=128", "EMU_EAGER_MMA")),
            "64_eager_mma": ("fwd_kernel.cuh", "emu_fwd_main.cpp", "emu_fwd_64_eager_mma", ("EMU_D=64", "EMU_EAGER_MMA")),
            "256_eager_mma": (["fwd256_kernel.cuh", "fwd_kernel.cuh"], "emu_fwd_main.cpp", "emu_fwd_256_eager_mma",
                              ("EMU_FWD256", "EMU_EAGER_MMA")),
            "fp8_eager_mma": (["fwd_fp8_kernel.cuh", "fwd_kernel.cuh"], "emu_fwd_main.cpp", "emu_fwd_fp8_eager_mma",
                              ("EMU_FWD_FP8", "EMU_EAGER_MMA")),
        })
    except FileNotFoundError:
        pytest.skip("g++ not available")


CASES = [
    # B, H, H_kv, N, d, causal, window
    (1, 1, 1, 128, 128, True, 0),       # one tile pair, second tile past N
    (1, 2, 2, 300, 128, True, 0),       # ragged: two CTA pairs, partial last tile
    (1, 2, 2, 300, 128, False, 0),
    (1, 2, 1, 520, 128, True, 100),     # causal window, shared K/V head
    (1, 4, 2, 400, 128, False, 50),     # two-sided window
    (1, 2, 2, 700, 64, False, 0),
    (2, 2, 1, 257, 64, True, 3),        # multi-query, narrow window, ragged
    (1, 1, 1, 1000, 64, True, 1),       # window 1: O = V
    # head dimension 256 (fa_fwd256_kernel: one query tile per CTA, 64-key K/V tiles)
    (1, 1, 1, 128, 256, True, 0),
    (1, 2, 2, 300, 256, True, 0),
    (1, 2, 2, 300, 256, False, 0),
    (1, 2, 1, 520, 256, True, 100),
    (1, 4, 2, 400, 256, False, 50),
    (2, 2, 1, 257, 256, True, 3),
]


@pytest.mark.parametrize("B,H,H_kv,N,d,causal,window", CASES)
def test_fwd_kernel_emulated(emu_fwd, B, H, H_kv, N, d, causal, window):
    _check_fwd_emulated(emu_fwd[d], [], B, H, H_kv, N, d, causal, window)


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", [
    (1, 2, 2, 300, True, 0), (2, 2, 1, 600, False, 0), (1, 4, 2, 520, True, 100), (1, 2, 2, 1000, False, 200)])
def test_fwd_kernel_emulated_eager_copies(emu_fwd, B, H, H_kv, N, causal, window):
    """fa_fwd_kernel with TMA copies that land as soon as they are issued: a load into a K/V ring
    slot before the products reading its previous tile have completed would overwrite it."""
    _check_fwd_emulated(emu_fwd["128_eager"], [], B, H, H_kv, N, 128, causal, window)


@pytest.mark.parametrize("kind,B,H,H_kv,N,d,causal,window,extra", [
    ("128_eager_mma", 1, 2, 2, 300, 128, True, 0, []),
    ("128_eager_mma", 2, 2, 1, 600, 128, False, 0, []),
    ("128_eager_mma", 1, 4, 2, 520, 128, True, 100, []),
    ("64_eager_mma", 1, 2, 2, 1000, 64, False, 200, []),
    ("256_eager_mma", 1, 2, 2, 300, 256, True, 0, []),
    ("256_eager_mma", 1, 4, 2, 400, 256, False, 50, [])])
def test_fwd_kernel_emulated_eager_mma(emu_fwd, kind, B, H, H_kv, N, d, causal, window, extra):
    """MMAs that run as soon as they are issued (the other legal extreme to running at the next
    commit): a product issued before its operands are ready (P in TMEM, a K/V tile) reads them
    too early."""
    _check_fwd_emulated(emu_fwd[kind], extra, B, H, H_kv, N, d, causal, window)


def _check_fwd_emulated(exe, extra, B, H, H_kv, N, d, causal, window):
    import subprocess
    wl = Workload("fwd_emu", B, H, N, d, causal, window, seed=91 + N + H_kv, H_kv=H_kv)
    q, k, v = make_inputs(wl)
    with tempfile.TemporaryDirectory() as tmp:
        pre = os.path.join(tmp, "x")
        for name, t in zip("qkv", (q, k, v)):
            t.contiguous().view(torch.int16).numpy().tofile(pre + "." + name)
        r = subprocess.run([exe, str(B), str(H), str(H_kv), str(N), str(int(causal)), str(window),
                            repr(wl.scale), pre] + extra, capture_output=True, text=True, timeout=900)
        assert r.returncode == 0, r.stdout[-1000:] + r.stderr[-4000:]
        o = np.fromfile(pre + ".o", dtype=np.uint16)
        lse = np.fromfile(pre + ".lse", dtype=np.float32).reshape(B, H, N)
    o = torch.from_numpy(o.view(np.int16).copy()).view(torch.bfloat16).reshape(q.shape).double().numpy()
    o_ref, l_ref = orc.attention_forward_shared_kv(q, k, v, wl.scale, causal, window)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "a row was not written"
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse - l_ref).max() <= L_MAX_ABS


@pytest.mark.parametrize("d", [128, 256])
def test_fwd_kernel_emulated_late_rescales(emu_fwd, d):
    """Keys that score ever higher along the sequence make many rows' maxima grow by more than
    2^8 after their first key tile, so the lazy rescale of O runs at later tiles (with the d = 256
    kernel's two S buffers it must first wait for the previous P V product)."""
    import subprocess
    N = 400
    g = torch.Generator().manual_seed(97)
    q, k, v = (torch.randn(1, 1, N, d, generator=g) for _ in range(3))
    qdir = q.mean(dim=2, keepdim=True)
    k = k + torch.linspace(0, 6.0, N).view(1, 1, N, 1) * qdir / qdir.norm() * 40.0
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    scale = 1.0 / d ** 0.5
    s = scale * (q.double() @ k.double().transpose(-1, -2))[0, 0].numpy()
    late = sum((s[i, :i + 1].max() - s[i, :min(64, i + 1)].max()) / np.log(2) > 8 for i in range(64, N))
    assert late > 100, late   # the case does exercise late rescales
    with tempfile.TemporaryDirectory() as tmp:
        pre = os.path.join(tmp, "x")
        for name, t in zip("qkv", (q, k, v)):
            t.contiguous().view(torch.int16).numpy().tofile(pre + "." + name)
        r = subprocess.run([emu_fwd[d], "1", "1", "1", str(N), "1", "0", repr(scale), pre],
                           capture_output=True, text=True, timeout=900)
        assert r.returncode == 0, r.stderr[-4000:]
        o = np.fromfile(pre + ".o", dtype=np.uint16)
        lse = np.fromfile(pre + ".lse", dtype=np.float32).reshape(1, 1, N)
    o = torch.from_numpy(o.view(np.int16).copy()).view(torch.bfloat16).reshape(q.shape).double().numpy()
    o_ref, l_ref = orc.attention_forward(q, k, v, scale, True, 0)
    assert np.isfinite(o).all()
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse - l_ref).max() <= L_MAX_ABS


FP8_CASES = [
    # B, H, H_kv, N, causal, window (d = 128; N a multiple of 16 for the transposed V)
    (1, 2, 2, 256, True, 0),
    (1, 2, 1, 400, True, 0),
    (1, 2, 2, 304, False, 0),
    (1, 4, 2, 512, True, 100),
    (2, 2, 1, 144, False, 40),
]


@pytest.mark.parametrize("B,H,H_kv,N,causal,window", FP8_CASES)
def test_fwd_fp8_kernel_emulated(emu_fwd, B, H, H_kv, N, causal, window):
    """The FP8 forward (E4M3 Q, K, V^T with per-tensor scales) against the oracle on the
    dequantised values.  Tolerance, derived: the kernel rounds each P to E4M3 before P V
    (relative error <= 2^-4 for normal values, absolute <= 2^-10 below E4M3's normal range) while l
    sums the exact P, so with w_j = exp(s_j - max s) over the allowed keys,
    |dO_c| <= sum_j max(2^-4 w_j, 2^-10) |V_jc| / sum_j w_j; plus bf16 rounding of O (2^-8 |O|) and
    1e-3 for the fp32 exponentials and sums.  L uses the exact P: the usual 1e-3."""
    import subprocess
    d = 128
    wl = Workload("fwd_fp8_emu", B, H, N, d, causal, window, seed=99 + N + H_kv, H_kv=H_kv)
    q8, k8, vt8, s_q, s_k, s_v = make_inputs_fp8(wl)
    with tempfile.TemporaryDirectory() as tmp:
        pre = os.path.join(tmp, "x")
        for name, t in zip("qkv", (q8, k8, vt8)):
            t.contiguous().numpy().tofile(pre + "." + name)
        r = subprocess.run([emu_fwd["fp8"], str(B), str(H), str(H_kv), str(N), str(int(causal)), str(window),
                            repr(wl.scale), pre, repr(s_q), repr(s_k), repr(s_v)],
                           capture_output=True, text=True, timeout=900)
        assert r.returncode == 0, r.stderr[-4000:]
        o = np.fromfile(pre + ".o", dtype=np.uint16)
        lse = np.fromfile(pre + ".lse", dtype=np.float32).reshape(B, H, N)
    o = torch.from_numpy(o.view(np.int16).copy()).view(torch.bfloat16).reshape(B, H, N, d).double().numpy()
    o_ref, l_ref = orc.attention_forward_fp8(q8, k8, vt8, s_q, s_k, s_v, wl.scale, causal, window)
    assert np.isfinite(o).all()
    assert np.abs(lse - l_ref).max() <= L_MAX_ABS
    q = s_q * orc.e4m3_to_float(q8.numpy())
    k = s_k * orc.e4m3_to_float(k8.numpy())
    v = s_v * np.swapaxes(orc.e4m3_to_float(vt8.numpy()), -1, -2)
    bound = fp8_o_bound(q, k, v, wl.scale, causal, window, o_ref)
    assert np.all(np.abs(o - o_ref) <= bound), float((np.abs(o - o_ref) - bound).max())


def test_fwd_fp8_kernel_emulated_eager_mma(emu_fwd):
    """The FP8 forward with MMAs that run as soon as they are issued: a P V product issued before
    the softmax warps staged P8 in shared memory would read it too early."""
    test_fwd_fp8_kernel_emulated({"fp8": emu_fwd["fp8_eager_mma"]}, 1, 4, 2, 512, True, 100)

"""The decode kernels' own CUDA source, run on the CPU under a SIMT emulation, vs the oracle.

Test infrastructure only.  tests/host_emu/ holds a host stand-in for the handful of device
primitives decode_kernel.cuh uses (barriers, warp shuffles, mbarriers, TMA tensor loads,
ldmatrix and the m16n8k16 MMA, emulated from their documented semantics).  The kernel source is compiled with
g++ under AddressSanitizer and UndefinedBehaviorSanitizer, so every global or shared-memory
access outside its buffer aborts the run; outputs start as NaN, so a row the kernels fail to
write fails the comparison.  This checks the kernels' index arithmetic, masks, split plan
and merges without a GPU; the fragment layouts themselves are checked only on the GPU
(tests/test_decode_parity.py).  The library never uses any of this.
"""

import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from oracle import attention as orc
from synthetic import Workload, make_inputs, make_inputs_fp8kv
from tests.parity import O_MAX_ABS, O_MEAN_ABS, L_MAX_ABS

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "exact_io_aware_77_b200", "csrc")


@pytest.fixture(scope="module")
def emu_binary_eager(tmp_path_factory):
    from tests.host_emu.build_emu import build
    try:
        return build(str(tmp_path_factory.mktemp("host_emu_eager")), "decode_kernel.cuh", "emu_main.cpp",
                     "emu_main_eager", defines=("EMU_EAGER_COPIES",))
    except FileNotFoundError:
        pytest.skip("g++ not available")


@pytest.fixture(scope="module")
def emu_binary(tmp_path_factory):
    from tests.host_emu.build_emu import build
    try:
        return build(str(tmp_path_factory.mktemp("host_emu")), "decode_kernel.cuh", "emu_main.cpp", "emu_main")
    except FileNotFoundError:
        pytest.skip("g++ not available")


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _run(exe, wl, seq_major=False, fp8=False):
    if fp8:
        q, k, v, s_k, s_v = make_inputs_fp8kv(wl)
    else:
        q, k, v = make_inputs(wl)
    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if seq_major:   # [B, N, heads, d] storage seen as [B, heads, N, d]
        store = [x.transpose(1, 2).contiguous() for x in (q, k, v)]
        views = [x.transpose(1, 2) for x in store]
        o_store = torch.zeros(B, Nq, H, d, dtype=torch.bfloat16)
        o_view = o_store.transpose(1, 2)
    else:
        store, views = [q, k, v], [q, k, v]
        o_store = o_view = torch.zeros(B, H, Nq, d, dtype=torch.bfloat16)
    strides = [s for t in views + [o_view] for s in t.stride()[:3]]
    with tempfile.TemporaryDirectory() as tmp:
        pre = os.path.join(tmp, "x")
        for name, t in zip("qkv", store):
            (t.contiguous().numpy() if t.dtype == torch.uint8 else _bits(t)).tofile(pre + "." + name)
        args = [B, H, Hkv, Nq, Nk, d, int(wl.causal), wl.window, repr(wl.scale)] + strides + \
               [t.numel() for t in store] + [o_store.numel(), pre]
        if fp8:
            args += [repr(s_k), repr(s_v)]
        r = subprocess.run([exe] + [str(a) for a in args], capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout + r.stderr[-4000:]
        o_bits = np.fromfile(pre + ".o", dtype=np.uint16)
        lse = np.fromfile(pre + ".lse", dtype=np.float32).reshape(B, H, Nq)
    o = torch.from_numpy(o_bits.view(np.int16).copy()).view(torch.bfloat16).reshape(o_store.shape)
    o = (o.transpose(1, 2) if seq_major else o).double().numpy()
    if fp8:
        o_ref, l_ref = orc.attention_forward_decode_fp8kv(q, k, v, s_k, s_v, wl.scale, wl.causal, wl.window)
    else:
        o_ref, l_ref = orc.attention_forward_decode(q, k, v, wl.scale, wl.causal, wl.window)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "a row was not written"
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (err.max(), err.mean())
    assert np.abs(lse - l_ref).max() <= L_MAX_ABS
    return r.stdout


CASES = [
    # B, H, H_kv, N_q, N_k, d, causal, window
    (1, 1, 1, 1, 1, 64, True, 0),
    (1, 4, 1, 1, 300, 128, True, 0),        # two splits
    (2, 8, 2, 3, 1000, 128, True, 0),       # seven splits, 12 rows
    (1, 4, 4, 20, 20, 64, True, 0),         # two row blocks
    (1, 2, 1, 5, 777, 128, True, 100),      # visited keys start past 0
    (1, 2, 1, 5, 777, 64, False, 50),       # two-sided window at the end of the keys
    (1, 2, 2, 37, 37, 128, False, 5),
    (1, 3, 3, 2, 40, 64, True, 1000),
    (1, 2, 2, 64, 4096, 128, True, 300),    # splits that some rows see no key of
    (1, 2, 1, 1, 8192, 64, True, 0),        # 64 splits: the merge reads them 32 at a time
    (1, 4, 1, 2, 700, 256, True, 0),        # head dimension 256, split merge with 8 columns per lane
    (1, 2, 2, 9, 100, 256, False, 20),
]


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,causal,window", CASES)
def test_decode_kernel_emulated(emu_binary, B, H, H_kv, N_q, N_k, d, causal, window):
    wl = Workload("decode_emu", B, H, N_k, d, causal, window, seed=71 + N_k + N_q, H_kv=H_kv, Nq=N_q)
    out = _run(emu_binary, wl)
    assert out.startswith("plan ")


FP8_CASES = [
    (1, 4, 1, 1, 300, 128, True, 0),
    (2, 8, 2, 3, 1000, 128, True, 0),
    (1, 4, 4, 20, 20, 64, True, 0),
    (1, 2, 1, 5, 777, 64, False, 50),
    (1, 2, 2, 64, 4096, 128, True, 300),
    (1, 4, 1, 2, 700, 256, True, 0),
]


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,causal,window", FP8_CASES)
def test_decode_fp8kv_kernel_emulated(emu_binary, B, H, H_kv, N_q, N_k, d, causal, window):
    """The FP8 K/V path (E4M3 codes, per-tensor scales) against the oracle on the dequantised cache."""
    wl = Workload("decode_fp8_emu", B, H, N_k, d, causal, window, seed=81 + N_k + N_q, H_kv=H_kv, Nq=N_q)
    _run(emu_binary, wl, fp8=True)


def test_decode_kernel_emulated_strided(emu_binary):
    wl = Workload("decode_emu_strided", 2, 4, 500, 128, True, 0, seed=72, H_kv=2, Nq=3)
    _run(emu_binary, wl, seq_major=True)


@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,causal,window", [
    (2, 8, 2, 3, 1000, 128, True, 0), (1, 2, 1, 5, 777, 64, False, 50), (1, 4, 1, 2, 700, 256, True, 0)])
def test_decode_kernel_emulated_eager_copies(emu_binary_eager, B, H, H_kv, N_q, N_k, d, causal, window):
    """TMA copies that land as soon as they are issued: a load refilling a ring stage that a
    lane of the warp still reads would overwrite those keys."""
    wl = Workload("decode_emu", B, H, N_k, d, causal, window, seed=71 + N_k + N_q, H_kv=H_kv, Nq=N_q)
    _run(emu_binary_eager, wl)


def test_decode_fp8kv_kernel_emulated_eager_copies(emu_binary_eager):
    """The FP8 K/V path (raw E4M3 ring, converted tiles) with TMA copies landing at issue."""
    wl = Workload("decode_fp8_emu", 2, 8, 1000, 128, True, 0, seed=81 + 1000 + 3, H_kv=2, Nq=3)
    _run(emu_binary_eager, wl, fp8=True)

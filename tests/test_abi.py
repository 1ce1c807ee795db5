"""The C-ABI library: it builds, loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (no GPU needed for any of this)."""

import ctypes

import pytest

from exact_io_aware_77_b200 import _lib
from exact_io_aware_77_b200.build import build


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def test_exports_every_header_symbol(lib):
    names = _lib.header_symbols()
    assert "fa_fwd" in names and "fa_check_status" in names
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings(lib):
    for code in _lib.STATUS_NAMES:
        s = _lib.status_string(code)
        assert s and s != "unknown status"
    assert _lib.status_string(999) == "unknown status"


A = 0x10000   # fake, 16-byte-aligned addresses: validation must fail before any use
GOOD = dict(B=1, H=2, N=128, d=64, scale=0.125, causal=0, window=0)


def _fwd(**kw):
    a = dict(GOOD)
    ptrs = kw.pop("ptrs", [A, A + 4096, A + 8192, A + 12288, A + 16384])
    a.update(kw)
    return _lib.fa_fwd(*ptrs, a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"], a["window"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[0, A, A, A, A]), "FA_ERR_NULL"),
    (dict(ptrs=[A, A, A, A, 0]), "FA_ERR_NULL"),
    (dict(B=0), "FA_ERR_SHAPE"),
    (dict(H=-1), "FA_ERR_SHAPE"),
    (dict(N=0), "FA_ERR_SHAPE"),
    (dict(B=1 << 20, H=1 << 20), "FA_ERR_SHAPE"),
    (dict(d=96), "FA_ERR_HEADDIM"),
    (dict(d=512), "FA_ERR_HEADDIM"),
    (dict(window=-1, causal=1), "FA_ERR_MASK"),
    (dict(causal=2), "FA_ERR_MASK"),
    (dict(scale=0.0), "FA_ERR_SCALE"),
    (dict(scale=-1.0), "FA_ERR_SCALE"),
    (dict(scale=float("inf")), "FA_ERR_SCALE"),
    (dict(scale=float("nan")), "FA_ERR_SCALE"),
    (dict(ptrs=[A + 8, A, A, A, A]), "FA_ERR_ALIGN"),
    (dict(ptrs=[A, A, A, A + 2, A]), "FA_ERR_ALIGN"),
    (dict(ptrs=[A, A, A, A, A + 2]), "FA_ERR_ALIGN"),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert _lib.STATUS_NAMES[_fwd(**kw)] == code


def _bwd(ws_bytes=1 << 30, **kw):
    a = dict(GOOD)
    ptrs = kw.pop("ptrs", [A + 4096 * i for i in range(9)])
    ws = kw.pop("ws", A + 65536)
    a.update(kw)
    return _lib.fa_bwd(*ptrs, a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"], a["window"],
                       ws, ws_bytes, None)


def test_workspace_size_formula(lib):
    for B, H, N, d in ((1, 1, 1, 64), (2, 32, 4096, 128), (1, 16, 32768, 128), (3, 5, 65, 64)):
        np_ = (N + 127) // 128 * 128
        assert _lib.fa_bwd_workspace_size(B, H, N, d) == 4 * B * H * np_ * (d + 2)
    assert _lib.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    assert _lib.fa_bwd_workspace_size(1, 1, 16, 80) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[A] * 8 + [0]), "FA_ERR_NULL"),
    (dict(ptrs=[0] + [A] * 8), "FA_ERR_NULL"),
    (dict(N=0), "FA_ERR_SHAPE"),
    (dict(d=32), "FA_ERR_HEADDIM"),
    (dict(window=-3), "FA_ERR_MASK"),
    (dict(scale=0.0), "FA_ERR_SCALE"),
    (dict(ws=0), "FA_ERR_WORKSPACE"),
    (dict(ws_bytes=100), "FA_ERR_WORKSPACE"),
    (dict(ws=A + 8), "FA_ERR_ALIGN"),
    (dict(ptrs=[A] * 5 + [A + 2] + [A] * 3), "FA_ERR_ALIGN"),
])
def test_bwd_rejects_bad_arguments(lib, kw, code):
    assert _lib.STATUS_NAMES[_bwd(**kw)] == code


@pytest.mark.parametrize("phases", [0, 8, -1])
def test_bwd_phases_rejects_bad_mask(lib, phases):
    ptrs = [A + 4096 * i for i in range(9)]
    st = _lib.fa_bwd_phases(*ptrs, 1, 2, 128, 64, 0.125, 0, 0, A + 65536, 1 << 30, phases, None)
    assert _lib.STATUS_NAMES[st] == "FA_ERR_PHASES"


@pytest.mark.parametrize("H,H_kv", [(4, 0), (4, 3), (4, 8), (6, -2)])
def test_shared_kv_head_counts_rejected(lib, H, H_kv):
    """H must be a whole multiple of H_kv >= 1, in the forward and the backward."""
    a = dict(GOOD, H=H)
    ptrs = [A + 4096 * i for i in range(9)]
    st = _lib.fa_fwd_gqa(*ptrs[:5], a["B"], H, H_kv, a["N"], a["d"], a["scale"], a["causal"], a["window"], None)
    assert _lib.STATUS_NAMES[st] == "FA_ERR_SHAPE"
    st = _lib.fa_bwd_gqa(*ptrs, a["B"], H, H_kv, a["N"], a["d"], a["scale"], a["causal"], a["window"],
                         A + 65536, 1 << 30, 7, None)
    assert _lib.STATUS_NAMES[st] == "FA_ERR_SHAPE"


def test_strided_entry_points_validate_strides(lib):
    """Strides must be positive multiples of 8 elements; the backward needs its strides."""
    good = [_lib.FaStrides(2 * 128 * 64, 128 * 64, 64) for _ in range(8)]
    ptrs = [A + 4096 * i for i in range(9)]
    a = dict(GOOD)
    for bad in (_lib.FaStrides(2 * 128 * 64, 128 * 64, 60), _lib.FaStrides(0, 128 * 64, 64),
                _lib.FaStrides(-64, 128 * 64, 64)):
        arr = (_lib.FaStrides * 8)(*good)
        arr[1] = bad
        st = _lib.fa_fwd_strided(*ptrs[:5], a["B"], a["H"], a["H"], a["N"], a["d"], ctypes.addressof(arr),
                                 a["scale"], a["causal"], a["window"], None)
        assert _lib.STATUS_NAMES[st] == "FA_ERR_ALIGN"
        st = _lib.fa_bwd_strided(*ptrs, a["B"], a["H"], a["H"], a["N"], a["d"], ctypes.addressof(arr), a["scale"],
                                 a["causal"], a["window"], A + 65536, 1 << 30, 7, None)
        assert _lib.STATUS_NAMES[st] == "FA_ERR_ALIGN"
    st = _lib.fa_bwd_strided(*ptrs, a["B"], a["H"], a["H"], a["N"], a["d"], None, a["scale"], a["causal"],
                             a["window"], A + 65536, 1 << 30, 7, None)
    assert _lib.STATUS_NAMES[st] == "FA_ERR_NULL"


def _dec(ws_bytes=1 << 30, **kw):
    a = dict(B=1, H=8, H_kv=2, N_q=1, N_k=4096, d=128, scale=0.125, causal=1, window=0)
    ptrs = kw.pop("ptrs", [A + 4096 * i for i in range(5)])
    ws = kw.pop("ws", A + 65536)
    st = kw.pop("strides", None)
    a.update(kw)
    return _lib.fa_fwd_decode(*ptrs, a["B"], a["H"], a["H_kv"], a["N_q"], a["N_k"], a["d"], st, a["scale"],
                              a["causal"], a["window"], ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[0] + [A] * 4), "FA_ERR_NULL"),
    (dict(ptrs=[A] * 4 + [0]), "FA_ERR_NULL"),
    (dict(N_q=0), "FA_ERR_SHAPE"),
    (dict(N_q=4097), "FA_ERR_SHAPE"),
    (dict(H_kv=3), "FA_ERR_SHAPE"),
    (dict(B=0), "FA_ERR_SHAPE"),
    (dict(d=96), "FA_ERR_HEADDIM"),
    (dict(window=-1), "FA_ERR_MASK"),
    (dict(causal=2), "FA_ERR_MASK"),
    (dict(scale=0.0), "FA_ERR_SCALE"),
    (dict(ws=0), "FA_ERR_WORKSPACE"),
    (dict(ws_bytes=100), "FA_ERR_WORKSPACE"),
    (dict(ws=A + 8), "FA_ERR_ALIGN"),
    (dict(ptrs=[A + 8] + [A] * 4), "FA_ERR_ALIGN"),
    (dict(ptrs=[A] * 4 + [A + 2]), "FA_ERR_ALIGN"),
])
def test_decode_rejects_bad_arguments(lib, kw, code):
    assert _lib.STATUS_NAMES[_dec(**kw)] == code


def test_decode_rejects_bad_strides(lib):
    arr = (_lib.FaStrides * 4)(*[_lib.FaStrides(8 * 4096 * 128, 4096 * 128, 128) for _ in range(4)])
    arr[2] = _lib.FaStrides(8 * 4096 * 128, 4096 * 128, 100)
    assert _lib.STATUS_NAMES[_dec(strides=ctypes.addressof(arr))] == "FA_ERR_ALIGN"


def test_decode_workspace_size(lib):
    """0 for an invalid problem and for keys that fit one split; otherwise whole splits of
    B*H*N_q rows of (d + 1) fp32 values each, at most 512 of them."""
    size = _lib.fa_decode_workspace_size
    assert size(1, 8, 3, 1, 100, 128, 1, 0) == 0          # H not a multiple of H_kv
    assert size(1, 8, 2, 5, 4, 128, 1, 0) == 0            # N_q > N_k
    assert size(1, 8, 2, 1, 200, 128, 1, 0) == 0          # 13 key steps: one split
    for B, H, H_kv, N_q, N_k, d, causal, window in ((8, 64, 8, 1, 32768, 128, 1, 0), (2, 16, 2, 1, 3000, 128, 1, 0),
                                                    (1, 8, 1, 4, 2049, 64, 0, 0), (1, 4, 4, 2, 1 << 20, 64, 0, 0)):
        n = size(B, H, H_kv, N_q, N_k, d, causal, window)
        per_split = B * H * N_q * (d + 1) * 4
        assert n > 0 and n % per_split == 0 and 2 <= n // per_split <= 512, (n, per_split)
    # head dimension 256 is a decode shape too (one resident CTA per SM: fewer slots, same rule)
    n = size(8, 64, 8, 1, 32768, 256, 1, 0)
    assert n > 0 and n % (8 * 64 * 257 * 4) == 0
    # a causal window leaves only the last keys to visit: the same as the keys alone
    assert size(1, 8, 2, 1, 32768, 128, 1, 1000) == size(1, 8, 2, 1, 1000, 128, 1, 0)


def _dec8(ws_bytes=1 << 30, **kw):
    a = dict(B=1, H=8, H_kv=2, N_q=1, N_k=4096, d=128, scale=0.125, causal=1, window=0, k_scale=0.01, v_scale=0.02)
    ptrs = kw.pop("ptrs", [A + 4096 * i for i in range(5)])
    ws = kw.pop("ws", A + 65536)
    st = kw.pop("strides", None)
    a.update(kw)
    return _lib.fa_fwd_decode_fp8kv(ptrs[0], ptrs[1], ptrs[2], a["k_scale"], a["v_scale"], ptrs[3], ptrs[4], a["B"],
                                    a["H"], a["H_kv"], a["N_q"], a["N_k"], a["d"], st, a["scale"], a["causal"],
                                    a["window"], ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[A, 0, A, A, A]), "FA_ERR_NULL"),
    (dict(N_q=4097), "FA_ERR_SHAPE"),
    (dict(H_kv=3), "FA_ERR_SHAPE"),
    (dict(d=96), "FA_ERR_HEADDIM"),
    (dict(d=512), "FA_ERR_HEADDIM"),
    (dict(window=-2), "FA_ERR_MASK"),
    (dict(k_scale=0.0), "FA_ERR_SCALE"),
    (dict(v_scale=-1.0), "FA_ERR_SCALE"),
    (dict(k_scale=float("inf")), "FA_ERR_SCALE"),
    (dict(v_scale=float("nan")), "FA_ERR_SCALE"),
    (dict(ws=0), "FA_ERR_WORKSPACE"),
    (dict(ptrs=[A, A + 8, A, A, A]), "FA_ERR_ALIGN"),
    (dict(ptrs=[A, A, A + 1, A, A]), "FA_ERR_ALIGN"),
])
def test_decode_fp8kv_rejects_bad_arguments(lib, kw, code):
    assert _lib.STATUS_NAMES[_dec8(**kw)] == code


def test_decode_fp8kv_code_strides_are_16_byte_multiples(lib):
    """The E4M3 arrays are read in 16-byte pieces: a stride of 8 codes is refused, 16 is not."""
    good = [_lib.FaStrides(8 * 4096 * 128, 4096 * 128, 128) for _ in range(4)]
    arr = (_lib.FaStrides * 4)(*good)
    arr[1] = _lib.FaStrides(2 * 4096 * 136, 4096 * 136, 136)      # K rows padded by 8 codes
    assert _lib.STATUS_NAMES[_dec8(strides=ctypes.addressof(arr))] == "FA_ERR_ALIGN"


def test_head_dim_256_workspace(lib):
    """d = 256 has a backward too (bwd256_kernel.cuh): the same workspace formula."""
    for B, H, N in ((1, 2, 128), (2, 4, 300)):
        np_ = (N + 127) // 128 * 128
        assert _lib.fa_bwd_workspace_size(B, H, N, 256) == 4 * B * H * np_ * (256 + 2)


def _f8(**kw):
    a = dict(B=1, H=2, H_kv=2, N=256, d=128, scale=0.125, causal=1, window=0, qs=0.01, ks=0.01, vs=0.01)
    ptrs = kw.pop("ptrs", [A + 4096 * i for i in range(5)])
    a.update(kw)
    return _lib.fa_fwd_fp8(ptrs[0], ptrs[1], ptrs[2], a["qs"], a["ks"], a["vs"], ptrs[3], ptrs[4], a["B"], a["H"],
                           a["H_kv"], a["N"], a["d"], a["scale"], a["causal"], a["window"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs=[0] + [A] * 4), "FA_ERR_NULL"),
    (dict(d=64), "FA_ERR_HEADDIM"),
    (dict(d=256), "FA_ERR_HEADDIM"),
    (dict(N=250), "FA_ERR_SHAPE"),
    (dict(H_kv=3), "FA_ERR_SHAPE"),
    (dict(qs=0.0), "FA_ERR_SCALE"),
    (dict(ks=float("inf")), "FA_ERR_SCALE"),
    (dict(vs=-1.0), "FA_ERR_SCALE"),
    (dict(window=-1), "FA_ERR_MASK"),
    (dict(ptrs=[A, A + 8, A, A, A]), "FA_ERR_ALIGN"),
])
def test_fwd_fp8_rejects_bad_arguments(lib, kw, code):
    assert _lib.STATUS_NAMES[_f8(**kw)] == code

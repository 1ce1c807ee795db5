"""bench.py's FLOP counts: the closed-form pair counts of banded masks agree with the oracle's
brute-force count, and the unbanded convention is 4 B H N^2 d, halved when causal."""

import pytest

import bench
from oracle import attention as orc


@pytest.mark.parametrize("n", [1, 7, 128, 300])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("window", [1, 3, 64, 500])
def test_band_pairs_match_oracle(n, causal, window):
    assert bench.band_pairs(n, causal, window) == orc.allowed_pairs(n, causal, window)


def test_flop_conventions():
    assert bench.fwd_flops(2, 32, 4096, 128, True) == 4.0 * 2 * 32 * 4096 ** 2 * 128 / 2
    assert bench.fwd_flops(4, 16, 2048, 64, False) == 4.0 * 4 * 16 * 2048 ** 2 * 64
    assert bench.bwd_flops(2, 32, 4096, 128, True) == 2.5 * bench.fwd_flops(2, 32, 4096, 128, True)
    # the long-context shape: 4 d per kept pair, not the causal-halved square
    pairs = orc.allowed_pairs(32768, True, 4096)
    assert bench.fwd_flops(1, 16, 32768, 128, True, 4096) == 4.0 * 16 * 128 * pairs


@pytest.mark.parametrize("n_q,n_k", [(1, 1), (1, 300), (3, 40), (17, 17), (5, 777)])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 1), (True, 30), (False, 4), (False, 100)])
def test_decode_pairs_match_oracle_mask(n_q, n_k, causal, window):
    """Decode rows stand at the last n_q key positions: the kept pairs are the oracle mask's."""
    assert bench.decode_pairs(n_q, n_k, causal, window) == int(
        orc.allowed_mask(n_q, n_k, causal, window, n_k - n_q).sum())


def test_decode_bytes():
    # the decode workload: one row per query head, every cached key read once
    b = bench.decode_bytes(8, 64, 8, 1, 32768, 128, True)
    assert b == 2 * 8 * 64 * 128 * 2 + 2 * 8 * 8 * 32768 * 128 * 2 + 8 * 64 * 4
    # an E4M3 cache halves the K and V bytes
    assert bench.decode_bytes(8, 64, 8, 1, 32768, 128, True, kv_elem_bytes=1) == \
        2 * 8 * 64 * 128 * 2 + 2 * 8 * 8 * 32768 * 128 + 8 * 64 * 4
    # a causal window reads only the keys the window keeps
    assert bench.decode_bytes(1, 1, 1, 1, 10000, 64, True, 100) == 2 * 64 * 2 + 2 * 100 * 64 * 2 + 4


def _roof(achieved):
    return {"bound": "tensor", "kernel": "k", "achieved": achieved, "peak": 1636.3, "unit": "TFLOP/s",
            "frac": round(achieved / 1636.3, 4), "peak_source": "measured burst bf16 (MEASURED_PEAKS.json)"}


def test_regime_fields_burst_and_sustained():
    """A timed region under 1 s is compared with the burst peak, a longer one with the
    sustained peak; both fractions and the clock-normalised kernel time are reported."""
    peaks = {"bf16_tflops": 1636.3, "bf16_tflops_sustained": 1375.0}
    clocks = {"sm_mhz": 1732.0, "sm_max_mhz": 1965.0, "samples": 13}
    r = _roof(900.0)
    cn = bench.regime_fields(r, clocks, 23.0, 0.3, peaks)
    assert r["regime"] == "burst" and r["peak"] == 1636.3 and r["frac"] == round(900.0 / 1636.3, 4)
    assert r["frac_of_sustained_peak"] == round(900.0 / 1375.0, 4)
    assert cn["kernel_ms_at_max_clock"] == round(0.3 * 1732.0 / 1965.0, 5)
    assert cn["achieved_at_max_clock"] == round(900.0 * 1965.0 / 1732.0, 1)
    assert cn["samples_in_window"] == 13
    r = _roof(900.0)
    bench.regime_fields(r, clocks, 1230.0, 0.3, peaks)
    assert r["regime"] == "sustained" and r["peak"] == 1375.0 and r["frac"] == round(900.0 / 1375.0, 4)
    assert "sustained" in r["peak_source"]
    # no clock samples: no clock-normalised figures, the regime still set
    r = _roof(900.0)
    assert bench.regime_fields(r, {"sm_mhz": None, "sm_max_mhz": None}, 10.0, 0.3, peaks) is None
    assert r["regime"] == "burst"

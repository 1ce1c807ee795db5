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

"""The persistent kernels' work-item schedules, compiled from fwd_persist_kernel.cuh and
bwd_persist_kernel.cuh and run on the host (tests/host_emu/emu_sched_main.cpp): every forward item
(head, query-tile pair) and every backward item (K/V head, key tile) goes to exactly one CTA for
every shape, grid size and item order tried, with the tile ranges of kv_tile_range / q_tile_range;
and on the causal and banded workloads the balanced order brings the largest CTA load within a
few percent of the mean.  CPU only."""

import subprocess

import pytest


@pytest.fixture(scope="module")
def sched_rows(tmp_path_factory):
    from tests.host_emu.build_emu import build
    d = str(tmp_path_factory.mktemp("host_emu_sched"))
    try:
        exe = build(d, ["fwd_persist_kernel.cuh", "fwd_kernel.cuh", "persist_sched.cuh", "bwd_persist_kernel.cuh",
                        "bwd_kernel.cuh", "fwd256_persist_kernel.cuh", "fwd256_kernel.cuh"], "emu_sched_main.cpp",
                    "emu_sched")
    except FileNotFoundError:
        pytest.skip("g++ not available")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [l for l in r.stdout.split("\n") if l.strip()]
    fwd = [l for l in lines if not l.startswith(("bwd", "f256", "grid"))]
    grid = [l for l in lines if l.startswith("grid")]
    assert len(grid) == 11
    bwd = [l for l in lines if l.startswith("bwd")]
    f256 = [l for l in lines if l.startswith("f256")]
    assert len(f256) == 14 * 2 * 8
    assert len(fwd) == 14 * 2 * 8   # shapes x item orders x grid sizes, one line each
    assert len(bwd) >= 14 * 2 * 8   # and per query heads per K/V head that divide the heads
    rows = {}
    for line in fwd:
        BH, N, causal, window, order, g, max_load, mean = line.split()
        rows[(int(BH), int(N), int(causal), int(window), int(order), int(g))] = (int(max_load), float(mean))
    for line in f256:
        _, BH, N, causal, window, order, g, max_load, mean = line.split()
        rows[("f256", int(BH), int(N), int(causal), int(window), int(order), int(g))] = (int(max_load), float(mean))
    for line in bwd:
        _, BH, group, N, causal, window, order, g, max_load, mean = line.split()
        rows[("bwd", int(BH), int(group), int(N), int(causal), int(window), int(order), int(g))] = (int(max_load),
                                                                                                   float(mean))
    for line in grid:
        _, heads, n_pos, chunk, mk_chunked, mk_head, mean = line.split()
        rows[("grid", int(heads), int(n_pos), int(chunk))] = (int(mk_chunked), int(mk_head), float(mean))
    return rows


def test_every_item_once(sched_rows):
    """The harness exits non-zero on any item taken twice or never, and prints a line per case."""
    assert (64, 4096, 1, 0, 1, 148) in sched_rows and (1, 1, 1, 0, 0, 1) in sched_rows


@pytest.mark.parametrize("shape", [(64, 4096, 1, 0), (16, 32768, 1, 4096), (16, 32768, 0, 4096)])
def test_balanced_order_evens_the_loads(sched_rows, shape):
    """148 CTAs: causal B2 H32 N4096, and N 32768 with a one- and a two-sided window of 4096."""
    head_max, mean = sched_rows[shape + (0, 148)]
    pair_max, mean2 = sched_rows[shape + (1, 148)]
    assert mean == mean2
    assert pair_max <= 1.03 * mean, (pair_max, mean)
    assert pair_max < head_max


@pytest.mark.parametrize("group,slack", [(1, 1.03), (4, 1.06)])
def test_backward_balanced_order(sched_rows, group, slack):
    """Causal B2 H32 N4096 (64 query heads), with 1 or 4 query heads per K/V head, 148 CTAs: the
    balanced (key-tile-major) order's largest load is within 3 % of the mean, or 6 % with 4 query
    heads per K/V head, whose 512 items (up to 129 load units each) are too coarse for less."""
    head_max, mean = sched_rows[("bwd", 64, group, 4096, 1, 0, 0, 148)]
    bal_max, _ = sched_rows[("bwd", 64, group, 4096, 1, 0, 1, 148)]
    assert bal_max <= slack * mean, (bal_max, mean)
    assert bal_max <= head_max


def test_d256_forward_balanced_order(sched_rows):
    """The d = 256 forward's items (one query tile each) at 148 CTAs on a causal N4096 shape with
    64 heads: the balanced order's largest load is within 3 % of the mean."""
    head_max, mean = sched_rows[("f256", 64, 4096, 1, 0, 0, 148)]
    bal_max, _ = sched_rows[("f256", 64, 4096, 1, 0, 1, 148)]
    assert bal_max <= 1.03 * mean, (bal_max, mean)
    assert bal_max <= head_max


def test_chunked_grid_order_shortens_the_causal_makespan(sched_rows):
    """grid_item (the one-item-per-CTA kernels' order): on the causal B2 H32 N4096 forward (64 heads
    of 16 query-tile pairs) the chunked order's makespan on 148 SMs is within 5 % of the mean load,
    where the head-major order leaves a tail of over 10 %."""
    chunked, head_major, mean = sched_rows[("grid", 64, 16, 16)]
    assert chunked <= 1.05 * mean, (chunked, mean)
    assert head_major >= 1.10 * mean, (head_major, mean)
    # the backward's key tiles in chunks of 8 K/V heads (grid_item covers every item: the harness)
    assert ("grid", 64, 32, 8) in sched_rows

"""The algorithmic work behind the bench line's roofline (CPU only).

Entry (i, j) of the rounding feeds every later entry of its row (one FMA per entry
to its right, through R-hat) and of its column (one FMA per entry below, through
L-hat): 2 (n - 1 - j) + 2 (m - 1 - i) flops, mn(m + n - 2) in all.  bench.py splits
that between the kernels by tile distance: the far-field kernel takes the targets
two or more 64-tiles away, the sweep kernel the rest (its own tile and the near
pulls from the neighbouring tile).  The roofline's "achieved" figure divides the
far-field share by the kernel's time, so the split is pinned here by brute force.
"""
import numpy as np
import pytest

import bench

TB = 64


def _brute(m, n):
    """(far, sweep) flops by classifying every (source, target) pair by tile distance."""
    far = sweep = 0
    for i in range(m):
        for j in range(n):
            J, I = j // TB, i // TB
            right = np.arange(j + 1, n) // TB - J      # tile distance of each target
            down = np.arange(i + 1, m) // TB - I
            far += 2 * (int(np.sum(right >= 2)) + int(np.sum(down >= 2)))
            sweep += 2 * (int(np.sum(right < 2)) + int(np.sum(down < 2)))
    return far, sweep


@pytest.mark.parametrize("m,n", [(1, 1), (64, 64), (65, 1), (130, 70), (200, 257), (3, 193)])
def test_far_and_sweep_shares_by_brute_force(m, n):
    far, sweep = _brute(m, n)
    assert bench.far_flops(m, n) == far
    assert bench.sweep_flops(m, n) == sweep


@pytest.mark.parametrize("m,n", [(4096, 4096), (4096, 14336), (8192, 28672), (1024, 8192),
                                 (1000, 3001)])
def test_shares_add_up_to_the_whole_rounding(m, n):
    assert bench.far_flops(m, n) + bench.sweep_flops(m, n) == m * n * (m + n - 2)


def test_the_headline_far_share():
    """The per-launch figure quoted for the 4096 x 4096 layer (173 far-field launches)."""
    assert bench.far_flops(4096, 4096) / 173 == pytest.approx(7.5759e8, rel=1e-4)

"""Parity helpers shared by the GPU tests: the near-tie replay checker.

The oracle defines the admissible outputs: the unique GPTQ-2D trajectory,
except that at an entry whose y/s lies within 1e-6 of a rounding boundary
(a near-tie) either neighbouring integer is admissible, and the trajectory
continues from the choice made.  `check_against_oracle` walks the candidate's
mismatches in anti-diagonal order and, at each, asks the oracle to take the
other neighbour there; the oracle itself refuses unless that entry is a
near-tie of its own (replayed) trajectory.  A mismatch that is not a near-tie
fails.  Only the choice between the oracle's own alternatives is read from
the candidate.
"""
import numpy as np

import oracle as O


class ParityReport:
    def __init__(self, result, flips, n_near_tie):
        self.result = result
        self.flips = flips
        self.n_near_tie = n_near_tie


def check_against_oracle(W, M_L, M_R, s, bits, clamp, Q_candidate, max_flips=64, grid=None):
    """``Q_candidate``: the candidate's integers q (for a grid variant, codes already
    converted back to q); ``grid``: the per-entry grid (oracle.expand_grid), if any."""
    Qc = np.asarray(Q_candidate, np.float64)
    flips = set()
    for _ in range(max_flips + 1):
        r = O.gptq2d_antidiagonal(W, M_L, M_R, s, bits, clamp, flip=flips, grid=grid)
        mism = np.argwhere(r.Q != Qc)
        if mism.size == 0:
            return ParityReport(r, flips, int(r.near_tie.sum()))
        d = mism.sum(axis=1)
        first = mism[d == d.min()]
        for i, j in first:
            assert r.near_tie[i, j], (
                f"Q differs at ({i},{j}) on anti-diagonal {i + j}: candidate {Qc[i, j]}, "
                f"oracle {r.Q[i, j]}, oracle y/s {r.T[i, j]!r} is not a near-tie")
            flips.add((int(i), int(j)))
    raise AssertionError(f"more than {max_flips} near-tie flips")

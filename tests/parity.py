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


class FixedPointReport:
    def __init__(self, n_entries, n_near_tie, n_other_neighbour):
        self.n_entries = n_entries
        self.n_near_tie = n_near_tie              # entries within the band of a boundary
        self.n_other_neighbour = n_other_neighbour  # near-ties where the candidate took the other side


def check_fixed_point(W, M_L, M_R, s, bits, clamp, Q_candidate, row_chunk=1024):
    """Every entry of a candidate output against the oracle's definition of y.

    y_ij is computed from the candidate's own integers (oracle.entry_values_all), so
    the check costs two matrix products however large the output.  Every entry that
    is not a near-tie must equal clamp(rint(y / s)); at a near-tie the candidate may
    take either neighbouring integer.  Since y_ij depends only on entries before
    (i, j) in the product order, this holds at every entry exactly when the candidate
    is the oracle's trajectory up to the near-tie choices.  Rows are processed in
    chunks of ``row_chunk`` to bound host memory."""
    W = np.asarray(W, np.float64)
    Qc = np.asarray(Q_candidate, np.float64)
    s = np.asarray(s, np.float64)
    m, n = W.shape
    lo, hi = O.grid_bounds(bits, clamp)
    n_tie = n_other = 0
    for r0 in range(0, m, row_chunk):
        r1 = min(m, r0 + row_chunk)
        T = O.entry_values_all(W, Qc, s, M_L, M_R, rows=(r0, r1)) / s[r0:r1, None]
        Qr = Qc[r0:r1]
        nt = O.near_tie(T, lo, hi)
        bad = (O.round_to_grid(T, lo, hi) != Qr) & ~nt
        if bad.any():
            idx = np.argwhere(bad)[:8]
            raise AssertionError(
                f"{int(bad.sum())} entries are not the rounding of their own y/s; first: " +
                ", ".join(f"({r0 + i},{j}): q={Qr[i, j]:g} t={T[i, j]!r}" for i, j in idx))
        # at a near-tie, the candidate's integer must be one of the two neighbours
        h = np.floor(T[nt]) + 0.5
        assert np.all((Qr[nt] == h - 0.5) | (Qr[nt] == h + 0.5))
        n_tie += int(nt.sum())
        n_other += int(np.count_nonzero(nt & (O.round_to_grid(T, lo, hi) != Qr)))
    return FixedPointReport(m * n, n_tie, n_other)

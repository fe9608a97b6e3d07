"""fp64 CPU oracle for GPTQ-2D two-sided adaptive rounding.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library (no kernels, headers, helpers, tables or pre/post-processing),
and the library never imports it.

What it computes (sources are the two on-topic pages):
  * mind-verse.de "Neue Ansätze ... durch GPTQ-2D", sections "GPTQ-2D: Eine
    Weiterentwicklung der adaptiven Rundung" (two-sided problem with bases on
    both sides of the residual) and "Geometrische Grundlagen und der Bezug zu
    Babai's Nearest Plane Algorithmus" (vectorisation turns the two-sided
    problem into a quadratic form whose Gram matrix is a Kronecker product;
    GPTQ is Babai's nearest-plane algorithm on it).
  * arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Abstract
    (same rounding as the quartic Kronecker feedback, cubic work, entries of
    one anti-diagonal rounded in parallel) and Analysis > Results / Methodology
    (exact 1-D GPTQ trajectory; rank-one separable feedback kept in a buffer).

Conventions (readings where the pages are silent):
  * W is m x n.  H_L (m x m) acts on the row index i, H_R (n x n) on the column
    index j.  Proxy loss  L(Q) = tr(dW^T H_L dW H_R),  dW = W - diag(s) Q, which
    is vec(dW)^T (H_R kron H_L) vec(dW) with column-major vec.
  * Entry (0, 0) is rounded first (GPTQ's index-0-first order).
  * Grid: q = clamp(rint(t), lo, hi) with rint = round half to even; without
    clamp the grid is all integers.  The error fed back is W - s q with the
    clamped q.
  * Per-row scales s_i are inputs (grid = s_i * Z on row i).

Functions, from most literal to fastest:
  O0  nearest_plane_by_definition   conditional minimiser, any linear extension
  O1  babai_kron_sweep              1-D GPTQ sweep over vec(W) on the mn x mn Gram
  O2  gptq2d_antidiagonal           the cubic anti-diagonal algorithm
and the special cases used as pins: RTN, 1-D GPTQ in OBS form, exhaustive
closest-vector search on tiny problems.  For checking large candidate outputs
entry by entry: entry_value (one entry) and entry_values_all (every entry, from
the candidate's own integers, by two matrix products).

Grid variants (the pages fix only a 4-bit integer grid; these are GPTQ's usual
ones): expand_grid turns group-wise scales and integer zero points into a
per-entry step and admissible range that O0, O1 and O2 take as ``grid``;
stored_codes / packed_codes / pack_nibbles give the bytes of the outputs.

The step before the path: gram / gram_batches form a Kronecker factor
H = X^T X / N (+ damping) from N rows of activations.

Hessians with k > 2 Kronecker factors (arxivlens, Abstract), W a k-way tensor:
  O1k babai_tensor_sweep            1-D GPTQ over the C-order flattening, explicit Gram
  O2k gptq_kron_hyperplane          hyperplane order, per-mode factors applied separately
      gptq_kron_via_2d              the same problem as a 2-D one with H_R = H_2 kron ... kron H_k
"""
from __future__ import annotations

import itertools
import numpy as np

NEAR_TIE_BAND = 1e-6


# --------------------------------------------------------------------------- #
# Grid and loss
# --------------------------------------------------------------------------- #
def grid_bounds(bits: int, clamp: bool):
    """Admissible integers: [-2^(bits-1), 2^(bits-1)-1] when clamping, else all of Z."""
    if not clamp:
        return -np.inf, np.inf
    return float(-(1 << (bits - 1))), float((1 << (bits - 1)) - 1)


def round_to_grid(t, lo, hi):
    """Nearest admissible integer along one coordinate: clamp(rint(t), lo, hi)."""
    return np.clip(np.rint(t), lo, hi)


def expand_grid(m, n, scales, bits, clamp, group_size=0, zeros=None):
    """Per-entry grid of GPTQ's grid variants: returns (S, LO, HI), each m x n, so
    that entry (i, j) rounds to S[i,j] * q with q an integer in [LO[i,j], HI[i,j]].

      * group_size 0: one scale per row (scales has m entries); else the columns
        form groups of group_size and scales is m x ceil(n / group_size).
      * zeros None: symmetric grid, q in [-2^(bits-1), 2^(bits-1)-1].
      * zeros given (integers, shaped like the scales): asymmetric grid, code
        c = q + z in [0, 2^bits - 1] and value S (c - z); for the integer q this
        is the range [-z, 2^bits - 1 - z].  With an integer z,
        clamp(rint(t + z)) - z = clamp(rint(t), -z, 2^bits - 1 - z), so the
        rounding is the same nearest admissible integer along the coordinate.
      * clamp False: every integer is admissible (zeros only shift the code).
    """
    sc = np.asarray(scales, np.float64).reshape(m, -1)
    col = np.arange(n) // group_size if group_size else np.zeros(n, np.int64)
    S = sc[:, col] if n else np.zeros((m, 0))
    if zeros is None:
        lo, hi = grid_bounds(bits, clamp)
        LO = np.full((m, n), lo)
        HI = np.full((m, n), hi)
    else:
        Z = np.asarray(zeros, np.float64).reshape(m, -1)[:, col] if n else np.zeros((m, 0))
        if clamp:
            LO = -Z
            HI = float((1 << bits) - 1) - Z
        else:
            LO = np.full((m, n), -np.inf)
            HI = np.full((m, n), np.inf)
    return S, LO, HI


def stored_codes(Q, m, n, bits, group_size=0, zeros=None):
    """The byte a caller receives for each entry: q itself on the symmetric grid,
    the unsigned code q + z on the asymmetric one."""
    Q = np.asarray(Q, np.float64)
    if zeros is None:
        return Q
    col = np.arange(n) // group_size if group_size else np.zeros(n, np.int64)
    return Q + np.asarray(zeros, np.float64).reshape(m, -1)[:, col]


def pack_nibbles(codes):
    """Two unsigned 4-bit codes per byte, row by row: byte k of a row holds the
    entry of column 2k in its low nibble and that of column 2k+1 in its high
    nibble (zero past the last column)."""
    c = np.asarray(codes, np.int64)
    m, n = c.shape
    if np.any((c < 0) | (c > 15)):
        raise ValueError("codes must lie in [0, 15]")
    out = np.zeros((m, (n + 1) // 2), np.uint8)
    out[:, :] = c[:, 0::2]
    out[:, : n // 2] |= (c[:, 1::2] << 4).astype(np.uint8)
    return out


def packed_codes(Q, m, n, bits, group_size=0, zeros=None):
    """Unsigned 4-bit code of every entry for packed output: q - lo on the symmetric
    grid (offset binary, lo = -2^(bits-1)), q + z on the asymmetric one."""
    if zeros is None:
        return np.asarray(Q, np.float64) + float(1 << (bits - 1))
    return stored_codes(Q, m, n, bits, group_size, zeros)


def proxy_loss(W, Q, s, H_L, H_R) -> float:
    """L(Q) = tr(dW^T H_L dW H_R), dW = W - S Q (the two-sided quadratic metric), with
    S = diag(s) for per-row scales or the per-entry grid steps (an m x n array)."""
    W = np.asarray(W, np.float64)
    s = np.asarray(s, np.float64)
    D = W - (s if s.ndim == 2 else s[:, None]) * np.asarray(Q, np.float64)
    return float(np.sum(D * (np.asarray(H_L, np.float64) @ D @ np.asarray(H_R, np.float64))))


def rtn(W, s, bits, clamp):
    """Round-to-nearest baseline: each entry independently, q = clamp(rint(W_ij / s_i))."""
    lo, hi = grid_bounds(bits, clamp)
    W = np.asarray(W, np.float64)
    return round_to_grid(W / np.asarray(s, np.float64)[:, None], lo, hi)


def near_tie(t, lo, hi, band=NEAR_TIE_BAND):
    """True where t lies within ``band`` of a rounding boundary k + 1/2 that separates
    two admissible integers (lo <= k < hi).  Values beyond hi + 1/2 or below lo - 1/2
    have no boundary: clamping sends both neighbours to the same integer."""
    t = np.asarray(t, np.float64)
    h = np.floor(t) + 0.5
    has_boundary = (h - 0.5 >= lo) & (h + 0.5 <= hi)
    return has_boundary & (np.abs(t - h) < band)


# --------------------------------------------------------------------------- #
# Factor of a Kronecker factor
# --------------------------------------------------------------------------- #
def reverse_cholesky(H):
    """Lower-triangular M with positive diagonal and M^T M = H.

    With M_L, M_R of this form, M = M_R kron M_L is lower triangular in
    column-major index order and M^T M = H_R kron H_L, so row p of M(x - z)
    involves only coordinates <= p: the triangular factor that makes the
    index-0-first nearest-plane sweep explicit.  Computed through LAPACK's
    ordinary Cholesky of the index-reversed matrix: if J H J = L L^T then
    M = J L^T J.
    """
    H = np.asarray(H, np.float64)
    L = np.linalg.cholesky(H[::-1, ::-1])
    return np.array(L.T[::-1, ::-1], order="C", copy=True)


# --------------------------------------------------------------------------- #
# O0: the definition
# --------------------------------------------------------------------------- #
def nearest_plane_by_definition(W, H_L, H_R, s, bits, clamp, order="row", grid=None):
    """Sequential nearest-plane rounding of vec(W) under G = H_R kron H_L, written
    as its definition (mind-verse.de, "Geometrische Grundlagen ..."): coordinates
    are fixed one at a time; the value rounded for coordinate p is the p-th
    coordinate of the real minimiser of (z - x)^T G (z - x) over the coordinates
    not yet fixed, with the fixed ones held at s*q.

    ``order`` is any linear extension of the product order on (i, j):
    "row" (row-major) or "col" (column-major).  ``grid`` = (S, LO, HI) from
    expand_grid replaces the per-row scales s and the bits/clamp range.
    Returns (Q, T) with T = y / s.  Dense solves of size mn: tiny problems only.
    """
    W = np.asarray(W, np.float64)
    m, n = W.shape
    S, LO, HI = grid if grid is not None else expand_grid(m, n, s, bits, clamp)
    G = np.kron(np.asarray(H_R, np.float64), np.asarray(H_L, np.float64))
    x = W.reshape(-1, order="F")                         # p = i + m j
    sv = S.reshape(-1, order="F")
    lov, hiv = LO.reshape(-1, order="F"), HI.reshape(-1, order="F")
    if order == "row":
        seq = [i + m * j for i in range(m) for j in range(n)]
    elif order == "col":
        seq = list(range(m * n))
    else:
        raise ValueError(order)
    fixed = np.zeros(m * n, bool)
    z = np.zeros(m * n)
    T = np.zeros(m * n)
    Q = np.zeros(m * n)
    for p in seq:
        r = np.flatnonzero(~fixed)
        f = np.flatnonzero(fixed)
        zr = x[r].copy()
        if f.size:
            # stationarity over the free block: G_rr (z_r - x_r) + G_rf (z_f - x_f) = 0
            zr = x[r] - np.linalg.solve(G[np.ix_(r, r)], G[np.ix_(r, f)] @ (z[f] - x[f]))
        y = zr[np.searchsorted(r, p)]
        T[p] = y / sv[p]
        Q[p] = round_to_grid(T[p], lov[p], hiv[p])
        z[p] = sv[p] * Q[p]
        fixed[p] = True
    return Q.reshape((m, n), order="F"), T.reshape((m, n), order="F")


# --------------------------------------------------------------------------- #
# O1: naive vectorised Babai / 1-D GPTQ sweep on the full Kronecker Gram
# --------------------------------------------------------------------------- #
def babai_kron_sweep(W, H_L, H_R, s, bits, clamp, grid=None):
    """The naive vectorised sweep whose trajectory GPTQ-2D reproduces (arxivlens,
    Analysis > Results; mind-verse.de, "Die algorithmische Neuerung"): one-sided
    GPTQ over all mn coordinates of vec(W) (column-major), with the Gram
    G = H_R kron H_L.  GPTQ form: U = upper Cholesky factor of G^{-1}; coordinate
    p is rounded, and its error, divided by U_pp, is propagated to the later
    coordinates along row p of U.  Quartic work; 64 x 64 at most.  ``grid`` =
    (S, LO, HI) from expand_grid replaces per-row scales and the bits/clamp range.
    Returns (Q, T) with T = (updated x_p) / s_p.
    """
    W = np.asarray(W, np.float64)
    m, n = W.shape
    S, LO, HI = grid if grid is not None else expand_grid(m, n, s, bits, clamp)
    G = np.kron(np.asarray(H_R, np.float64), np.asarray(H_L, np.float64))
    U = np.linalg.cholesky(np.linalg.inv(G)).T            # U^T U = G^{-1}, upper
    x = W.reshape(-1, order="F").copy()
    sv = S.reshape(-1, order="F")
    lov, hiv = LO.reshape(-1, order="F"), HI.reshape(-1, order="F")
    N = m * n
    Q = np.zeros(N)
    T = np.zeros(N)
    for p in range(N):
        T[p] = x[p] / sv[p]
        Q[p] = round_to_grid(T[p], lov[p], hiv[p])
        e = (x[p] - sv[p] * Q[p]) / U[p, p]
        x[p + 1:] -= e * U[p, p + 1:]
    return Q.reshape((m, n), order="F"), T.reshape((m, n), order="F")


# --------------------------------------------------------------------------- #
# O2: the cubic anti-diagonal algorithm
# --------------------------------------------------------------------------- #
class Result:
    """Output of gptq2d_antidiagonal: Q, T = y/s, the Babai-identity loss, flags."""

    def __init__(self, Q, T, loss_identity, n_clamped, near_tie_mask, flipped):
        self.Q = Q
        self.T = T
        self.loss_identity = loss_identity
        self.n_clamped = n_clamped
        self.near_tie = near_tie_mask
        self.flipped = flipped


def gptq2d_antidiagonal(W, M_L, M_R, s, bits, clamp, flip=None, band=NEAR_TIE_BAND, grid=None):
    """GPTQ-2D: round W anti-diagonal by anti-diagonal (arxivlens Abstract;
    mind-verse.de "Die algorithmische Neuerung") with the rank-one separable
    feedback kept in an accumulated buffer (arxivlens, Analysis > Results and
    Methodology).

    With M_L, M_R the lower factors (M^T M = H), rounding entry (i, j) sees
        y_ij = W_ij + (sum_{i'<=i, j'<=j, (i',j') != (i,j)} M_L[i,i'] dW[i',j'] M_R[j,j'])
                       / (M_L[i,i] M_R[j,j]),
    i.e. row (i,j) of (M_R kron M_L) applied to the errors already made.  The
    buffer P holds P[i', j] = sum_{j' <= j, done} dW[i', j'] M_R[j, j'] (right
    feedback); the left factor is applied to a column of P when an entry is
    rounded.  Entries of anti-diagonal d = i + j only depend on earlier
    anti-diagonals, so each one is handled as a vector.  Work is mn(m + n).

    ``flip``: optional set of (i, j) where the other neighbouring integer is
    taken.  Every such entry must be a near-tie (|t - (k + 1/2)| < band) in this
    run's own trajectory, else ValueError: the flip set only selects among the
    roundings that the near-tie rule admits.

    ``grid``: optional (S, LO, HI) from expand_grid (group-wise scales, zero
    points): entry (i, j) then rounds to S[i,j] * q, q in [LO[i,j], HI[i,j]], in
    place of the per-row scales s and the bits/clamp range.

    Returns a Result with Q, T = y/s, the loss via the Babai identity
    sum d_ij^2 (y_ij - s_i q_ij)^2, the clamp count and the near-tie mask.
    """
    W = np.asarray(W, np.float64)
    M_L = np.asarray(M_L, np.float64)
    M_R = np.asarray(M_R, np.float64)
    m, n = W.shape
    S, LO, HI = grid if grid is not None else expand_grid(m, n, s, bits, clamp)
    flip = set() if flip is None else set(flip)
    P = np.zeros((m, n))
    Q = np.zeros((m, n))
    T = np.zeros((m, n))
    tie = np.zeros((m, n), bool)
    loss = 0.0
    n_clamped = 0
    done_flips = set()
    for d in range(m + n - 1):
        i = np.arange(max(0, d - n + 1), min(d, m - 1) + 1)
        j = d - i
        # left factor applied to column j of P; M_L[i, i'] = 0 for i' > i drops the rest
        fb = np.einsum("ek,ke->e", M_L[i, :], P[:, j])
        dij = M_L[i, i] * M_R[j, j]
        y = W[i, j] + fb / dij
        sd, lo, hi = S[i, j], LO[i, j], HI[i, j]
        t = y / sd
        q_raw = np.rint(t)
        q = np.clip(q_raw, lo, hi)
        nt = near_tie(t, lo, hi, band)
        if flip:
            for e in range(i.size):
                key = (int(i[e]), int(j[e]))
                if key in flip:
                    if not nt[e]:
                        raise ValueError(f"flip requested at {key}, not a near-tie (t={t[e]!r})")
                    h = np.floor(t[e]) + 0.5
                    q[e] = h + 0.5 if q[e] == h - 0.5 else h - 0.5
                    done_flips.add(key)
        n_clamped += int(np.count_nonzero(q != q_raw))
        delta = W[i, j] - sd * q
        # right feedback: P[i, j'] += delta * M_R[j', j]; zero for j' < j (M_R lower)
        P[i, :] += delta[:, None] * M_R[:, j].T
        loss += float(np.sum((dij * (y - sd * q)) ** 2))
        Q[i, j] = q
        T[i, j] = t
        tie[i, j] = nt
    if done_flips != flip:
        raise ValueError(f"flips never reached: {sorted(flip - done_flips)}")
    return Result(Q, T, loss, n_clamped, tie, done_flips)


def gptq2d(W, H_L, H_R, s, bits, clamp, **kw):
    """Factor both Kronecker factors, then run the anti-diagonal algorithm."""
    return gptq2d_antidiagonal(W, reverse_cholesky(H_L), reverse_cholesky(H_R), s, bits, clamp, **kw)


def entry_value(W, Q, s, M_L, M_R, i, j):
    """y_ij computed directly from its definition, given the integers already chosen
    for the dominated quadrant {i' <= i, j' <= j} minus (i, j) itself.  O(ij) work;
    used to check single sampled entries of large outputs.  s: per-row scales or
    the m x n per-entry grid steps."""
    W = np.asarray(W, np.float64)
    s = np.asarray(s, np.float64)
    S = s[: i + 1, : j + 1] if s.ndim == 2 else s[: i + 1, None]   # per-entry or per-row steps
    D = W[: i + 1, : j + 1] - S * np.asarray(Q[: i + 1, : j + 1], np.float64)
    D[i, j] = 0.0
    fb = np.asarray(M_L[i, : i + 1], np.float64) @ D @ np.asarray(M_R[j, : j + 1], np.float64)
    return W[i, j] + fb / (float(M_L[i, i]) * float(M_R[j, j]))


def entry_values_all(W, Q, s, M_L, M_R, rows=None):
    """y_ij of every entry (of rows r0..r1-1 when ``rows`` = (r0, r1)), each from its
    definition, given a candidate's integers Q everywhere.

    With D = W - S Q and d_ij = M_L[i,i] M_R[j,j], the feedback sum of entry (i, j)
    over its dominated quadrant minus (i, j) itself is (M_L D M_R^T)_ij - d_ij D_ij:
    M_L and M_R are lower triangular, so the product only reaches i' <= i and
    j' <= j (arxivlens, Analysis > Results: row (i, j) of the Kronecker triangular
    factor applied to the errors).  Hence
        y = W + (M_L D M_R^T - d * D) / d
    for all entries at once: two matrix products.  This is entry_value for every
    (i, j); for rows r0..r1-1 only M_L[r0:r1, :r1] and D[:r1] are needed.

    A candidate Q is the trajectory of the sweep (up to the near-tie choices) iff
    every entry satisfies q_ij = clamp(rint(y_ij / s_ij)) with y from Q itself:
    y_ij depends only on entries rounded before (i, j), so the first entry, in any
    linear extension of the product order, that breaks the equality is where Q
    leaves the trajectory.
    """
    W = np.asarray(W, np.float64)
    s = np.asarray(s, np.float64)
    m, n = W.shape
    r0, r1 = (0, m) if rows is None else (int(rows[0]), int(rows[1]))
    S = s if s.ndim == 2 else np.broadcast_to(s[:, None], (m, n))
    D = W[:r1] - S[:r1] * np.asarray(Q[:r1], np.float64)
    ML = np.asarray(M_L, np.float64)
    MR = np.asarray(M_R, np.float64)
    F = (ML[r0:r1, :r1] @ D) @ MR.T
    d = np.diag(ML)[r0:r1, None] * np.diag(MR)[None, :]
    return W[r0:r1] + (F - d * D[r0:r1]) / d


# --------------------------------------------------------------------------- #
# Special cases used as pins
# --------------------------------------------------------------------------- #
def gptq_1d_obs(w, H, s, bits, clamp, bounds=None):
    """Textbook one-sided GPTQ on a vector (mind-verse.de, "GPTQ-2D: Eine
    Weiterentwicklung ...": one-sided rounding with triangular feedback), in the
    optimal-brain-surgeon form rather than the Cholesky form: round coordinate
    p, move the remaining coordinates by -err * Hinv[p, rest] / Hinv[p, p],
    then remove p from the inverse (Hinv -= Hinv[:, p] Hinv[p, :] / Hinv[p, p]).
    Index 0 first.  Returns q."""
    w = np.asarray(w, np.float64).copy()
    s = np.broadcast_to(np.asarray(s, np.float64), w.shape)
    if bounds is None:
        lo, hi = grid_bounds(bits, clamp)
        lo, hi = np.full(w.shape, lo), np.full(w.shape, hi)
    else:
        lo, hi = (np.broadcast_to(np.asarray(b, np.float64), w.shape) for b in bounds)
    Hinv = np.linalg.inv(np.asarray(H, np.float64))
    k = w.size
    q = np.zeros(k)
    for p in range(k):
        q[p] = round_to_grid(w[p] / s[p], lo[p], hi[p])
        err = w[p] - s[p] * q[p]
        w -= err * Hinv[p, :] / Hinv[p, p]
        Hinv = Hinv - np.outer(Hinv[:, p], Hinv[p, :]) / Hinv[p, p]
    return q


def closest_vector_exhaustive(W, H_L, H_R, s, bits, clamp, radius=2, center=None):
    """Exact minimiser of the proxy loss over the integer box center +- radius
    (center defaults to RTN), by evaluating the loss at every point.  Tiny
    problems only (mn <= 9 with radius 2).  Returns (Q, loss)."""
    W = np.asarray(W, np.float64)
    m, n = W.shape
    lo, hi = grid_bounds(bits, clamp)
    c = rtn(W, s, bits, clamp) if center is None else np.asarray(center, np.float64)
    axes = [np.clip(np.arange(c.flat[p] - radius, c.flat[p] + radius + 1), lo, hi)
            for p in range(m * n)]
    axes = [np.unique(a) for a in axes]
    best, bestQ = np.inf, None
    sv = np.asarray(s, np.float64)
    H_L = np.asarray(H_L, np.float64)
    H_R = np.asarray(H_R, np.float64)
    for combo in itertools.product(*axes):
        Qc = np.array(combo).reshape(m, n)
        D = W - sv[:, None] * Qc
        val = float(np.sum(D * (H_L @ D @ H_R)))
        if val < best:
            best, bestQ = val, Qc
    return bestQ, best


def sphere_decode(W, H_L, H_R, s, bits, clamp):
    """Exact closest-vector point by depth-first Schnorr-Euchner enumeration over
    coordinates in column-major order, using M = M_R kron M_L (lower) so that the
    partial sum of squared residual rows is monotone.  The first leaf visited
    takes the nearest integer at every level, i.e. the nearest-plane point.
    Returns (Q_opt, loss_opt, Q_first_leaf)."""
    W = np.asarray(W, np.float64)
    m, n = W.shape
    lo, hi = grid_bounds(bits, clamp)
    M = np.kron(reverse_cholesky(H_R), reverse_cholesky(H_L))
    x = W.reshape(-1, order="F")
    sv = np.tile(np.asarray(s, np.float64), n)
    N = m * n
    best = [np.inf, None]
    first = [None]
    z = np.zeros(N)

    def rec(p, partial):
        if p == N:
            if first[0] is None:
                first[0] = z.copy()
            if partial < best[0]:
                best[0], best[1] = partial, z.copy()
            return
        # residual row p: M[p,p] (x_p - z_p) + sum_{p'<p} M[p,p'] (x_p' - z_p')
        off = M[p, :p] @ (x[:p] - z[:p])
        c = (x[p] + off / M[p, p]) / sv[p]
        k0 = round_to_grid(c, lo, hi)
        cand = [k0]
        for step in range(1, 64):
            for k in (k0 + step, k0 - step) if c >= k0 else (k0 - step, k0 + step):
                if lo <= k <= hi:
                    cand.append(k)
        cand.sort(key=lambda k: abs(c - k))
        for k in cand:
            r = M[p, p] * sv[p] * (c - k)
            nxt = partial + r * r
            if nxt >= best[0]:
                break
            z[p] = sv[p] * k
            rec(p + 1, nxt)
        z[p] = 0.0

    rec(0, 0.0)
    to_q = lambda v: (v / sv).reshape((m, n), order="F")
    return to_q(best[1]), best[0], to_q(first[0])


# --------------------------------------------------------------------------- #
# Hessians with more than two Kronecker factors (arxivlens, Abstract: the
# algorithm extends to any number of Kronecker factors)
# --------------------------------------------------------------------------- #
# Reading: W is a k-way tensor of shape (m_1, ..., m_k), stored in C order (last
# index fastest); H_j (m_j x m_j) acts on mode j, so the proxy loss is
#     L(Q) = sum_{i, i'} dW[i] dW[i'] prod_j H_j[i_j, i'_j]
# and on the C-order flattening the Gram is H_1 kron H_2 kron ... kron H_k.  Scales
# are per index of mode 1 (the output channel), as the per-row scales of the 2-D
# case.  With two factors this is the 2-D problem with H_L = H_1, H_R = H_2.


def kron_gram(Hs):
    """G = H_1 kron ... kron H_k: the Gram of the C-order flattening."""
    G = np.ones((1, 1))
    for H in Hs:
        G = np.kron(G, np.asarray(H, np.float64))
    return G


def babai_tensor_sweep(W, Hs, s, bits, clamp):
    """1-D GPTQ over all coordinates of the tensor in C order (a linear extension
    of the product order on multi-indices), on the explicit Gram kron_gram(Hs):
    the same form as babai_kron_sweep (upper Cholesky factor of G^{-1}, each
    rounding error divided by the pivot and pushed along its row).  Returns (Q, T)
    shaped like W.  Tiny problems only (the Gram is N x N, N = W.size).
    """
    W = np.asarray(W, np.float64)
    lo, hi = grid_bounds(bits, clamp)
    G = kron_gram(Hs)
    U = np.linalg.cholesky(np.linalg.inv(G)).T
    x = W.reshape(-1).copy()
    N = x.size
    sv = np.repeat(np.asarray(s, np.float64), N // W.shape[0])   # mode 1 is the slowest index
    Q = np.zeros(N)
    T = np.zeros(N)
    for p in range(N):
        T[p] = x[p] / sv[p]
        Q[p] = round_to_grid(T[p], lo, hi)
        e = (x[p] - sv[p] * Q[p]) / U[p, p]
        x[p + 1:] -= e * U[p, p + 1:]
    return Q.reshape(W.shape), T.reshape(W.shape)


def mode_product(X, M, j):
    """(X x_j M)[..., a, ...] = sum_b M[a, b] X[..., b, ...] (mode-j product)."""
    return np.moveaxis(np.tensordot(M, X, axes=([1], [j])), 0, j)


def gptq_kron_hyperplane(W, Ms, s, bits, clamp):
    """GPTQ with a k-factor Kronecker Hessian, hyperplane by hyperplane.

    With lower factors M_j (M_j^T M_j = H_j), the triangular factor of the
    flattened problem is M_1 kron ... kron M_k, so the value rounded at entry i
    is
        y_i = W_i + (dW x_1 M_1 x_2 M_2 ... x_k M_k)_i / prod_j M_j[i_j, i_j]
    with dW = 0 on the entries not rounded yet (i itself included): each mode's
    factor applied separately (the separable feedback), and only the dominated
    orthant {i' <= i} contributes because every M_j is lower triangular.  The
    entries of one hyperplane i_1 + ... + i_k = d depend only on earlier
    hyperplanes, so each hyperplane is rounded as one vector.  Evaluated from
    scratch for every hyperplane: small tensors only.

    Returns a Result (Q, T = y/s, loss by the nearest-plane identity, clamp count,
    near-tie mask), arrays shaped like W.
    """
    W = np.asarray(W, np.float64)
    Ms = [np.asarray(M, np.float64) for M in Ms]
    if len(Ms) != W.ndim or any(M.shape != (d, d) for M, d in zip(Ms, W.shape)):
        raise ValueError("one square factor per mode")
    s = np.asarray(s, np.float64)
    lo, hi = grid_bounds(bits, clamp)
    idx = np.indices(W.shape)
    level = idx.sum(axis=0)
    diag = np.ones(W.shape)
    for j, M in enumerate(Ms):
        diag = diag * np.diag(M)[idx[j]]
    srow = s[idx[0]]
    D = np.zeros(W.shape)
    Q = np.zeros(W.shape)
    T = np.zeros(W.shape)
    tie = np.zeros(W.shape, bool)
    loss = 0.0
    n_clamped = 0
    for d in range(int(level.max()) + 1 if W.size else 0):
        F = D
        for j, M in enumerate(Ms):
            F = mode_product(F, M, j)
        sel = level == d
        y = W[sel] + F[sel] / diag[sel]
        t = y / srow[sel]
        q_raw = np.rint(t)
        q = np.clip(q_raw, lo, hi)
        n_clamped += int(np.count_nonzero(q != q_raw))
        D[sel] = W[sel] - srow[sel] * q
        loss += float(np.sum((diag[sel] * (y - srow[sel] * q)) ** 2))
        Q[sel] = q
        T[sel] = t
        tie[sel] = near_tie(t, lo, hi)
    return Result(Q, T, loss, n_clamped, tie, set())


def proxy_loss_tensor(W, Q, s, Hs):
    """L(Q) = sum dW[i] dW[i'] prod_j H_j[i_j, i'_j], dW = W - s Q (s along mode 1)."""
    W = np.asarray(W, np.float64)
    D = W - np.asarray(s, np.float64).reshape((-1,) + (1,) * (W.ndim - 1)) * np.asarray(Q, np.float64)
    HD = D
    for j, H in enumerate(Hs):
        HD = mode_product(HD, np.asarray(H, np.float64), j)
    return float(np.sum(D * HD))


def kron_factor(Ms):
    """M_1 kron ... kron M_k of lower factors: lower triangular, and the reverse
    Cholesky factor of H_1 kron ... kron H_k (uniqueness of the factor with a
    positive diagonal)."""
    return kron_gram(Ms)


def gptq_kron_via_2d(W, Ms, s, bits, clamp, **kw):
    """The k-factor problem as a 2-D one: rows = mode 1 (H_L = H_1), columns = modes
    2..k flattened in C order (H_R = H_2 kron ... kron H_k, factor M_2 kron ... kron
    M_k).  Column-major vec of that m_1 x (m_2...m_k) matrix orders the coordinates
    by a linear extension of the k-way product order, and its factor has the
    k-way dominated-orthant sparsity, so the anti-diagonal algorithm computes the
    same rounding.  Returns the 2-D Result (arrays m_1 x N/m_1)."""
    W = np.asarray(W, np.float64)
    W2 = W.reshape(W.shape[0], -1)
    M_R = kron_factor(Ms[1:]) if len(Ms) > 1 else np.ones((1, 1))
    return gptq2d_antidiagonal(W2, Ms[0], M_R, s, bits, clamp, **kw)


# --------------------------------------------------------------------------- #
# The Kronecker factors from calibration activations (the step before the
# path: arxivlens, Analysis > Limitations, fixed bases A, B whose Grams are
# factored; Future work, "Gram factorizations")
# --------------------------------------------------------------------------- #
# Reading: a factor is the Gram of its basis, H = A^T A, with A = X / sqrt(N) for N
# rows of activations X (N x k), i.e. H = X^T X / N, plus GPTQ's usual damping of
# the diagonal by a fraction of its mean (the pages give no damping; it keeps a
# rank-deficient Gram positive definite).


def gram(X, damp=0.0):
    """H = X^T X / N + damp * mean(diag(X^T X / N)) * I, in fp64 (X upcast exactly)."""
    X = np.asarray(X, np.float64)
    N = X.shape[0]
    H = X.T @ X / N
    H[np.diag_indices_from(H)] += damp * float(np.mean(np.diag(H))) if H.size else 0.0
    return H


def gram_batches(batches, damp=0.0):
    """The same Gram accumulated over batches of rows: sum of X_b^T X_b over all
    batches, divided by the total row count, then damped."""
    S = None
    N = 0
    for X in batches:
        X = np.asarray(X, np.float64)
        S = X.T @ X if S is None else S + X.T @ X
        N += X.shape[0]
    H = S / N
    H[np.diag_indices_from(H)] += damp * float(np.mean(np.diag(H)))
    return H

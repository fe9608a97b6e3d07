"""Pins for the oracle's grid variants: group-wise scales, asymmetric grids with
integer zero points, and packed 4-bit output.

The pages fix only a 4-bit integer grid (mind-verse.de "Neue Ansätze ... durch
GPTQ-2D", section "Quantisierung von Large Language Models").  The variants are
GPTQ's usual ones: a scale per (row, group of columns), and a code c in
[0, 2^bits - 1] standing for s (c - z) with an integer zero point z.  Each test
ties the variant to something other than the oracle's own anti-diagonal code:
the definition (conditional minimiser) and the naive Kronecker sweep with the
same per-entry grid, the per-row path in the cases that reduce to it, a closed
form (RTN in code space), textbook 1-D GPTQ with per-coordinate grids, the loss
identity, and bytes derived by hand for the packed format.
"""
import os

import numpy as np
import pytest

import oracle as O
import workloads as WL

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _spd(rng, k):
    X = WL.student_t_activations(rng, 4 * k, k)
    return WL.damped_gram(X).astype(np.float64)


def _grid_case(seed, m, n, G, asym, bits=3):
    rng = np.random.default_rng(700 + 13 * seed + 5 * m + n + 3 * G + int(asym))
    W = rng.uniform(-1, 1, (m, n)) * rng.uniform(0.2, 2.0, (m, 1))
    H_L, H_R = _spd(rng, m), _spd(rng, n)
    if asym:
        S, Z = WL.group_minmax_grid(W, bits, G)
        S = S * rng.uniform(0.6, 1.0, S.shape)   # tighter grids: more clamping
        return W, H_L, H_R, S.astype(np.float64), Z
    S = WL.group_absmax_scales(W, bits, G if G else n).astype(np.float64)
    return W, H_L, H_R, S * rng.uniform(0.5, 1.0, S.shape), None


CASES = [(3, 4, 2), (4, 6, 3), (2, 7, 2), (5, 3, 0), (3, 5, 4), (1, 6, 2), (6, 1, 1)]


@pytest.mark.parametrize("m,n,G", CASES, ids=lambda *a: None)
@pytest.mark.parametrize("asym", [False, True])
@pytest.mark.parametrize("clamp", [False, True])
@pytest.mark.parametrize("seed", [0, 1])
def test_grid_variants_definition_sweep_and_antidiagonal_agree(m, n, G, asym, clamp, seed):
    W, H_L, H_R, S, Z = _grid_case(seed, m, n, G, asym)
    grid = O.expand_grid(m, n, S, 3, clamp, G, Z)
    Q0r, T0r = O.nearest_plane_by_definition(W, H_L, H_R, None, 3, clamp, "row", grid=grid)
    Q0c, T0c = O.nearest_plane_by_definition(W, H_L, H_R, None, 3, clamp, "col", grid=grid)
    Q1, T1 = O.babai_kron_sweep(W, H_L, H_R, None, 3, clamp, grid=grid)
    r2 = O.gptq2d_antidiagonal(W, O.reverse_cholesky(H_L), O.reverse_cholesky(H_R), None, 3,
                               clamp, grid=grid)
    for Q, T in ((Q0r, T0r), (Q0c, T0c), (Q1, T1)):
        np.testing.assert_array_equal(Q, r2.Q)
        np.testing.assert_allclose(T, r2.T, rtol=0, atol=1e-9)
    _, LO, HI = grid
    assert np.all(r2.Q >= LO) and np.all(r2.Q <= HI)


@pytest.mark.parametrize("clamp", [False, True])
def test_one_group_and_equal_group_scales_reduce_to_per_row(clamp):
    rng = np.random.default_rng(31)
    m, n = 7, 10
    W = rng.normal(0, 1, (m, n))
    H_L, H_R = _spd(rng, m), _spd(rng, n)
    s = rng.uniform(0.2, 0.6, m)
    ref = O.gptq2d(W, H_L, H_R, s, 4, clamp)
    ML, MR = O.reverse_cholesky(H_L), O.reverse_cholesky(H_R)
    for G, S in ((n, s[:, None]), (16, s[:, None]), (3, np.repeat(s[:, None], 4, 1))):
        r = O.gptq2d_antidiagonal(W, ML, MR, None, 4, clamp, grid=O.expand_grid(m, n, S, 4, clamp, G))
        np.testing.assert_array_equal(r.Q, ref.Q)
        np.testing.assert_array_equal(r.T, ref.T)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_midpoint_zero_point_is_the_symmetric_grid(bits):
    """z = 2^(bits-1) makes the code range [0, 2^bits - 1] the symmetric range shifted."""
    rng = np.random.default_rng(40 + bits)
    m, n, G = 6, 8, 4
    W = rng.normal(0, 1, (m, n))
    H_L, H_R = _spd(rng, m), _spd(rng, n)
    S = rng.uniform(0.1, 0.5, (m, 2))
    Z = np.full((m, 2), 1 << (bits - 1))
    ML, MR = O.reverse_cholesky(H_L), O.reverse_cholesky(H_R)
    ra = O.gptq2d_antidiagonal(W, ML, MR, None, bits, True, grid=O.expand_grid(m, n, S, bits, True, G, Z))
    rs = O.gptq2d_antidiagonal(W, ML, MR, None, bits, True, grid=O.expand_grid(m, n, S, bits, True, G))
    np.testing.assert_array_equal(ra.Q, rs.Q)
    codes = O.stored_codes(ra.Q, m, n, bits, G, Z)
    np.testing.assert_array_equal(codes - (1 << (bits - 1)), rs.Q)


def test_identity_metric_is_rtn_in_code_space():
    """H = I: every entry rounds alone, c = clamp(rint(W / s + z), 0, 2^bits - 1)."""
    rng = np.random.default_rng(50)
    m, n, G, bits = 5, 12, 4, 4
    W = rng.normal(0, 1, (m, n))
    S, Z = WL.group_minmax_grid(W, bits, G)
    r = O.gptq2d_antidiagonal(W, np.eye(m), np.eye(n), None, bits, True,
                              grid=O.expand_grid(m, n, S, bits, True, G, Z))
    col = np.arange(n) // G
    Se = S.astype(np.float64)[:, col]
    Ze = Z.astype(np.float64)[:, col]
    expect = np.clip(np.rint(W / Se + Ze), 0, (1 << bits) - 1)
    np.testing.assert_array_equal(O.stored_codes(r.Q, m, n, bits, G, Z), expect)


@pytest.mark.parametrize("asym", [False, True])
def test_one_sided_metrics_are_textbook_gptq_with_per_entry_grids(asym):
    rng = np.random.default_rng(60 + asym)
    m, n, G = 6, 9, 3
    W = rng.normal(0, 1, (m, n))
    H = _spd(rng, n), _spd(rng, m)
    if asym:
        S, Z = WL.group_minmax_grid(W, 3, G)
    else:
        S, Z = WL.group_absmax_scales(W, 3, G), None
    S, LO, HI = O.expand_grid(m, n, S, 3, True, G, Z)
    grid = (S, LO, HI)
    r = O.gptq2d_antidiagonal(W, np.eye(m), O.reverse_cholesky(H[0]), None, 3, True, grid=grid)
    for i in range(m):      # H_L = I: rows are independent 1-D problems along j
        np.testing.assert_array_equal(r.Q[i], O.gptq_1d_obs(W[i], H[0], S[i], 3, True, (LO[i], HI[i])))
    r = O.gptq2d_antidiagonal(W[:, :m], O.reverse_cholesky(H[1]), np.eye(m), None, 3, True,
                              grid=(S[:, :m], LO[:, :m], HI[:, :m]))
    for j in range(m):      # H_R = I: columns along i
        np.testing.assert_array_equal(r.Q[:, j], O.gptq_1d_obs(W[:, j], H[1], S[:, j], 3, True,
                                                                (LO[:, j], HI[:, j])))


@pytest.mark.parametrize("asym", [False, True])
def test_loss_identity_with_per_entry_grid(asym):
    W, H_L, H_R, S, Z = _grid_case(9, 6, 8, 3, asym)
    grid = O.expand_grid(6, 8, S, 3, True, 3, Z)
    r = O.gptq2d_antidiagonal(W, O.reverse_cholesky(H_L), O.reverse_cholesky(H_R), None, 3, True,
                              grid=grid)
    assert O.proxy_loss(W, r.Q, grid[0], H_L, H_R) == pytest.approx(r.loss_identity, rel=1e-10)


def _read_packed():
    rows = []
    with open(os.path.join(GOLDEN, "packed_nibbles.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            left, right = line.split("|")
            kind, bits, *vals = left.split()
            rows.append((kind, int(bits), [int(v) for v in vals], bytes.fromhex(right.replace(" ", ""))))
    return rows


@pytest.mark.parametrize("row", _read_packed(), ids=lambda r: " ".join(map(str, r[2])))
def test_packed_nibbles_golden(row):
    kind, bits, vals, expect = row
    v = np.array([vals], np.float64)
    codes = O.packed_codes(v, 1, v.shape[1], bits) if kind == "sym" else v
    assert O.pack_nibbles(codes).tobytes() == expect


def test_minmax_grid_covers_each_group():
    """Harness check: every (row, group) range lies inside its representable range."""
    rng = np.random.default_rng(70)
    W = rng.normal(0, 1, (9, 37))
    S, Z = WL.group_minmax_grid(W, 4, 8)
    col = np.arange(37) // 8
    Se, Ze = S.astype(np.float64)[:, col], Z.astype(np.float64)[:, col]
    assert np.all(W >= Se * (0 - Ze) - Se * 0.5 - 1e-12)
    assert np.all(W <= Se * (15 - Ze) + Se * 0.5 + 1e-12)

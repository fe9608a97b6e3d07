"""Pins for the oracle of the step before the path: a Kronecker factor as the Gram of
its basis, H = X^T X / N plus diagonal damping (arxivlens "GPTQ-2D: Cubic-Time
Two-Sided Adaptive Rounding", Analysis > Limitations and Future work: fixed bases
whose Gram factorizations are prepared; the damping is GPTQ's usual one, a reading).
"""
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows():
    out = []
    for line in open(os.path.join(GOLDEN, "gram_3x2.txt")):
        if line.startswith("#") or not line.strip():
            continue
        xs, damp, hs = line.split("|")
        X = np.array([[float(v) for v in r.split()] for r in xs.split(";")])
        out.append((X, float(damp), np.array([float(v) for v in hs.split()]).reshape(2, 2)))
    return out


@pytest.mark.parametrize("case", _rows(), ids=["damped", "plain"])
def test_gram_hand_example(case):
    X, damp, H = case
    np.testing.assert_allclose(O.gram(X, damp), H, rtol=1e-15, atol=0)


def test_gram_entries_are_column_dot_products_and_batches_add():
    """Entry (i, j) is the mean over rows of X[:, i] X[:, j] (brute force), and the
    batched form equals the one-shot form for any split of the rows."""
    rng = np.random.default_rng(1)
    X = rng.normal(0, 1, (37, 6))
    H = O.gram(X, 0.0)
    for i in range(6):
        for j in range(6):
            assert H[i, j] == pytest.approx(sum(X[r, i] * X[r, j] for r in range(37)) / 37, rel=1e-13)
    Hb = O.gram_batches([X[:5], X[5:20], X[20:]], 0.1)
    np.testing.assert_allclose(Hb, O.gram(X, 0.1), rtol=1e-13, atol=1e-14)


def test_damping_shifts_the_spectrum_by_a_fraction_of_the_mean_diagonal():
    """A rank-deficient Gram (fewer rows than columns) becomes positive definite: its
    smallest eigenvalue is exactly damp * mean(diag)."""
    rng = np.random.default_rng(2)
    X = rng.normal(0, 1, (3, 8))
    H = O.gram(X, 0.05)
    mu = float(np.mean(np.diag(O.gram(X, 0.0))))
    assert np.linalg.eigvalsh(H).min() == pytest.approx(0.05 * mu, rel=1e-9)

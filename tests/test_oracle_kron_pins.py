"""Pins for the oracle of Hessians with more than two Kronecker factors
(arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Abstract: the
algorithm extends to any number of Kronecker factors).

Each test ties the k-way oracle to something other than itself: the 1-D GPTQ
sweep on the explicit N x N Gram, textbook 1-D GPTQ along each mode when every
other factor is the identity, RTN for diagonal metrics, the closed form of the
Kronecker factor, the nearest-plane loss identity and bound, and the
independence of the result from the order of modes 2..k.
"""
import itertools

import numpy as np
import pytest

import oracle as O
import workloads as WL


def _spd(rng, k):
    X = WL.student_t_activations(rng, 4 * k, k)
    return WL.damped_gram(X).astype(np.float64)


def _case(seed, shape):
    rng = np.random.default_rng(1000 + 37 * seed + sum(shape) * 11 + len(shape))
    W = rng.uniform(-4, 4, shape)
    Hs = [_spd(rng, d) for d in shape]
    s = rng.uniform(0.3, 1.5, shape[0])
    return W, Hs, s


SHAPES = [(2, 3, 2), (3, 2, 4), (1, 3, 3), (3, 1, 2), (4, 3, 1), (2, 2, 2, 2), (3, 2, 1, 2)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("clamp", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_hyperplane_matches_naive_sweep_and_2d_reduction(shape, clamp, seed):
    W, Hs, s = _case(seed, shape)
    Ms = [O.reverse_cholesky(H) for H in Hs]
    Q1, T1 = O.babai_tensor_sweep(W, Hs, s, 3, clamp)
    rk = O.gptq_kron_hyperplane(W, Ms, s, 3, clamp)
    r2 = O.gptq_kron_via_2d(W, Ms, s, 3, clamp)
    np.testing.assert_array_equal(rk.Q, Q1)
    np.testing.assert_allclose(rk.T, T1, rtol=0, atol=1e-9)
    np.testing.assert_array_equal(r2.Q.reshape(shape), Q1)
    np.testing.assert_allclose(r2.T.reshape(shape), T1, rtol=0, atol=1e-9)
    assert r2.loss_identity == pytest.approx(rk.loss_identity, rel=1e-10)


@pytest.mark.parametrize("clamp", [False, True])
def test_two_factors_is_the_2d_problem(clamp):
    W, Hs, s = _case(5, (6, 7))
    rk = O.gptq_kron_hyperplane(W, [O.reverse_cholesky(H) for H in Hs], s, 4, clamp)
    r2 = O.gptq2d(W, Hs[0], Hs[1], s, 4, clamp)
    np.testing.assert_array_equal(rk.Q, r2.Q)
    np.testing.assert_allclose(rk.T, r2.T, rtol=0, atol=1e-10)


@pytest.mark.parametrize("clamp", [False, True])
def test_diagonal_metrics_give_rtn(clamp):
    rng = np.random.default_rng(8)
    shape = (4, 3, 5)
    W = rng.normal(0, 1, shape)
    s = rng.uniform(0.1, 0.4, 4)
    Ms = [np.diag(np.sqrt(rng.uniform(0.5, 3, d))) for d in shape]
    r = O.gptq_kron_hyperplane(W, Ms, s, 4, clamp)
    lo, hi = O.grid_bounds(4, clamp)
    np.testing.assert_array_equal(r.Q, np.clip(np.rint(W / s[:, None, None]), lo, hi))


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("clamp", [False, True])
def test_one_nontrivial_factor_is_textbook_gptq_along_its_mode(mode, clamp):
    """All factors but H_mode equal to I: every fibre along that mode is rounded by
    1-D GPTQ (OBS form) with H_mode, independently of the others."""
    rng = np.random.default_rng(20 + mode)
    shape = (5, 4, 6)
    W = rng.normal(0, 1, shape)
    s = rng.uniform(0.2, 0.5, shape[0])
    H = _spd(rng, shape[mode])
    Ms = [np.eye(d) for d in shape]
    Ms[mode] = O.reverse_cholesky(H)
    r = O.gptq_kron_hyperplane(W, Ms, s, 3, clamp)
    others = [range(d) for k, d in enumerate(shape) if k != mode]
    for rest in itertools.product(*others):
        sl = list(rest)
        sl.insert(mode, slice(None))
        sl = tuple(sl)
        sv = s if mode == 0 else s[sl[0]]
        np.testing.assert_array_equal(r.Q[sl], O.gptq_1d_obs(W[sl], H, sv, 3, clamp))


def test_modes_after_the_first_can_be_reordered():
    """Order independence: swapping modes 2 and 3 (with their factors) transposes
    the result, although the C-order sweep of the swapped tensor visits the
    coordinates in another order."""
    W, Hs, s = _case(3, (3, 4, 5))
    Ms = [O.reverse_cholesky(H) for H in Hs]
    a = O.gptq_kron_hyperplane(W, Ms, s, 3, True)
    b = O.gptq_kron_hyperplane(W.transpose(0, 2, 1), [Ms[0], Ms[2], Ms[1]], s, 3, True)
    np.testing.assert_array_equal(a.Q, b.Q.transpose(0, 2, 1))
    Q1, _ = O.babai_tensor_sweep(W.transpose(0, 2, 1), [Hs[0], Hs[2], Hs[1]], s, 3, True)
    np.testing.assert_array_equal(a.Q, Q1.transpose(0, 2, 1))


def test_kron_factor_is_the_reverse_cholesky_of_the_kron_gram():
    rng = np.random.default_rng(9)
    Hs = [_spd(rng, d) for d in (3, 4, 2)]
    K = O.kron_factor([O.reverse_cholesky(H) for H in Hs])
    np.testing.assert_allclose(K, O.reverse_cholesky(O.kron_gram(Hs)), rtol=1e-10, atol=1e-10)
    assert np.all(np.triu(K, 1) == 0)


@pytest.mark.parametrize("clamp", [False, True])
def test_loss_identity_and_bound(clamp):
    W, Hs, s = _case(4, (3, 3, 4))
    Ms = [O.reverse_cholesky(H) for H in Hs]
    r = O.gptq_kron_hyperplane(W, Ms, s, 3, clamp)
    assert O.proxy_loss_tensor(W, r.Q, s, Hs) == pytest.approx(r.loss_identity, rel=1e-9)
    if not clamp:
        d2 = np.ones(W.shape)
        idx = np.indices(W.shape)
        for j, M in enumerate(Ms):
            d2 = d2 * np.diag(M)[idx[j]] ** 2
        assert r.loss_identity <= 0.25 * float(np.sum(d2 * s[idx[0]] ** 2)) * (1 + 1e-12)


def test_mode_product_on_a_matrix_is_left_and_right_multiplication():
    """On a matrix, the mode-0 product is A X and the mode-1 product is X B^T."""
    rng = np.random.default_rng(7)
    X, A, B = rng.normal(size=(3, 5)), rng.normal(size=(3, 3)), rng.normal(size=(5, 5))
    np.testing.assert_allclose(O.mode_product(X, A, 0), A @ X, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(O.mode_product(X, B, 1), X @ B.T, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("shape", [(3, 4), (2, 3, 4), (2, 2, 3, 2)])
def test_mode_products_are_the_kronecker_matrix_on_the_flattening(shape):
    """Applying M_j along every mode j is M_1 kron ... kron M_k acting on the C-order
    flattening (mode 1 slowest), the identity behind the separable feedback; checked
    against numpy's Kronecker product of the explicit matrices."""
    rng = np.random.default_rng(sum(shape) + len(shape))
    X = rng.normal(size=shape)
    Ms = [rng.normal(size=(d, d)) for d in shape]
    Y = X
    for j, M in enumerate(Ms):
        Y = O.mode_product(Y, M, j)
    K = Ms[0]
    for M in Ms[1:]:
        K = np.kron(K, M)
    np.testing.assert_allclose(Y.reshape(-1), K @ X.reshape(-1), rtol=1e-12, atol=1e-12)

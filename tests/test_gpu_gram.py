"""GPU parity of the Kronecker factors from activations (gptq2d_gram_accumulate /
gptq2d_gram_finalize, tcgen05 tensor cores, bf16 operands, fp32 accumulation) against
the oracle's Gram (arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding",
Analysis > Limitations and Future work: the fixed bases' Grams).

Bar:
  * small-integer activations (|x| <= 4, rows <= 4096): every product and partial sum
    is an integer below 2^24, exact in fp32 whatever the summation order, so the
    lower block triangle must equal X^T X bit for bit, and nothing else is written;
  * real activations: within the fp32 summation bound (rows + 16) 2^-23 (|X|^T |X|)
    (products of bf16 values are exact in fp32);
  * finalize: H / N + damp * mean(diag) within fp32 rounding of the oracle's fp64 value;
  * the factor prepared from it rounds W exactly as the oracle does with that factor.
"""
import numpy as np
import pytest

import oracle as O
import workloads as WL
from tests.parity import check_against_oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from two_sided_adaptive_b200 import build as gbuild
    gbuild.build()
    import two_sided_adaptive_b200 as g
    return g


def _ws(g):
    return torch.zeros(256, dtype=torch.uint8, device="cuda")


def _lower_block_mask(k, b=128):
    i = np.arange(k)[:, None] // b
    j = np.arange(k)[None, :] // b
    return j <= i


@pytest.mark.parametrize("rows,k", [(1, 8), (5, 8), (64, 128), (100, 136), (300, 256),
                                    (4096, 384), (130, 520), (63, 64), (129, 1024),
                                    (257, 1160)])
def test_integer_activations_are_exact(g, rows, k):
    rng = np.random.default_rng(rows * 1000 + k)
    X = rng.integers(-4, 5, (rows, k)).astype(np.float32)
    H = torch.full((k, k), float("nan"), dtype=torch.float32, device="cuda")
    g.gram_accumulate(torch.from_numpy(X).cuda().to(torch.bfloat16), H, accumulate=False,
                      workspace=_ws(g))
    torch.cuda.synchronize()
    Hg = H.cpu().numpy()
    ref = X.astype(np.int64).T @ X.astype(np.int64)
    m = _lower_block_mask(k)
    np.testing.assert_array_equal(Hg[m], ref[m].astype(np.float32))
    assert np.all(np.isnan(Hg[~m]))  # nothing outside the lower block triangle is written


@pytest.mark.parametrize("rows,k", [(200, 5000), (65, 6664)])
def test_many_tiles_per_cluster_pair_exact(g, rows, k):
    """Widths with more 256 x 256 tiles than three per SM pair (210 and 351 tiles on
    74 pairs): each pair reuses both tensor-memory accumulators, so the epilogue's
    hand-back to the MMA thread is exercised.  Two batches (overwrite, then add)."""
    rng = np.random.default_rng(rows + k)
    X1 = rng.integers(-4, 5, (rows, k)).astype(np.float32)
    X2 = rng.integers(-4, 5, (rows // 2 + 1, k)).astype(np.float32)
    H = torch.full((k, k), float("nan"), dtype=torch.float32, device="cuda")
    ws = _ws(g)
    g.gram_accumulate(torch.from_numpy(X1).cuda().to(torch.bfloat16), H, accumulate=False,
                      workspace=ws)
    g.gram_accumulate(torch.from_numpy(X2).cuda().to(torch.bfloat16), H, accumulate=True,
                      workspace=ws)
    torch.cuda.synchronize()
    Hg = H.cpu().numpy()
    # small integers: every sum is exact in fp64 (and in fp32 on the GPU)
    X1d, X2d = X1.astype(np.float64), X2.astype(np.float64)
    ref = X1d.T @ X1d + X2d.T @ X2d
    m = _lower_block_mask(k)
    np.testing.assert_array_equal(Hg[m], ref[m].astype(np.float32))
    assert np.all(np.isnan(Hg[~m]))


def test_real_activations_within_fp32_bound(g):
    rng = np.random.default_rng(7)
    rows, k = 2048, 256
    X = WL.student_t_activations(rng, rows, k)
    Xb = torch.from_numpy(X.astype(np.float32)).cuda().to(torch.bfloat16)
    Xd = Xb.double().cpu().numpy()
    H = torch.zeros((k, k), dtype=torch.float32, device="cuda")  # entries above the block triangle stay untouched
    g.gram_accumulate(Xb, H, accumulate=False, workspace=_ws(g))
    torch.cuda.synchronize()
    Hg = H.cpu().numpy().astype(np.float64)
    ref = Xd.T @ Xd
    bound = (rows + 16) * 2.0 ** -23 * (np.abs(Xd).T @ np.abs(Xd))
    m = _lower_block_mask(k)
    assert np.all(np.abs(Hg - ref)[m] <= bound[m])


def test_batches_finalize_and_damping(g):
    rng = np.random.default_rng(8)
    k = 200
    batches = [rng.integers(-3, 4, (r, k)).astype(np.float32) for r in (70, 1, 333)]
    ws = _ws(g)
    H = torch.empty((k, k), dtype=torch.float32, device="cuda")
    for b, X in enumerate(batches):
        g.gram_accumulate(torch.from_numpy(X).cuda().to(torch.bfloat16), H, accumulate=b > 0,
                          workspace=ws)
    g.gram_finalize(H, sum(x.shape[0] for x in batches), 0.01, workspace=ws)
    torch.cuda.synchronize()
    ref = O.gram_batches(batches, 0.01)
    low = np.tril(np.ones((k, k), bool))
    np.testing.assert_allclose(H.cpu().numpy()[low], ref[low], rtol=2 ** -23, atol=0)


def test_zero_rows_give_zero(g):
    k = 136
    H = torch.full((k, k), 5.0, dtype=torch.float32, device="cuda")
    X = torch.empty((0, k), dtype=torch.bfloat16, device="cuda")
    g.gram_accumulate(X, H, accumulate=False, workspace=_ws(g))
    torch.cuda.synchronize()
    m = _lower_block_mask(k)
    assert np.all(H.cpu().numpy()[m] == 0.0)


def test_gram_prepare_quantize_chain(g):
    """Activations -> Grams on the tensor cores -> factors -> rounding: the rounding
    equals the oracle's with factors from LAPACK of the same (GPU-formed) Grams."""
    rng = np.random.default_rng(9)
    m, n = 136, 200
    XL = WL.student_t_activations(rng, 4 * m, m).astype(np.float32)
    XR = WL.student_t_activations(rng, 4 * n, n).astype(np.float32)
    HL = g.gram([torch.from_numpy(XL).cuda().to(torch.bfloat16)], 0.01)
    HR = g.gram([torch.from_numpy(XR[:300]).cuda().to(torch.bfloat16),
                 torch.from_numpy(XR[300:]).cuda().to(torch.bfloat16)], 0.01)
    ML, MR = g.prepare_pair(HL, HR)
    W = rng.normal(0, 0.02, (m, n)).astype(np.float32)
    s = WL.absmax_scales(W.astype(np.float64), 4)
    Q, st = g.quantize(torch.from_numpy(W).cuda(), ML, MR, torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    sym = lambda H: np.tril(H) + np.tril(H, -1).T
    HLc = sym(HL.cpu().numpy().astype(np.float64))
    HRc = sym(HR.cpu().numpy().astype(np.float64))
    rep = check_against_oracle(W.astype(np.float64), O.reverse_cholesky(HLc), O.reverse_cholesky(HRc),
                               s.astype(np.float64), 4, True, Q.cpu().numpy())
    assert g.stats_dict(st)["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)


@pytest.mark.slow
def test_attention_width_gram_sampled(g):
    """The 4096-wide Gram of 4096 activation rows (the attention layer's recipe), in the
    bench's configuration: 256 sampled entries against fp64 dot products."""
    rng = np.random.default_rng(10)
    rows, k = 4096, 4096
    X = WL.student_t_activations(rng, rows, k).astype(np.float32)
    Xb = torch.from_numpy(X).cuda().to(torch.bfloat16)
    H = g.gram([Xb], 0.0)
    torch.cuda.synchronize()
    Xd = Xb.double().cpu().numpy()
    Hg = H.cpu().numpy()
    idx = rng.integers(0, k, (256, 2))
    for i, j in idx:
        i, j = max(i, j), min(i, j)
        ref = Xd[:, i] @ Xd[:, j] / rows
        bound = (rows + 16) * 2.0 ** -23 * (np.abs(Xd[:, i]) @ np.abs(Xd[:, j])) / rows + \
            abs(ref) * 2.0 ** -23
        assert abs(Hg[i, j] - ref) <= bound

"""Randomised GPU parity: seeded draws of shape, W dtype, bits, clamp and grid variant
(per-row / group-wise scales, symmetric / zero points, byte / packed output), each
rounded through gptq2d_quantize_grid and checked against the oracle with the near-tie
replay (arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Abstract: the
same rounding as the naive Kronecker sweep).  The draws are fixed by the seed, so a
failure reproduces."""
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


def _draw(seed):
    rng = np.random.default_rng(9000 + seed)
    m = int(rng.integers(1, 200))
    n = int(rng.integers(1, 200))
    wdt = [torch.float32, torch.bfloat16, torch.float64][int(rng.integers(0, 3))]
    clamp = bool(rng.random() < 0.85)
    bits = int(rng.integers(2, 9)) if clamp else 4
    G = [0, 8, 16, 24, 32, 64, 128][int(rng.integers(0, 7))]
    asym = clamp and rng.random() < 0.5
    packed = clamp and bits <= 4 and rng.random() < 0.5
    return rng, m, n, wdt, bits, clamp, G, asym, packed


@pytest.mark.parametrize("seed", range(16))
def test_random_grid_problem_matches_oracle(g, seed):
    rng, m, n, wdt, bits, clamp, G, asym, packed = _draw(seed)
    W = rng.normal(0, 0.05, (m, n))
    H_L = WL.damped_gram(WL.student_t_activations(rng, 3 * m + 8, m))
    H_R = WL.damped_gram(WL.student_t_activations(rng, 3 * n + 8, n))
    ML, MR = O.reverse_cholesky(H_L.astype(np.float64)), O.reverse_cholesky(H_R.astype(np.float64))
    Wt = torch.from_numpy(W).cuda().to(wdt)
    Wd = Wt.double().cpu().numpy()
    if asym:
        S, Z = WL.group_minmax_grid(Wd, bits, G)
    else:
        S = WL.group_absmax_scales(Wd, bits, G if G else max(n, 1)) if clamp else \
            (np.full((m, 1), 0.01, np.float32))
        Z = None
    Geff = G if (asym or clamp) else 0
    Qb, st = g.quantize_grid(Wt, torch.from_numpy(ML).cuda(), torch.from_numpy(MR).cuda(),
                             torch.from_numpy(S).cuda(), bits, clamp, group_size=Geff,
                             zeros=torch.from_numpy(Z).cuda() if Z is not None else None,
                             packed=packed)
    torch.cuda.synchronize()
    st = g.stats_dict(st)
    B = Qb.cpu().numpy().astype(np.int64)
    if packed:
        codes = np.zeros((m, n), np.int64)
        codes[:, 0::2] = B[:, : (n + 1) // 2] & 15
        codes[:, 1::2] = (B[:, : n // 2] >> 4) & 15
    else:
        codes = B if Z is not None else Qb.cpu().numpy().astype(np.int8).astype(np.int64)
    col = np.arange(n) // (Geff or max(n, 1))
    if Z is not None:
        q = codes - Z.astype(np.int64)[:, col]
    elif packed:
        q = codes - (1 << (bits - 1))
    else:
        q = codes
    grid = O.expand_grid(m, n, S.astype(np.float64), bits, clamp, Geff, Z)
    rep = check_against_oracle(Wd, ML, MR, None, bits, clamp, q, grid=grid)
    assert st["status"] == 0
    assert st["n_clamped"] == rep.result.n_clamped
    assert st["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5, abs=1e-300)

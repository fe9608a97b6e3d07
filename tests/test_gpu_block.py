"""GPU tests of gptq2d_quantize_block: a block of layers whose factor preparation
overlaps the rounding of the previous layer (library-internal streams of their own,
two factor slots).  Every layer's Q and statistics must be bit-identical to that
layer alone through gptq2d_prepare_pair + gptq2d_quantize_grid (the same kernels in
the same order: deterministic), which the other GPU tests tie to the oracle; one layer
is also checked against the oracle directly.  A non-SPD factor is reported by layer.
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


def _spd(rng, k):
    return WL.damped_gram(WL.student_t_activations(rng, 4 * k, k))


def _layer(seed, m, n, kind):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.02, (m, n)).astype(np.float32)
    sp = {"W": torch.from_numpy(W).cuda().to(torch.bfloat16),
          "H_L": torch.from_numpy(_spd(rng, m)).cuda(), "H_R": torch.from_numpy(_spd(rng, n)).cuda()}
    Wd = sp["W"].double().cpu().numpy()
    if kind == "row":
        sp.update(scales=torch.from_numpy(WL.absmax_scales(Wd, 4)).cuda(), bits=4)
    elif kind == "asym_g32_packed":
        S, Z = WL.group_minmax_grid(Wd, 4, 32)
        sp.update(scales=torch.from_numpy(S).cuda(), zeros=torch.from_numpy(Z).cuda(), bits=4,
                  group_size=32, packed=True)
    else:  # symmetric INT3, groups of 16
        sp.update(scales=torch.from_numpy(WL.group_absmax_scales(Wd, 3, 16)).cuda(), bits=3,
                  group_size=16)
    return sp


def _alone(g, sp):
    ML, MR = g.prepare_pair(sp["H_L"], sp["H_R"])
    return g.quantize_grid(sp["W"], ML, MR, sp["scales"], sp.get("bits", 4), sp.get("clamp", True),
                           group_size=sp.get("group_size", 0), zeros=sp.get("zeros"),
                           packed=sp.get("packed", False))


def test_block_equals_layers_alone(g):
    specs = [_layer(1, 200, 330, "row"), _layer(2, 130, 96, "asym_g32_packed"),
             _layer(3, 64, 200, "sym_g16"), _layer(4, 33, 70, "row"), _layer(5, 150, 150, "row")]
    Qs, sts = g.quantize_block(specs)
    torch.cuda.synchronize()
    for sp, Q, st in zip(specs, Qs, sts):
        Qa, sta = _alone(g, sp)
        torch.cuda.synchronize()
        assert torch.equal(Q, Qa)
        assert torch.equal(st, sta)
        assert g.stats_dict(st)["status"] == 0
    # the first layer against the oracle as well
    sp = specs[0]
    sym = lambda H: np.tril(H) + np.tril(H, -1).T
    HL = sym(sp["H_L"].double().cpu().numpy())
    HR = sym(sp["H_R"].double().cpu().numpy())
    check_against_oracle(sp["W"].double().cpu().numpy(), O.reverse_cholesky(HL), O.reverse_cholesky(HR),
                         sp["scales"].double().cpu().numpy(), 4, True, Qs[0].cpu().numpy())


def test_single_layer_and_repeat_are_deterministic(g):
    specs = [_layer(7, 100, 70, "row")]
    Q1, s1 = g.quantize_block(specs)
    Q2, s2 = g.quantize_block(specs)
    torch.cuda.synchronize()
    assert torch.equal(Q1[0], Q2[0]) and torch.equal(s1[0], s2[0])


def test_empty_block(g):
    assert g.quantize_block([]) == ([], [])


@pytest.mark.parametrize("side", [0, 1])
def test_not_spd_factor_is_reported_by_layer(g, side):
    specs = [_layer(11, 80, 90, "row"), _layer(12, 70, 75, "row"), _layer(13, 66, 99, "row")]
    key = "H_L" if side == 0 else "H_R"
    H = specs[2][key].cpu().numpy().copy()
    H[5, 5] = -1.0
    specs[2][key] = torch.from_numpy(H).cuda()
    with pytest.raises(g.GPTQ2DError) as ei:
        g.quantize_block(specs)
    assert ei.value.status == g.Status.NOT_SPD
    assert f"layer 2 factor {side}" in str(ei.value)

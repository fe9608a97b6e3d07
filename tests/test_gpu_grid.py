"""GPU parity of the grid variants through gptq2d_quantize_grid: group-wise scales,
asymmetric grids with integer zero points, packed 4-bit output (the pages fix only
a 4-bit integer grid, mind-verse.de "Neue Ansätze ... durch GPTQ-2D", section
"Quantisierung von Large Language Models"; these are GPTQ's usual variants).

Bar: the integers q are bit-exact against the oracle with the same per-entry grid
(near-tie replay of tests/parity.py); the stored bytes are exactly the oracle's
codes (oracle.stored_codes / packed_codes / pack_nibbles); statistics as for the
per-row path; the per-row call of the same entry point equals gptq2d_quantize bit
for bit.
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


def dev(a, dtype=None):
    t = torch.from_numpy(np.array(a, order="C", copy=True))
    return (t.to(dtype) if dtype is not None else t).cuda()


def _problem(seed, m, n):
    pb = WL.small(seed, m=m, n=n)
    return (pb.W.astype(np.float32), O.reverse_cholesky(pb.H_L), O.reverse_cholesky(pb.H_R))


def _grid_inputs(W, bits, G, asym):
    if asym:
        S, Z = WL.group_minmax_grid(W, bits, G)
        return S, Z
    if G:
        return WL.group_absmax_scales(W, bits, G), None
    return WL.absmax_scales(W, bits)[:, None], None


def _q_from_bytes(Qb, m, n, bits, G, Z, packed):
    """Integers q from the stored bytes (unpacking written from the format)."""
    B = np.asarray(Qb).astype(np.int64)
    if packed:
        codes = np.zeros((m, n), np.int64)
        codes[:, 0::2] = B[:, : (n + 1) // 2] & 15
        codes[:, 1::2] = (B[:, : n // 2] >> 4) & 15
        if Z is None:
            return codes - (1 << (bits - 1)), codes
    else:
        codes = B if Z is not None else np.asarray(Qb).astype(np.int8).astype(np.int64)
        if Z is None:
            return codes, codes
    col = np.arange(n) // (G or n)
    return codes - np.asarray(Z, np.int64)[:, col], codes


CASES = [  # m, n, group size, asymmetric, bits, clamp, packed
    (100, 130, 32, False, 4, True, False),
    (100, 130, 32, True, 4, True, False),
    (100, 130, 32, True, 4, True, True),
    (77, 150, 8, True, 3, True, True),
    (77, 150, 8, False, 3, True, True),
    (130, 200, 40, True, 4, True, False),
    (64, 192, 128, True, 2, True, False),
    (90, 70, 0, True, 4, True, True),
    (90, 70, 70, False, 4, True, True),
    (60, 90, 16, False, 4, False, False),
    (129, 65, 24, True, 8, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "m%d_n%d_G%d_%s_b%d_%s_%s" % (
    c[0], c[1], c[2], "asym" if c[3] else "sym", c[4], "clamp" if c[5] else "free",
    "packed" if c[6] else "bytes"))
def test_grid_variant_matches_oracle(g, case):
    m, n, G, asym, bits, clamp, packed = case
    W, ML, MR = _problem(3 + m + n, m, n)
    S, Z = _grid_inputs(W.astype(np.float64), bits, G, asym)
    if not clamp:
        S = (S * 0.5).astype(np.float32)
    Qb, st = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(S), bits, clamp, group_size=G,
                             zeros=dev(Z) if Z is not None else None, packed=packed)
    torch.cuda.synchronize()
    st = g.stats_dict(st)
    q, codes = _q_from_bytes(Qb.cpu().numpy(), m, n, bits, G, Z, packed)
    grid = O.expand_grid(m, n, S.astype(np.float64), bits, clamp, G, Z)
    rep = check_against_oracle(W.astype(np.float64), ML, MR, None, bits, clamp, q, grid=grid)
    r = rep.result
    assert st["status"] == 0 and st["n_nonfinite"] == 0
    assert st["n_clamped"] == r.n_clamped
    assert abs(st["n_near_tie"] - rep.n_near_tie) <= len(rep.flips) + 2
    assert st["proxy_loss"] == pytest.approx(r.loss_identity, rel=1e-5)
    # the stored bytes are exactly the oracle's codes for the (replayed) trajectory
    if packed:
        expect = O.pack_nibbles(O.packed_codes(r.Q, m, n, bits, G, Z))
        np.testing.assert_array_equal(Qb.cpu().numpy(), expect)
    else:
        np.testing.assert_array_equal(codes, O.stored_codes(r.Q, m, n, bits, G, Z))


def test_per_row_grid_equals_quantize(g):
    W, ML, MR = _problem(1, 150, 140)
    s = WL.absmax_scales(W.astype(np.float64), 4)
    Q0, st0 = g.quantize(dev(W), dev(ML), dev(MR), dev(s), 4, True)
    Q1, st1 = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(s), 4, True)
    Q2, st2 = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(np.repeat(s[:, None], 3, 1)), 4, True,
                              group_size=64)
    torch.cuda.synchronize()
    for Q, st in ((Q1, st1), (Q2, st2)):
        assert torch.equal(Q0, Q)
        assert torch.equal(st0, st)


def test_packed_bytes_equal_packing_of_the_byte_output(g):
    W, ML, MR = _problem(2, 96, 101)
    S, Z = WL.group_minmax_grid(W.astype(np.float64), 4, 32)
    a = dict(group_size=32, zeros=dev(Z))
    Qb, _ = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(S), 4, True, **a)
    Qp, _ = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(S), 4, True, packed=True, **a)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Qp.cpu().numpy(), O.pack_nibbles(Qb.cpu().numpy()))


def test_bad_group_scale_is_reported(g):
    W, ML, MR = _problem(4, 70, 96)
    S = WL.group_absmax_scales(W.astype(np.float64), 4, 32)
    S[5, 1] = 0.0
    S[60, 2] = np.nan
    _, st = g.quantize_grid(dev(W), dev(ML), dev(MR), dev(S), 4, True, group_size=32)
    torch.cuda.synchronize()
    st = g.stats_dict(st)
    assert st["status"] == g.Status.NONFINITE and st["n_nonfinite"] >= 2


def _gpu_gram(X):
    Xt = torch.from_numpy(X).cuda()
    return (Xt.T @ Xt).cpu().numpy()


@pytest.mark.slow
def test_attention_layer_groupwise_asymmetric_packed_prefix(g):
    """The 4096 x 4096 INT4 layer with 128-column asymmetric groups and packed output,
    in the bench's launch configuration: the leading 320 x 256 block against the oracle
    (the prefix property: the dominated quadrant of an entry lies inside the prefix)."""
    pb = WL.attn(0, matmul=_gpu_gram)
    Wt = dev(pb.W).to(torch.bfloat16)
    Wd = Wt.double().cpu().numpy()
    S, Z = WL.group_minmax_grid(Wd, 4, 128)
    ML, MR = g.prepare_pair(torch.from_numpy(pb.H_L).cuda(), torch.from_numpy(pb.H_R).cuda())
    Qp, st = g.quantize_grid(Wt, ML, MR, dev(S), 4, True, group_size=128, zeros=dev(Z), packed=True)
    torch.cuda.synchronize()
    st = g.stats_dict(st)
    assert st["status"] == 0
    pm, pn = 320, 256
    q, _ = _q_from_bytes(Qp.cpu().numpy()[:pm, : pn // 2], pm, pn, 4, 128, Z[:pm, :2], True)
    MLc, MRc = ML.cpu().numpy(), MR.cpu().numpy()
    grid = O.expand_grid(pm, pn, S[:pm, :2].astype(np.float64), 4, True, 128, Z[:pm, :2])
    check_against_oracle(Wd[:pm, :pn], MLc[:pm, :pm], MRc[:pn, :pn], None, 4, True, q, grid=grid)

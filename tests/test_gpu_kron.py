"""GPU parity for Hessians with more than two Kronecker factors (arxivlens
"GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Abstract: the algorithm
extends to any number of Kronecker factors), through the C ABI.

The k-way tensor (m_1, ..., m_k) is rounded as the m_1 x (m_2...m_k) problem with
M_R = M_2 kron ... kron M_k (gptq2d_kron_factor).  Bar:
  * the Kronecker factor equals the oracle's (np.kron of the same factors) to
    fp64 rounding of a product of nf doubles (relative 1e-14), with exact zeros
    wherever a column digit exceeds the row digit;
  * Q is bit-exact against the k-way oracle (the reduced 2-D oracle with the
    near-tie replay of tests/parity.py; the CPU pins tie it to the hyperplane
    and naive-sweep oracles), the proxy loss within 1e-5 relative.
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
    X = WL.student_t_activations(rng, 4 * k, k)
    return WL.damped_gram(X).astype(np.float64)


def _case(seed, shape):
    rng = np.random.default_rng(5000 + 31 * seed + sum(shape) * 7 + len(shape))
    W = rng.normal(0, 0.02, shape).astype(np.float32)
    Hs = [_spd(rng, d) for d in shape]
    s = WL.absmax_scales(W.reshape(shape[0], -1).astype(np.float64), 4).astype(np.float32)
    return W, Hs, s


def _digits(x, dims):
    out = []
    for d in reversed(dims):
        out.append(x % d)
        x //= d
    return np.stack(out[::-1])


@pytest.mark.parametrize("dims", [(3, 4), (5, 2, 3), (2,) * 8, (64, 64), (1, 7), (13,)],
                         ids=lambda d: "x".join(map(str, d)))
def test_kron_factor_matches_oracle(g, dims):
    rng = np.random.default_rng(sum(dims))
    Ms = [O.reverse_cholesky(_spd(rng, d)) for d in dims]
    # fill the strict upper triangles with garbage: the kernel must not read them
    Mg = []
    for M in Ms:
        G = M + np.triu(rng.normal(0, 1, M.shape), 1)
        Mg.append(torch.from_numpy(G).cuda())
    K = g.kron_factor(Mg).cpu().numpy()
    Kref = O.kron_factor(Ms)
    n = Kref.shape[0]
    rd = _digits(np.arange(n)[:, None].repeat(n, 1), dims)
    cd = _digits(np.arange(n)[None, :].repeat(n, 0), dims)
    zero = np.any(cd > rd, axis=0)
    assert np.all(K[zero] == 0.0)
    np.testing.assert_allclose(K[~zero], Kref[~zero], rtol=1e-14, atol=0)


def test_kron_factor_rejects_bad_arguments(g):
    L = g.lib()
    import ctypes
    M = torch.eye(4, dtype=torch.float64, device="cuda")
    ptrs = (ctypes.c_void_p * 2)(M.data_ptr(), M.data_ptr())
    dims = (ctypes.c_int64 * 2)(4, 4)
    lds = (ctypes.c_int64 * 2)(4, 4)
    out = torch.empty((16, 16), dtype=torch.float64, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.gptq2d_kron_factor(2, ptrs, dims, lds, out.data_ptr(), 15, s) == g.Status.INVALID_ARG
    assert L.gptq2d_kron_factor(9, ptrs, dims, lds, out.data_ptr(), 16, s) == g.Status.INVALID_ARG
    # the output may not overlap a factor
    ptrs_alias = (ctypes.c_void_p * 2)(out.data_ptr(), M.data_ptr())
    assert L.gptq2d_kron_factor(2, ptrs_alias, dims, lds, out.data_ptr(), 16, s) == g.Status.INVALID_ARG
    assert L.gptq2d_kron_factor(2, ptrs, dims, lds, out.data_ptr(), 16, s) == g.Status.OK
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(), np.eye(16))


SHAPES = [(70, 9, 13), (33, 5, 7, 3), (130, 8, 8, 2), (1, 64, 3), (64, 1, 70),
          (40, 2, 2, 2, 2, 2, 2, 2), (97, 3, 41)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("bits,clamp", [(4, True), (3, True), (4, False)])
def test_kway_rounding_matches_oracle(g, shape, bits, clamp):
    W, Hs, s = _case(bits + 3 * clamp, shape)
    s = s if clamp else (s * 4).astype(np.float32)
    Ms = [O.reverse_cholesky(H) for H in Hs]
    # the k-way problem through the library: GPU Kronecker factor, GPU rounding
    MR = g.kron_factor([torch.from_numpy(M).cuda() for M in Ms[1:]]) if len(Ms) > 2 \
        else torch.from_numpy(Ms[1]).cuda()
    W2 = torch.from_numpy(W.reshape(shape[0], -1)).cuda()
    Q, st = g.quantize(W2, torch.from_numpy(Ms[0]).cuda(), MR,
                       torch.from_numpy(s).cuda(), bits, clamp)
    torch.cuda.synchronize()
    Qg = Q.cpu().numpy()
    st = g.stats_dict(st)
    s64 = s.astype(np.float64)
    rep = check_against_oracle(W.reshape(shape[0], -1).astype(np.float64), Ms[0],
                               O.kron_factor(Ms[1:]), s64, bits, clamp, Qg)
    assert st["status"] == 0
    assert st["n_clamped"] == rep.result.n_clamped
    assert st["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)
    if not rep.flips:
        # the k-way hyperplane oracle gives the same rounding
        rk = O.gptq_kron_hyperplane(W.astype(np.float64), Ms, s64, bits, clamp)
        np.testing.assert_array_equal(rk.Q.reshape(shape[0], -1), Qg)


def test_quantize_tensor_end_to_end(g):
    """prepare each mode's factor on the GPU, form M_R, round: the k-way tensor result."""
    shape = (96, 6, 11, 2)
    W, Hs, s = _case(11, shape)
    Q, st = g.quantize_tensor(torch.from_numpy(W).cuda(), [torch.from_numpy(H).cuda() for H in Hs],
                              torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    assert tuple(Q.shape) == shape
    Ms = [O.reverse_cholesky(H) for H in Hs]
    rep = check_against_oracle(W.reshape(shape[0], -1).astype(np.float64), Ms[0],
                               O.kron_factor(Ms[1:]), s.astype(np.float64), 4, True,
                               Q.cpu().numpy().reshape(shape[0], -1))
    assert g.stats_dict(st)["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)
    assert O.proxy_loss_tensor(W.astype(np.float64), Q.cpu().numpy(), s.astype(np.float64), Hs) == \
        pytest.approx(rep.result.loss_identity, rel=1e-6)


# The per-mode right factor (gptq2d_quantize_kron): trailing modes whose last sizes
# multiply to m_in in {8, 16, 32, 64}.  Shapes with one to four outer modes, a tile
# holding 1, 2, 4 or 8 outer indices, ragged last column and row tiles, and right
# feedback two or more tiles away (n >= 192).
PER_MODE = [(97, 16, 16), (70, 24, 32), (65, 3, 4, 16), (300, 6, 8, 8), (100, 12, 64),
            (48, 2, 3, 2, 8), (200, 5, 16), (33, 3, 8), (130, 8, 8, 2),
            (40, 2, 2, 2, 2, 2, 2, 2), (64, 4, 2), (130, 64)]


@pytest.mark.parametrize("shape", PER_MODE, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("bits,clamp", [(4, True), (3, True), (4, False)])
def test_per_mode_rounding_matches_oracle(g, shape, bits, clamp):
    assert g.kron_inner_size(shape[1:]) > 0
    W, Hs, s = _case(7 * bits + clamp, shape)
    s = s if clamp else (s * 4).astype(np.float32)
    Ms = [O.reverse_cholesky(H) for H in Hs]
    W2 = torch.from_numpy(W.reshape(shape[0], -1)).cuda()
    Q, st = g.quantize_kron(W2, torch.from_numpy(Ms[0]).cuda(),
                            [torch.from_numpy(M).cuda() for M in Ms[1:]],
                            torch.from_numpy(s).cuda(), bits, clamp)
    torch.cuda.synchronize()
    Qg = Q.cpu().numpy()
    st = g.stats_dict(st)
    s64 = s.astype(np.float64)
    rep = check_against_oracle(W.reshape(shape[0], -1).astype(np.float64), Ms[0],
                               O.kron_factor(Ms[1:]), s64, bits, clamp, Qg)
    assert st["status"] == 0
    assert st["n_clamped"] == rep.result.n_clamped
    assert st["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)
    if not rep.flips and len(shape) <= 4:
        rk = O.gptq_kron_hyperplane(W.astype(np.float64), Ms, s64, bits, clamp)
        np.testing.assert_array_equal(rk.Q.reshape(shape[0], -1), Qg)


def test_per_mode_equals_the_dense_kronecker_factor(g):
    """The two routes of the library agree entry for entry away from near-ties, and the
    per-mode one needs no n x n matrix: its workspace is smaller by n^2 doubles, less
    the inner factor's 64 x 64, at n = 768."""
    shape = (128, 12, 64)
    W, Hs, s = _case(3, shape)
    Ms = [torch.from_numpy(O.reverse_cholesky(H)).cuda() for H in Hs]
    W2 = torch.from_numpy(W.reshape(shape[0], -1)).cuda()
    sc = torch.from_numpy(s).cuda()
    Qk, stk = g.quantize_kron(W2, Ms[0], Ms[1:], sc, 4, True)
    Qd, std = g.quantize(W2, Ms[0], g.kron_factor(Ms[1:]), sc, 4, True)
    torch.cuda.synchronize()
    a, b = g.stats_dict(stk), g.stats_dict(std)
    diff = int((Qk != Qd).sum())
    assert diff <= a["n_near_tie"] + b["n_near_tie"]
    if diff == 0:
        assert a["proxy_loss"] == pytest.approx(b["proxy_loss"], rel=1e-12)
    n = 12 * 64
    assert g.quantize_workspace_size(128, n) - g.quantize_kron_workspace_size(128, [12, 64]) >= \
        8 * (n * n - 64 * 64)


def test_per_mode_rejects_shapes_it_does_not_cover(g):
    """A last mode of 3 (no suffix product of 8..64 dividing 64): INVALID_ARG, and the
    workspace query says 0; quantize_tensor then takes the dense route."""
    assert g.quantize_kron_workspace_size(16, [5, 3]) == 0
    shape = (16, 5, 3)
    W, Hs, s = _case(1, shape)
    Ms = [torch.from_numpy(O.reverse_cholesky(H)).cuda() for H in Hs]
    with pytest.raises(g.GPTQ2DError):
        g.quantize_kron(torch.from_numpy(W.reshape(16, -1)).cuda(), Ms[0], Ms[1:],
                        torch.from_numpy(s).cuda(), 4, True)
    Q, st = g.quantize_tensor(torch.from_numpy(W).cuda(), [torch.from_numpy(H).cuda() for H in Hs],
                              torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    assert g.stats_dict(st)["status"] == 0


def test_quantize_tensor_per_mode_end_to_end(g):
    """prepare each mode's factor on the GPU and round with the per-mode right factor
    (the default route for these modes): the k-way tensor result and its loss."""
    shape = (96, 6, 4, 16)
    assert g.kron_inner_size(shape[1:]) == 64
    W, Hs, s = _case(12, shape)
    Q, st = g.quantize_tensor(torch.from_numpy(W).cuda(), [torch.from_numpy(H).cuda() for H in Hs],
                              torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    Ms = [O.reverse_cholesky(H) for H in Hs]
    rep = check_against_oracle(W.reshape(shape[0], -1).astype(np.float64), Ms[0],
                               O.kron_factor(Ms[1:]), s.astype(np.float64), 4, True,
                               Q.cpu().numpy().reshape(shape[0], -1))
    assert g.stats_dict(st)["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)
    assert O.proxy_loss_tensor(W.astype(np.float64), Q.cpu().numpy(), s.astype(np.float64), Hs) == \
        pytest.approx(rep.result.loss_identity, rel=1e-6)


@pytest.mark.parametrize("wdt", ["bfloat16", "float64"])
def test_per_mode_weight_dtypes(g, wdt):
    """The per-mode sweep is instantiated per weight type: bf16 and fp64 W against the
    oracle on the same (upcast) weights."""
    shape = (97, 16, 16)
    W, Hs, s = _case(21, shape)
    Wt = torch.from_numpy(W.reshape(shape[0], -1)).to(getattr(torch, wdt)).cuda()
    W64 = Wt.double().cpu().numpy()
    Ms = [O.reverse_cholesky(H) for H in Hs]
    Q, st = g.quantize_kron(Wt, torch.from_numpy(Ms[0]).cuda(),
                            [torch.from_numpy(M).cuda() for M in Ms[1:]],
                            torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    rep = check_against_oracle(W64, Ms[0], O.kron_factor(Ms[1:]), s.astype(np.float64), 4, True,
                               Q.cpu().numpy())
    assert g.stats_dict(st)["status"] == 0
    assert g.stats_dict(st)["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)


def test_per_mode_zero_rows(g):
    """m = 0: nothing to round; the statistics are zero and the status OK."""
    Ms = [torch.eye(d, dtype=torch.float64, device="cuda") for d in (8, 8, 8)]
    W = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    s = torch.empty(0, dtype=torch.float32, device="cuda")
    Q, st = g.quantize_kron(W, torch.empty((0, 0), dtype=torch.float64, device="cuda"), Ms[1:],
                            s, 4, True)
    torch.cuda.synchronize()
    d = g.stats_dict(st)
    assert d["status"] == 0 and d["n_clamped"] == 0 and d["proxy_loss"] == 0.0


@pytest.mark.parametrize("shape", [(40, 32, 3), (24, 16, 128), (30, 64, 3, 3), (36, 5, 8, 8, 2)],
                         ids=lambda s: "x".join(map(str, s)))
def test_quantize_tensor_reorders_trailing_modes(g, shape):
    """Trailing modes whose given order has no inner group of 8..64 (a last mode of 3
    or 128) are rounded with the eligible modes moved last; the result, put back in
    W's order, is the oracle's rounding of the original order (the rounding depends
    only on each entry's dominated orthant)."""
    order = g.per_mode_order(shape[1:])
    assert order is not None and order != list(range(len(shape) - 1))
    W, Hs, s = _case(31, shape)
    Q, st = g.quantize_tensor(torch.from_numpy(W).cuda(), [torch.from_numpy(H).cuda() for H in Hs],
                              torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    assert tuple(Q.shape) == shape
    Ms = [O.reverse_cholesky(H) for H in Hs]
    rep = check_against_oracle(W.reshape(shape[0], -1).astype(np.float64), Ms[0],
                               O.kron_factor(Ms[1:]), s.astype(np.float64), 4, True,
                               Q.cpu().numpy().reshape(shape[0], -1))
    d = g.stats_dict(st)
    assert d["status"] == 0
    assert d["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)


KRON_GRID = [  # tensor shape, group size, asymmetric, bits, packed
    ((70, 24, 32), 32, True, 4, True),
    ((65, 3, 4, 16), 64, False, 4, False),
    ((97, 16, 16), 16, True, 3, False),
    ((48, 2, 3, 2, 8), 8, True, 4, True),
]


@pytest.mark.parametrize("case", KRON_GRID, ids=lambda c: "x".join(map(str, c[0])) + "_G%d_%s_b%d_%s" % (
    c[1], "asym" if c[2] else "sym", c[3], "packed" if c[4] else "bytes"))
def test_per_mode_grid_variant_matches_oracle(g, case):
    """gptq2d_quantize_kron_grid: group-wise scales along the flattened trailing modes,
    integer zero points and packed 4-bit codes on the per-mode route, against the
    oracle's rounding with the same per-entry grid; the stored bytes are the oracle's
    codes."""
    shape, G, asym, bits, packed = case
    W, Hs, _ = _case(41, shape)
    m, n = shape[0], int(np.prod(shape[1:]))
    W2 = W.reshape(m, n).astype(np.float64)
    if asym:
        S, Z = WL.group_minmax_grid(W2, bits, G)
    else:
        S, Z = WL.group_absmax_scales(W2, bits, G), None
    Ms = [O.reverse_cholesky(H) for H in Hs]
    Qb, st = g.quantize_kron(torch.from_numpy(W.reshape(m, n)).cuda(), torch.from_numpy(Ms[0]).cuda(),
                             [torch.from_numpy(M).cuda() for M in Ms[1:]],
                             torch.from_numpy(np.ascontiguousarray(S, np.float32)).cuda(), bits, True,
                             group_size=G, zeros=torch.from_numpy(Z).cuda() if Z is not None else None,
                             packed=packed)
    torch.cuda.synchronize()
    B = Qb.cpu().numpy().astype(np.int64)
    if packed:
        codes = np.zeros((m, n), np.int64)
        codes[:, 0::2] = B[:, : (n + 1) // 2] & 15
        codes[:, 1::2] = (B[:, : n // 2] >> 4) & 15
        q = codes - (1 << (bits - 1)) if Z is None else codes - np.asarray(Z, np.int64)[:, np.arange(n) // G]
    else:
        codes = B if Z is not None else Qb.cpu().numpy().astype(np.int8).astype(np.int64)
        q = codes if Z is None else codes - np.asarray(Z, np.int64)[:, np.arange(n) // G]
    grid = O.expand_grid(m, n, S.astype(np.float64), bits, True, G, Z)
    rep = check_against_oracle(W2, Ms[0], O.kron_factor(Ms[1:]), None, bits, True, q, grid=grid)
    d = g.stats_dict(st)
    assert d["status"] == 0 and d["n_nonfinite"] == 0
    assert d["n_clamped"] == rep.result.n_clamped
    assert d["proxy_loss"] == pytest.approx(rep.result.loss_identity, rel=1e-5)
    if packed:
        np.testing.assert_array_equal(Qb.cpu().numpy(),
                                      O.pack_nibbles(O.packed_codes(rep.result.Q, m, n, bits, G, Z)))
    else:
        np.testing.assert_array_equal(codes, O.stored_codes(rep.result.Q, m, n, bits, G, Z))


@pytest.mark.parametrize("shape,route", [((70, 24, 32), "per-mode"), ((40, 6, 11, 2), "dense")])
def test_quantize_tensor_grid_routes(g, shape, route):
    """quantize_tensor with group-wise asymmetric INT4 scales: the per-mode route where
    the given order allows it, the dense one otherwise; both equal the other route's
    direct call and the oracle's rounding on the same grid."""
    W, Hs, _ = _case(51, shape)
    m, n = shape[0], int(np.prod(shape[1:]))
    W2 = W.reshape(m, n).astype(np.float64)
    G = 8 if n % 8 == 0 else n
    S, Z = WL.group_minmax_grid(W2, 4, G)
    args = dict(group_size=G, zeros=torch.from_numpy(Z).cuda())
    Q, st = g.quantize_tensor(torch.from_numpy(W).cuda(), [torch.from_numpy(H).cuda() for H in Hs],
                              torch.from_numpy(np.ascontiguousarray(S, np.float32)).cuda(), 4, True,
                              **args)
    torch.cuda.synchronize()
    assert (g.kron_inner_size(shape[1:]) > 0) == (route == "per-mode")
    codes = Q.cpu().numpy().reshape(m, n).astype(np.int64)
    q = codes - np.asarray(Z, np.int64)[:, np.arange(n) // G]
    Ms = [O.reverse_cholesky(H) for H in Hs]
    grid = O.expand_grid(m, n, S.astype(np.float64), 4, True, G, Z)
    rep = check_against_oracle(W2, Ms[0], O.kron_factor(Ms[1:]), None, 4, True, q, grid=grid)
    assert g.stats_dict(st)["status"] == 0
    np.testing.assert_array_equal(codes, O.stored_codes(rep.result.Q, m, n, 4, G, Z))


@pytest.mark.slow
def test_per_mode_4096x64x64_every_entry(g):
    """The per-mode route at full size (the kron3 bench's 4096 x 64 x 64 tensor, INT4,
    bf16 weights): every one of the 16.8 M entries is the rounding of its own y computed
    from the GPU's integers with the dense Kronecker factor (tests/parity.py fixed
    point), and the in-kernel loss equals the oracle's identity from the same check."""
    from tests.parity import check_fixed_point
    rng = np.random.default_rng(4096)
    dims = (4096, 64, 64)
    Hs = [_spd(rng, d) for d in dims]
    W = rng.normal(0, 0.02, dims).astype(np.float32)
    m, n = 4096, 4096
    Wb = torch.from_numpy(W.reshape(m, n)).to(torch.bfloat16)
    W64 = Wb.double().numpy()
    s = WL.absmax_scales(W64, 4).astype(np.float32)
    Ms = [O.reverse_cholesky(H) for H in Hs]
    Q, st = g.quantize_kron(Wb.cuda(), torch.from_numpy(Ms[0]).cuda(),
                            [torch.from_numpy(M).cuda() for M in Ms[1:]],
                            torch.from_numpy(s).cuda(), 4, True)
    torch.cuda.synchronize()
    d = g.stats_dict(st)
    assert d["status"] == 0
    rep = check_fixed_point(W64, Ms[0], O.kron_factor(Ms[1:]), s.astype(np.float64), 4, True,
                            Q.cpu().numpy())
    assert rep.n_entries == m * n
    print(f"per-mode 4096x64x64: {rep.n_entries} entries checked, near-ties {rep.n_near_tie} "
          f"(GPU counted {d['n_near_tie']}), other neighbour taken at {rep.n_other_neighbour}")

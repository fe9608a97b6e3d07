"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
entry point declared in include/gptq2d.h, sizes workspaces, and rejects invalid
arguments before enqueuing anything."""
import ctypes
import os
import re

import pytest

import two_sided_adaptive_b200 as g
from two_sided_adaptive_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    return g.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "gptq2d.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq2d_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("gptq2d_prepare", "gptq2d_quantize", "gptq2d_round_host",
                 "gptq2d_prepare_workspace_size", "gptq2d_quantize_workspace_size"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(0, 8):
        assert L.gptq2d_status_string(code).startswith(b"GPTQ2D_")
    assert b"unknown" in L.gptq2d_status_string(99)


def test_version_and_counter(L):
    assert L.gptq2d_version() >> 16 == 1
    assert g.launch_count() >= 0


def test_workspace_sizes(L):
    assert g.prepare_workspace_size(4096) >= 8
    ws = g.quantize_workspace_size(4096, 4096)
    assert ws >= 3 * 4096 * 4096 * 8              # P, E and the errors, fp64
    assert g.quantize_workspace_size(100, 70) >= 3 * 128 * 128 * 8  # padded to 64-tiles
    assert g.quantize_workspace_size(-1, 5) == 0
    assert g.quantize_workspace_size(0, 5) > 0
    assert g.round_host_workspace_size(64, 64, g.DTYPE_F32, g.DTYPE_F32) > g.quantize_workspace_size(64, 64)
    assert g.round_host_workspace_size(64, 64, 9, g.DTYPE_F32) == 0


def _q(L, **kw):
    a = dict(W=16, wdt=0, m=4, n=4, ldw=4, ML=16, ldl=4, MR=16, ldr=4, s=16, bits=4, clamp=1,
             Q=16, ldq=4, st=16, ws=256, wsb=1 << 30, stream=None)
    a.update(kw)
    return L.gptq2d_quantize(a["W"], a["wdt"], a["m"], a["n"], a["ldw"], a["ML"], a["ldl"], a["MR"],
                             a["ldr"], a["s"], a["bits"], a["clamp"], a["Q"], a["ldq"], a["st"],
                             a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("bad", [dict(bits=1), dict(bits=9), dict(clamp=2), dict(wdt=7),
                                 dict(ldw=3), dict(ldl=3), dict(ldr=2), dict(ldq=1), dict(m=-1),
                                 dict(W=None), dict(ML=None), dict(MR=None), dict(s=None),
                                 dict(Q=None), dict(st=None), dict(m=1 << 21)])
def test_quantize_rejects_invalid_arguments(L, bad):
    assert _q(L, **bad) == g.Status.INVALID_ARG


@pytest.mark.parametrize("bad", [dict(ws=None), dict(ws=272), dict(wsb=100)])
def test_quantize_rejects_bad_workspace(L, bad):
    assert _q(L, **bad) == g.Status.WORKSPACE


def test_prepare_rejects_invalid_arguments(L):
    piv = ctypes.c_int64(0)
    P = L.gptq2d_prepare
    assert P(16, 1, 4, 4, 32, 4, 256, 256, None, None) == g.Status.INVALID_ARG   # bf16 H
    assert P(16, 0, -1, 4, 32, 4, 256, 256, None, None) == g.Status.INVALID_ARG
    assert P(16, 0, 4, 3, 32, 4, 256, 256, None, None) == g.Status.INVALID_ARG
    assert P(16, 0, 4, 4, 32, 3, 256, 256, None, None) == g.Status.INVALID_ARG
    assert P(None, 0, 4, 4, 32, 4, 256, 256, None, None) == g.Status.INVALID_ARG
    assert P(16, 0, 4, 4, 16, 4, 256, 256, None, None) == g.Status.INVALID_ARG   # M aliases H
    assert P(16, 0, 4, 4, 32, 4, 264, 256, None, None) == g.Status.WORKSPACE    # misaligned
    assert P(16, 0, 4, 4, 32, 4, 256, 0, None, None) == g.Status.WORKSPACE
    assert P(16, 0, 0, 0, 32, 0, 256, 256, None, ctypes.byref(piv)) == g.Status.OK and piv.value == -1


def test_round_host_rejects_invalid_arguments(L):
    R = L.gptq2d_round_host
    args = [16, 0, 8, 8, 16, 16, 0, 16, 4, 1, 16, 16, 256, 1 << 30, None, None, None]
    assert R(*args[:6], 1, *args[7:]) == g.Status.INVALID_ARG      # bf16 factors
    assert R(*args[:2], 0, *args[3:]) == g.Status.INVALID_ARG      # m = 0
    assert R(*args[:8], 1, *args[9:]) == g.Status.INVALID_ARG      # bits = 1
    assert R(*args[:12], 256, 10, *args[14:]) == g.Status.WORKSPACE


def test_wait_timeout_check_rejects_limits_out_of_range(L):
    # argument checks come before any CUDA call
    for bad in (0, 999, 10_000_000_001, -5):
        assert L.gptq2d_check_wait_timeout(ctypes.c_int64(bad), None) == 1  # INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(g, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(g, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        g.lib()


def _kron(L, nf=2, ptrs=(4096, 8192), dims=(4, 4), lds=(4, 4), out=1 << 20, ldo=16):
    P = (ctypes.c_void_p * len(ptrs))(*ptrs) if ptrs is not None else None
    D = (ctypes.c_int64 * len(dims))(*dims) if dims is not None else None
    S = (ctypes.c_int64 * len(lds))(*lds) if lds is not None else None
    return L.gptq2d_kron_factor(nf, P, D, S, out, ldo, None)


@pytest.mark.parametrize("bad", [dict(nf=0), dict(nf=9), dict(ptrs=None), dict(dims=None),
                                 dict(lds=None), dict(dims=(4, -1)), dict(lds=(3, 4)),
                                 dict(ldo=15), dict(out=None), dict(dims=(1 << 11, 1 << 10)),
                                 dict(ptrs=(4096, 0)), dict(out=4096 + 8)])
def test_kron_factor_rejects_invalid_arguments(L, bad):
    """Checked on the host before anything is enqueued (no GPU needed): factor count,
    null arrays, sizes, leading dimensions, n = prod dims <= 2^20, an output that
    overlaps a factor."""
    assert _kron(L, **bad) == g.Status.INVALID_ARG


def test_kron_factor_with_a_zero_dimension_is_a_no_op(L):
    assert _kron(L, dims=(4, 0), out=None) == g.Status.OK


def _qg(L, grid=None, **kw):
    gr = dict(bits=4, clamp=1, group_size=0, scales=16, ld_scales=1, zeros=None, packed=0)
    gr.update(grid or {})
    a = dict(W=16, wdt=0, m=4, n=20, ldw=20, ML=16, ldl=4, MR=16, ldr=20, Q=16, ldq=20, st=16,
             ws=256, wsb=1 << 30)
    a.update(kw)
    G = g._Grid(**gr)  # the binding's gptq2d_grid layout
    return L.gptq2d_quantize_grid(a["W"], a["wdt"], a["m"], a["n"], a["ldw"], a["ML"], a["ldl"],
                                  a["MR"], a["ldr"], ctypes.byref(G), a["Q"], a["ldq"], a["st"],
                                  a["ws"], a["wsb"], None)


@pytest.mark.parametrize("grid,kw", [
    (dict(bits=5, packed=1), {}),                 # packed needs bits <= 4
    (dict(clamp=0, packed=1), {}),                # and a clamped grid
    (dict(packed=2), {}),
    (dict(group_size=12), {}),                    # groups: multiples of 8 (or >= n)
    (dict(group_size=-8), {}),
    (dict(group_size=8, ld_scales=2), {}),        # 20 columns in groups of 8: 3 per row
    (dict(scales=None), {}),
    (dict(packed=1), dict(ldq=9)),                # packed rows need ceil(20 / 2) bytes
    (dict(), dict(ldq=19)),
    (dict(bits=1), {}),
    (dict(zeros=4096, clamp=0), {}),              # zero points need a clamped grid
])
def test_quantize_grid_rejects_invalid_arguments(L, grid, kw):
    assert _qg(L, grid, **kw) == g.Status.INVALID_ARG


def test_quantize_grid_rejects_a_null_grid(L):
    assert L.gptq2d_quantize_grid(16, 0, 4, 4, 4, 16, 4, 16, 4, None, 16, 4, 16, 256, 1 << 30,
                                  None) == g.Status.INVALID_ARG


def _ga(L, **kw):
    a = dict(X=4096, dt=g.DTYPE_BF16, rows=16, k=64, ldx=64, H=8192, ldh=64, acc=0, ws=256, wsb=256)
    a.update(kw)
    return L.gptq2d_gram_accumulate(a["X"], a["dt"], a["rows"], a["k"], a["ldx"], a["H"], a["ldh"],
                                    a["acc"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("bad", [dict(dt=g.DTYPE_F32), dict(k=60, ldx=64, ldh=64), dict(ldx=68),
                                 dict(ldx=60), dict(X=4096 + 8), dict(H=None), dict(ldh=63),
                                 dict(acc=2), dict(rows=-1), dict(X=None), dict(rows=2 ** 31)])
def test_gram_accumulate_rejects_invalid_arguments(L, bad):
    """Checked on the host: bf16 only, k and ldx multiples of 8, a 16-byte aligned X,
    rows that fit the 32-bit TMA row coordinate."""
    assert _ga(L, **bad) == g.Status.INVALID_ARG


@pytest.mark.parametrize("bad,code", [(dict(ws=None), "WORKSPACE"), (dict(wsb=255), "WORKSPACE"),
                                      (dict(ws=272), "WORKSPACE")])
def test_gram_accumulate_rejects_bad_workspace(L, bad, code):
    assert _ga(L, **bad) == getattr(g.Status, code)


def test_gram_finalize_rejects_invalid_arguments(L):
    f = L.gptq2d_gram_finalize
    assert f(8192, 64, 64, 0, 0.01, 256, 256, None, None) == g.Status.INVALID_ARG     # no rows
    assert f(8192, 64, 64, 10, -0.5, 256, 256, None, None) == g.Status.INVALID_ARG    # damp < 0
    assert f(8192, 64, 63, 10, 0.01, 256, 256, None, None) == g.Status.INVALID_ARG    # ldh < k
    assert f(8192, 64, 64, 10, 0.01, 0, 256, None, None) == g.Status.WORKSPACE
    assert L.gptq2d_gram_workspace_size() >= 12


def test_block_rejects_invalid_arguments(L):
    """Checked on the host before anything is enqueued."""
    assert L.gptq2d_quantize_block(None, -1, None, 0, None, None, None, None) == g.Status.INVALID_ARG
    assert L.gptq2d_quantize_block(None, 2, None, 0, None, None, None, None) == g.Status.INVALID_ARG
    assert L.gptq2d_quantize_block(None, 0, None, 0, None, None, None, None) == g.Status.OK
    lay = (g._Layer * 1)()
    lay[0] = g._Layer(4096, g.DTYPE_BF16, 64, 64, 64, 8192, 64, 8192, 64, 7,   # bad Gram dtype
                      g._Grid(4, 1, 0, 16, 1, None, 0), 16, 64, 16)
    assert L.gptq2d_quantize_block(lay, 1, 256, 1 << 40, None, None, None, None) == g.Status.INVALID_ARG
    lay[0].h_dtype = g.DTYPE_F32
    lay[0].ldhl = 63
    assert L.gptq2d_quantize_block(lay, 1, 256, 1 << 40, None, None, None, None) == g.Status.INVALID_ARG
    lay[0].ldhl = 64
    lay[0].grid.bits = 9
    assert L.gptq2d_quantize_block(lay, 1, 256, 1 << 40, None, None, None, None) == g.Status.INVALID_ARG
    lay[0].grid.bits = 4
    assert L.gptq2d_quantize_block(lay, 1, 256, 10, None, None, None, None) == g.Status.WORKSPACE
    assert L.gptq2d_block_workspace_size(lay, 1) >= 2 * 2 * 64 * 64 * 8


def test_proxy_loss_workspace_size(L):
    assert L.gptq2d_proxy_loss_workspace_size(-1, 4) == 0
    assert L.gptq2d_proxy_loss_workspace_size(0, 5) == 256
    # two tile-padded fp64 buffers and one double per 64 x 64 tile
    assert L.gptq2d_proxy_loss_workspace_size(100, 70) == 2 * 128 * 128 * 8 + 256


@pytest.mark.parametrize("bad", [
    dict(m=-1), dict(bits=1), dict(bits=9), dict(clamp=2), dict(W=None), dict(scales=None),
    dict(ML=None), dict(ldw=5), dict(ldl=9), dict(ldr=5), dict(Q=16, ldq=3), dict(loss=None),
    dict(w_dtype=7)])
def test_proxy_loss_rejects_invalid_arguments(L, bad):
    a = dict(W=16, w_dtype=0, m=10, n=6, ldw=6, Q=None, ldq=6, scales=16, bits=4, clamp=1,
             ML=16, ldl=10, MR=16, ldr=6, loss=16, ws=256, ws_bytes=1 << 20)
    a.update(bad)
    assert L.gptq2d_proxy_loss(a["W"], a["w_dtype"], a["m"], a["n"], a["ldw"], a["Q"], a["ldq"],
                               a["scales"], a["bits"], a["clamp"], a["ML"], a["ldl"], a["MR"],
                               a["ldr"], a["loss"], a["ws"], a["ws_bytes"], None) == \
        g.Status.INVALID_ARG


@pytest.mark.parametrize("ws, nbytes", [(None, 1 << 20), (256 + 8, 1 << 20), (256, 1000)])
def test_proxy_loss_rejects_bad_workspace(L, ws, nbytes):
    assert L.gptq2d_proxy_loss(16, 0, 10, 6, 6, None, 6, 16, 4, 1, 16, 10, 16, 6, 16, ws, nbytes,
                               None) == g.Status.WORKSPACE


def _qk(L, dims=(16, 16), nf=None, ws_bytes=None, **kw):
    """gptq2d_quantize_kron with fake (never dereferenced) pointers: host checks only."""
    nf = len(dims) if nf is None else nf
    n = 1
    for d in dims:
        n *= d
    a = dict(W=4096, dt=g.DTYPE_F32, m=32, ldw=n, ML=8192, ldl=32, S=12288,
             bits=4, clamp=1, Q=16384, ldq=n, st=20480, ws=256)
    a.update(kw)
    k = max(len(dims), 1)
    ptrs = (ctypes.c_void_p * k)(*([24576] * k))
    da = (ctypes.c_int64 * k)(*dims)
    lds = (ctypes.c_int64 * k)(*dims)
    wsb = L.gptq2d_quantize_kron_workspace_size(a["m"], len(dims), da) if ws_bytes is None else ws_bytes
    return L.gptq2d_quantize_kron(a["W"], a["dt"], a["m"], a["ldw"], a["ML"], a["ldl"], nf, ptrs,
                                  da, lds, a["S"], a["bits"], a["clamp"], a["Q"], a["ldq"], a["st"],
                                  a["ws"], wsb, None)


def test_quantize_kron_workspace_size(L):
    """Zero when the per-mode path does not apply or the sizes are out of range; else it
    omits the n x n normalised right factor of the dense route."""
    ws = lambda m, dims: L.gptq2d_quantize_kron_workspace_size(
        m, len(dims), (ctypes.c_int64 * len(dims))(*dims))
    assert ws(64, [5, 3]) == 0        # suffix products 3, 15: none divides 64 and is >= 8
    assert ws(64, [128]) == 0         # 128 does not divide 64
    assert ws(64, [4]) == 0           # 4 < 8
    assert ws(64, [0]) == 0
    assert ws(64, [2 ** 11, 2 ** 10]) == 0  # more than 2^20 columns
    assert ws(64, [3, 8]) > 0 and ws(64, [64, 64]) > 0
    n = 64 * 64
    # the dense route's n x n right factor against the inner factor's 64 x 64
    assert L.gptq2d_quantize_workspace_size(64, n) - ws(64, [64, 64]) >= 8 * (n * n - 64 * 64)


@pytest.mark.parametrize("kw,code", [
    (dict(nf=0), "INVALID_ARG"), (dict(nf=9), "INVALID_ARG"),
    (dict(dims=(5, 3)), "INVALID_ARG"),             # the per-mode path does not apply
    (dict(bits=9), "INVALID_ARG"), (dict(clamp=2), "INVALID_ARG"),
    (dict(ldw=255), "INVALID_ARG"), (dict(ldl=31), "INVALID_ARG"), (dict(ldq=10), "INVALID_ARG"),
    (dict(W=None), "INVALID_ARG"), (dict(st=None), "INVALID_ARG"), (dict(dt=7), "INVALID_ARG"),
    (dict(ws_bytes=1024), "WORKSPACE"), (dict(ws=None), "WORKSPACE"), (dict(ws=272), "WORKSPACE"),
])
def test_quantize_kron_rejects_invalid_arguments(L, kw, code):
    assert _qk(L, **kw) == getattr(g.Status, code)


def test_quantize_kron_checks_pointers_before_any_launch(L):
    """Valid sizes but host addresses: rejected as INVALID_ARG by the device-pointer
    check (nothing is launched)."""
    assert _qk(L) == g.Status.INVALID_ARG


def test_per_mode_order_moves_an_inner_group_last():
    """The chosen order of the trailing modes ends in modes whose sizes multiply to the
    largest of 64, 32, 16, 8 any subset reaches (checked by brute force), keeps the
    other modes' order, and keeps the given order when it already reaches it."""
    import itertools
    cases = [[64, 64], [32, 128], [3, 3, 64], [3, 3, 256], [24, 5], [16, 128], [2, 128],
             [5, 3], [8, 8, 2], [6, 4, 16], [12, 64], [64, 12], [3, 41], [2] * 7, [1, 7, 4, 2]]
    for dims in cases:
        best = 0
        for r in range(1, len(dims) + 1):
            for sel in itertools.combinations(range(len(dims)), r):
                p = 1
                for i in sel:
                    p *= dims[i]
                if p in (8, 16, 32, 64):
                    best = max(best, p)
        order = g.per_mode_order(dims)
        if best == 0:
            assert order is None, dims
            continue
        assert sorted(order) == list(range(len(dims)))
        assert g.kron_inner_size([dims[i] for i in order]) == best, (dims, order)
        if g.kron_inner_size(dims) == best:
            assert order == list(range(len(dims)))


def test_per_mode_eligibility_agrees_between_library_and_binding():
    """The library's workspace query (0 when the per-mode path does not apply) and the
    binding's kron_inner_size agree on every trailing-mode list up to three modes of
    sizes 1..12, 16, 32, 64, 100, 128."""
    import itertools
    sizes = list(range(1, 13)) + [16, 32, 64, 100, 128]
    for k in (1, 2, 3):
        for dims in itertools.product(sizes, repeat=k):
            if k == 3 and (dims[0] > 4 or dims[1] > 8):
                continue  # keep the sweep small
            arr = (ctypes.c_int64 * k)(*dims)
            lib_ok = L_global().gptq2d_quantize_kron_workspace_size(16, k, arr) > 0
            assert lib_ok == (g.kron_inner_size(dims) > 0), dims


def L_global():
    return g.lib()


def test_library_per_mode_order_equals_the_binding():
    """gptq2d_per_mode_order (C, host only) returns the binding's order and the inner
    size that order gives, on every list up to three modes of sizes 1..12, 16, 32, 64,
    100, 128; invalid arguments give -1."""
    import itertools
    L = g.lib()
    sizes = list(range(1, 13)) + [16, 32, 64, 100, 128]
    for k in (1, 2, 3):
        for dims in itertools.product(sizes, repeat=k):
            if k == 3 and (dims[0] > 4 or dims[1] > 8):
                continue
            da = (ctypes.c_int64 * k)(*dims)
            oa = (ctypes.c_int * k)()
            r = L.gptq2d_per_mode_order(k, da, oa)
            want = g.per_mode_order(list(dims))
            if want is None:
                assert r == 0 and list(oa) == list(range(k)), dims
            else:
                assert list(oa) == want, (dims, list(oa), want)
                assert r == g.kron_inner_size([dims[i] for i in want]), dims
    oa = (ctypes.c_int * 2)()
    assert L.gptq2d_per_mode_order(0, (ctypes.c_int64 * 1)(8), oa) == -1
    assert L.gptq2d_per_mode_order(2, (ctypes.c_int64 * 2)(8, 0), oa) == -1
    assert L.gptq2d_per_mode_order(2, None, oa) == -1

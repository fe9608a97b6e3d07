"""gptq2d_quantize_noalloc, the rounding entry point for callers that cannot allocate
device memory (it uses the library's static device scratch instead of a caller
workspace).  Called through the C ABI and compared with gptq2d_quantize, the entry
point that takes a workspace, on consecutive calls with different problems, so that
scratch left behind by one call cannot leak into the next.

Kept in a file that pytest collects last: it shares one static array across calls.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
import workloads as WL
from tests.parity import check_against_oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-5


@pytest.fixture(scope="module")
def g():
    from two_sided_adaptive_b200 import build as gbuild
    gbuild.build()
    import two_sided_adaptive_b200 as g
    return g


def _dev(a):
    return torch.from_numpy(np.array(a, order="C", copy=True)).cuda()


def _noalloc(g, W, ML, MR, s, bits, clamp):
    """Direct C-ABI call of gptq2d_quantize_noalloc on the current torch stream."""
    m, n = W.shape
    Q = torch.full((m, n), 99, dtype=torch.int8, device="cuda")
    st = torch.full((g.STATS_WORDS,), -7, dtype=torch.int64, device="cuda")
    rc = g.lib().gptq2d_quantize_noalloc(
        W.data_ptr(), g._dtype_code(W), m, n, W.stride(0), ML.data_ptr(), ML.stride(0),
        MR.data_ptr(), MR.stride(0), s.data_ptr(), bits, int(clamp), Q.data_ptr(), n,
        st.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == g.Status.OK, g.lib().gptq2d_status_string(rc)
    torch.cuda.synchronize()
    return Q, st


def test_noalloc_matches_workspace_entry_point(g):
    problems = [WL.small(0, 320, 256), WL.small(1, 130, 449), WL.small(0, 320, 256)]
    for k, pb in enumerate(problems):
        W, s = _dev(pb.W), _dev(pb.scales)
        ML = g.prepare(_dev(pb.H_L))
        MR = g.prepare(_dev(pb.H_R))
        Qw, stw = g.quantize(W, ML, MR, s, pb.bits, pb.clamp)
        Qn, stn = _noalloc(g, W, ML, MR, s, pb.bits, pb.clamp)
        assert torch.equal(Qn, Qw), f"call {k}: Q differs from gptq2d_quantize"
        dn, dw = g.stats_dict(stn), g.stats_dict(stw)
        assert dn["proxy_loss"] == pytest.approx(dw["proxy_loss"], rel=LOSS_RTOL)
        assert {k2: dn[k2] for k2 in dn if k2 != "proxy_loss"} == \
               {k2: dw[k2] for k2 in dw if k2 != "proxy_loss"}
    # and the first problem against the fp64 oracle
    pb = problems[0]
    check_against_oracle(pb.W.astype(np.float64), O.reverse_cholesky(pb.H_L),
                         O.reverse_cholesky(pb.H_R), pb.scales.astype(np.float64), pb.bits,
                         pb.clamp, Qn.cpu().numpy())


def test_noalloc_call_allocates_no_device_memory(g):
    """After a first call on the device (which resolves the scratch address and loads the
    library's kernels), further calls leave both torch's allocator and the device's free
    memory untouched: the scratch is the static array, the outputs are the caller's."""
    pb = WL.small(2, 200, 136)
    W, s = _dev(pb.W), _dev(pb.scales)
    ML, MR = g.prepare(_dev(pb.H_L)), g.prepare(_dev(pb.H_R))
    m, n = W.shape
    Q = torch.empty((m, n), dtype=torch.int8, device="cuda")
    st = torch.empty((g.STATS_WORDS,), dtype=torch.int64, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        rc = g.lib().gptq2d_quantize_noalloc(
            W.data_ptr(), g._dtype_code(W), m, n, W.stride(0), ML.data_ptr(), ML.stride(0),
            MR.data_ptr(), MR.stride(0), s.data_ptr(), pb.bits, int(pb.clamp), Q.data_ptr(), n,
            st.data_ptr(), stream)
        assert rc == g.Status.OK, g.lib().gptq2d_status_string(rc)

    call()
    torch.cuda.synchronize()
    Q0 = Q.clone()
    before_torch = torch.cuda.memory_stats()["allocation.all.allocated"]
    before_free = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    assert torch.cuda.memory_stats()["allocation.all.allocated"] == before_torch
    assert torch.cuda.mem_get_info()[0] == before_free
    assert torch.equal(Q, Q0)


def test_noalloc_rejects_problems_beyond_the_static_scratch(g):
    cap = 48 << 20
    assert g.quantize_workspace_size(1024, 1024) <= cap < g.quantize_workspace_size(2048, 2048)
    rc = g.lib().gptq2d_quantize_noalloc(16, 0, 2048, 2048, 2048, 16, 2048, 16, 2048, 16, 4, 1,
                                         16, 2048, 16, None)
    assert rc == g.Status.WORKSPACE

"""Python binding of libgptq2d, the sm_100a GPTQ-2D two-sided adaptive rounding library.

Thin ctypes layer over the C ABI in ``include/gptq2d.h``: it turns torch tensors
into raw device pointers, sizes and the current CUDA stream, allocates outputs
and workspaces with torch, and raises on a non-OK status.  Every step of the
path runs in the library's CUDA kernels; there is no CPU fallback, and every
call fails loudly when the compiled library is missing.

    M_L = prepare(H_L); M_R = prepare(H_R)                # H = M^T M, M lower
    Q, stats = quantize(W, M_L, M_R, scales, bits=4)      # int8 Q, device stats
"""
from __future__ import annotations

import ctypes
import functools
import os

import numpy as np

__all__ = [
    "Status", "GPTQ2DError", "lib", "library_path", "prepare", "quantize", "round_host",
    "kron_factor", "prepare_kron", "quantize_tensor", "MAX_KRON_FACTORS", "quantize_grid",
    "quantize_kron", "quantize_kron_workspace_size", "kron_inner_size", "per_mode_order",
    "gram_accumulate", "gram_finalize", "gram", "quantize_block", "block_workspace_size",
    "stats_dict", "launch_count", "prepare_workspace_size", "quantize_workspace_size",
    "round_host_workspace_size", "quantize_noalloc", "proxy_loss", "check_wait_timeout",
    "profile_enable",
    "profile_reset", "profile_read", "profile_timeline",
    "KERNEL_CLASSES", "STATS_WORDS", "DTYPE_F32", "DTYPE_BF16", "DTYPE_F64",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libgptq2d.so")

DTYPE_F32, DTYPE_BF16, DTYPE_F64 = 0, 1, 2
STATS_WORDS = 6  # gptq2d_stats: double + 5 x int64
MAX_KRON_FACTORS = 8  # GPTQ2D_MAX_KRON_FACTORS


class Status:
    OK = 0
    INVALID_ARG = 1
    NOT_SPD = 2
    NONFINITE = 3
    WORKSPACE = 4
    TIMEOUT = 5
    CUDA = 6
    RANGE = 7


class GPTQ2DError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {lib().gptq2d_status_string(status).decode()}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


_LIB = None
_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p


class _Grid(ctypes.Structure):
    """gptq2d_grid"""
    _fields_ = [("bits", ctypes.c_int), ("clamp", ctypes.c_int), ("group_size", _c_i64),
                ("scales", _c_p), ("ld_scales", _c_i64), ("zeros", _c_p), ("packed", ctypes.c_int)]


class _Layer(ctypes.Structure):
    """gptq2d_layer"""
    _fields_ = [("W", _c_p), ("w_dtype", ctypes.c_int), ("m", _c_i64), ("n", _c_i64),
                ("ldw", _c_i64), ("H_L", _c_p), ("ldhl", _c_i64), ("H_R", _c_p), ("ldhr", _c_i64),
                ("h_dtype", ctypes.c_int), ("grid", _Grid), ("Q", _c_p), ("ldq", _c_i64),
                ("stats", _c_p)]


def lib():
    """The loaded shared library (built in-tree by two_sided_adaptive_b200.build)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(library_path):
            raise RuntimeError(f"libgptq2d.so is not built ({library_path}); "
                               "run: python -m two_sided_adaptive_b200.build")
        L = ctypes.CDLL(library_path)
        L.gptq2d_status_string.restype = ctypes.c_char_p
        L.gptq2d_status_string.argtypes = [ctypes.c_int]
        L.gptq2d_version.restype = ctypes.c_int
        L.gptq2d_launch_count.restype = _c_i64
        L.gptq2d_check_wait_timeout.restype = ctypes.c_int
        L.gptq2d_check_wait_timeout.argtypes = [_c_i64, _c_p]
        L.gptq2d_profile_enable.restype = None
        L.gptq2d_profile_enable.argtypes = [ctypes.c_int]
        L.gptq2d_profile_read.restype = ctypes.c_int
        L.gptq2d_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(_c_i64),
                                          ctypes.POINTER(ctypes.c_double)]
        L.gptq2d_profile_reset.restype = None
        L.gptq2d_profile_timeline.restype = ctypes.c_int
        L.gptq2d_profile_timeline.argtypes = [_c_i64, _c_p, _c_p, _c_p, ctypes.POINTER(_c_i64)]
        L.gptq2d_prepare_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_prepare_workspace_size.argtypes = [_c_i64]
        L.gptq2d_prepare.restype = ctypes.c_int
        L.gptq2d_prepare.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_p, _c_i64, _c_p,
                                     ctypes.c_size_t, _c_p, ctypes.POINTER(_c_i64)]
        L.gptq2d_prepare_pair.restype = ctypes.c_int
        L.gptq2d_prepare_pair.argtypes = [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, ctypes.c_int,
                                          _c_p, _c_i64, _c_p, _c_i64, _c_p, ctypes.c_size_t, _c_p,
                                          ctypes.POINTER(_c_i64), ctypes.POINTER(ctypes.c_int)]
        L.gptq2d_prepare_info.restype = ctypes.c_int
        L.gptq2d_prepare_info.argtypes = [_c_p, _c_p, ctypes.POINTER(_c_i64)]
        L.gptq2d_block_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_block_workspace_size.argtypes = [ctypes.POINTER(_Layer), ctypes.c_int]
        L.gptq2d_quantize_block.restype = ctypes.c_int
        L.gptq2d_quantize_block.argtypes = [ctypes.POINTER(_Layer), ctypes.c_int, _c_p,
                                            ctypes.c_size_t, _c_p, ctypes.POINTER(_c_i64),
                                            ctypes.POINTER(_c_i64), ctypes.POINTER(ctypes.c_int)]
        L.gptq2d_gram_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_gram_accumulate.restype = ctypes.c_int
        L.gptq2d_gram_accumulate.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_i64,
                                             ctypes.c_int, _c_p, ctypes.c_size_t, _c_p]
        L.gptq2d_gram_finalize.restype = ctypes.c_int
        L.gptq2d_gram_finalize.argtypes = [_c_p, _c_i64, _c_i64, _c_i64, ctypes.c_double, _c_p,
                                           ctypes.c_size_t, _c_p, ctypes.POINTER(ctypes.c_int)]
        L.gptq2d_kron_factor.restype = ctypes.c_int
        L.gptq2d_kron_factor.argtypes = [ctypes.c_int, _c_p, _c_p, _c_p, _c_p, _c_i64, _c_p]
        L.gptq2d_quantize_kron_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_quantize_kron_workspace_size.argtypes = [_c_i64, ctypes.c_int, _c_p]
        L.gptq2d_per_mode_order.restype = ctypes.c_int
        L.gptq2d_per_mode_order.argtypes = [ctypes.c_int, _c_p, _c_p]
        L.gptq2d_quantize_kron_grid.restype = ctypes.c_int
        L.gptq2d_quantize_kron_grid.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_p, _c_i64,
                                                ctypes.c_int, _c_p, _c_p, _c_p,
                                                ctypes.POINTER(_Grid), _c_p, _c_i64, _c_p, _c_p,
                                                ctypes.c_size_t, _c_p]
        L.gptq2d_quantize_kron.restype = ctypes.c_int
        L.gptq2d_quantize_kron.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_p, _c_i64,
                                           ctypes.c_int, _c_p, _c_p, _c_p, _c_p, ctypes.c_int,
                                           ctypes.c_int, _c_p, _c_i64, _c_p, _c_p, ctypes.c_size_t,
                                           _c_p]
        L.gptq2d_quantize_grid.restype = ctypes.c_int
        L.gptq2d_quantize_grid.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_i64,
                                           _c_p, _c_i64, ctypes.POINTER(_Grid), _c_p, _c_i64, _c_p,
                                           _c_p, ctypes.c_size_t, _c_p]
        L.gptq2d_quantize_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_quantize_workspace_size.argtypes = [_c_i64, _c_i64]
        L.gptq2d_quantize.restype = ctypes.c_int
        L.gptq2d_quantize.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_i64,
                                      _c_p, _c_i64, _c_p, ctypes.c_int, ctypes.c_int, _c_p,
                                      _c_i64, _c_p, _c_p, ctypes.c_size_t, _c_p]
        L.gptq2d_quantize_noalloc.restype = ctypes.c_int
        L.gptq2d_quantize_noalloc.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p,
                                              _c_i64, _c_p, _c_i64, _c_p, ctypes.c_int,
                                              ctypes.c_int, _c_p, _c_i64, _c_p, _c_p]
        L.gptq2d_proxy_loss_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_proxy_loss_workspace_size.argtypes = [_c_i64, _c_i64]
        L.gptq2d_proxy_loss.restype = ctypes.c_int
        L.gptq2d_proxy_loss.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_i64, _c_p, _c_i64,
                                        _c_p, ctypes.c_int, ctypes.c_int, _c_p, _c_i64, _c_p,
                                        _c_i64, _c_p, _c_p, ctypes.c_size_t, _c_p]
        L.gptq2d_round_host_workspace_size.restype = ctypes.c_size_t
        L.gptq2d_round_host_workspace_size.argtypes = [_c_i64, _c_i64, ctypes.c_int, ctypes.c_int]
        L.gptq2d_round_host.restype = ctypes.c_int
        L.gptq2d_round_host.argtypes = [_c_p, ctypes.c_int, _c_i64, _c_i64, _c_p, _c_p,
                                        ctypes.c_int, _c_p, ctypes.c_int, ctypes.c_int, _c_p,
                                        _c_p, _c_p, ctypes.c_size_t, _c_p,
                                        ctypes.POINTER(_c_i64), ctypes.POINTER(ctypes.c_int)]
        _LIB = L
    return _LIB


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().gptq2d_launch_count())


def check_wait_timeout(limit_ns: int, stream=None) -> int:
    """Runs the device-side bounded wait on an mbarrier that nothing completes
    (gptq2d_check_wait_timeout); returns the status, Status.TIMEOUT when the wait
    gave up as it must."""
    return int(lib().gptq2d_check_wait_timeout(int(limit_ns), _stream(stream)))


KERNEL_CLASSES = ("prep_panel", "prep_trailing", "sweep", "propagate", "other")


def profile_enable(on: bool = True) -> None:
    """Bracket every library launch with CUDA events on its stream (gptq2d_profile_enable)."""
    lib().gptq2d_profile_enable(int(on))


def profile_reset() -> None:
    lib().gptq2d_profile_reset()


def profile_read() -> dict:
    """{kernel class: (launches, total device ms)} of the launches recorded so far."""
    out = {}
    for k, name in enumerate(KERNEL_CLASSES):
        n, ms = _c_i64(0), ctypes.c_double(0.0)
        rc = lib().gptq2d_profile_read(k, ctypes.byref(n), ctypes.byref(ms))
        if rc != Status.OK:
            raise GPTQ2DError(rc, "gptq2d_profile_read")
        out[name] = (int(n.value), float(ms.value))
    return out


def profile_timeline():
    """[(kernel class, start ms, end ms)] of the recorded launches, relative to the first."""
    n = _c_i64(0)
    rc = lib().gptq2d_profile_timeline(0, None, None, None, ctypes.byref(n))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_profile_timeline")
    cls = (ctypes.c_int32 * max(1, n.value))()
    t0 = (ctypes.c_double * max(1, n.value))()
    t1 = (ctypes.c_double * max(1, n.value))()
    rc = lib().gptq2d_profile_timeline(n.value, cls, t0, t1, ctypes.byref(n))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_profile_timeline")
    return [(KERNEL_CLASSES[cls[i]], t0[i], t1[i]) for i in range(n.value)]


def prepare_workspace_size(k: int) -> int:
    return int(lib().gptq2d_prepare_workspace_size(k))


def quantize_workspace_size(m: int, n: int) -> int:
    return int(lib().gptq2d_quantize_workspace_size(m, n))


def round_host_workspace_size(m: int, n: int, w_dtype: int, h_dtype: int) -> int:
    return int(lib().gptq2d_round_host_workspace_size(m, n, w_dtype, h_dtype))


# --------------------------------------------------------------------------- #
# torch marshalling
# --------------------------------------------------------------------------- #
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    codes = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float64: DTYPE_F64}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _ld(t) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride (row-major)")
    return t.stride(0)


def _stream(stream):
    """The stream to enqueue on: the current device's current stream, or ``stream``,
    which must belong to the current device (the library launches on the current
    device, and every wrapper makes its tensors' device current first)."""
    torch = _torch()
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if stream.device.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {stream.device}, the tensors on cuda:"
                         f"{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _check_device(*ts):
    """Every given tensor (None skipped) must live on the current CUDA device, which the
    wrapper has made the tensors' own (see _device_scoped)."""
    torch = _torch()
    cur = torch.cuda.current_device() if torch.cuda.is_available() else None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if t.device.index != cur:
            raise ValueError(f"all tensors of a call must share one device: {t.device} "
                             f"is not cuda:{cur}")


def _first_cuda_device(objs):
    for o in objs:
        if hasattr(o, "is_cuda") and hasattr(o, "device"):
            if o.is_cuda:
                return o.device
        elif isinstance(o, dict):
            d = _first_cuda_device(o.values())
            if d is not None:
                return d
        elif isinstance(o, (list, tuple)):
            d = _first_cuda_device(o)
            if d is not None:
                return d
    return None


def _device_scoped(fn):
    """Runs the wrapper with the device of its first CUDA tensor argument current, so
    that the library's kernels, its per-device streams and its static scratch all
    belong to the device that holds the data (a tensor on another device is then
    rejected by _check_device instead of being dereferenced by the wrong GPU)."""
    @functools.wraps(fn)
    def wrapper(*args, **kw):
        dev = _first_cuda_device(list(args) + list(kw.values()))
        if dev is None:
            return fn(*args, **kw)
        with _torch().cuda.device(dev):
            return fn(*args, **kw)
    return wrapper


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    # 256-byte alignment: torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


@_device_scoped
def prepare(H, *, out=None, workspace=None, stream=None, check: bool = True):
    """Lower-triangular M with M^T M = H (fp64), by gptq2d_prepare.  H: k x k fp32/fp64 on
    the GPU (lower triangle read).  ``check`` synchronizes and raises on a non-SPD H."""
    torch = _torch()
    _check_device(H, out, workspace)
    k = H.shape[0]
    if H.dim() != 2 or H.shape[1] != k:
        raise ValueError("H must be square")
    M = out if out is not None else torch.empty((k, k), dtype=torch.float64, device=H.device)
    ws = _workspace(prepare_workspace_size(k), H.device, workspace)
    piv = _c_i64(-1)
    rc = lib().gptq2d_prepare(H.data_ptr(), _dtype_code(H), k, _ld(H), M.data_ptr(), _ld(M),
                              ws.data_ptr(), ws.numel(), _stream(stream),
                              ctypes.byref(piv) if check else None)
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_prepare", f"pivot {piv.value}" if rc == Status.NOT_SPD else "")
    return M


@_device_scoped
def prepare_pair(H_L, H_R, *, out_l=None, out_r=None, workspace=None, stream=None,
                 check: bool = True):
    """Both factors at once (gptq2d_prepare_pair): the two factorizations run concurrently
    on library-internal streams joined back to ``stream``.  Returns (M_L, M_R)."""
    torch = _torch()
    _check_device(H_L, H_R, out_l, out_r, workspace)
    if H_L.dtype != H_R.dtype:
        raise ValueError("H_L and H_R must share a dtype")
    m, n = H_L.shape[0], H_R.shape[0]
    ML = out_l if out_l is not None else torch.empty((m, m), dtype=torch.float64, device=H_L.device)
    MR = out_r if out_r is not None else torch.empty((n, n), dtype=torch.float64, device=H_L.device)
    ws = _workspace(512, H_L.device, workspace)
    piv, which = _c_i64(-1), ctypes.c_int(-1)
    rc = lib().gptq2d_prepare_pair(H_L.data_ptr(), m, _ld(H_L), H_R.data_ptr(), n, _ld(H_R),
                                   _dtype_code(H_L), ML.data_ptr(), _ld(ML), MR.data_ptr(), _ld(MR),
                                   ws.data_ptr(), ws.numel(), _stream(stream),
                                   ctypes.byref(piv) if check else None,
                                   ctypes.byref(which) if check else None)
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_prepare_pair",
                          f"factor {which.value} pivot {piv.value}" if rc == Status.NOT_SPD else "")
    return ML, MR


@_device_scoped
def gram_accumulate(X, H, *, accumulate: bool, workspace, stream=None):
    """gptq2d_gram_accumulate: H's lower 128-block triangle (+)= X^T X for a bf16 batch X
    (rows x k on the GPU; k a multiple of 8) on the tensor cores.  ``workspace``: a device
    uint8 tensor of at least gptq2d_gram_workspace_size() bytes, kept until finalize."""
    torch = _torch()
    _check_device(X, H, workspace)
    if X.dtype != torch.bfloat16 or H.dtype != torch.float32:
        raise ValueError("X must be bf16 and H fp32")
    rows, k = X.shape
    rc = lib().gptq2d_gram_accumulate(X.data_ptr(), DTYPE_BF16, rows, k, _ld(X) if rows else k,
                                      H.data_ptr(), _ld(H), int(bool(accumulate)),
                                      workspace.data_ptr(), workspace.numel(), _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_gram_accumulate")
    return H


@_device_scoped
def gram_finalize(H, total_rows: int, damp: float = 0.01, *, workspace, stream=None,
                  check: bool = True):
    """gptq2d_gram_finalize: H <- H / total_rows with damp * mean(diag) added to the
    diagonal.  ``check`` synchronizes and raises if a bounded wait gave up."""
    _check_device(H, workspace)
    st = ctypes.c_int(0)
    rc = lib().gptq2d_gram_finalize(H.data_ptr(), H.shape[0], _ld(H), int(total_rows), float(damp),
                                    workspace.data_ptr(), workspace.numel(), _stream(stream),
                                    ctypes.byref(st) if check else None)
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_gram_finalize")
    return H


@_device_scoped
def gram(batches, damp: float = 0.01, *, out=None, stream=None):
    """The damped Gram X^T X / N + damp * mean(diag) I of bf16 activation batches (each
    rows x k on the GPU), accumulated on the tensor cores.  Returns H (fp32 k x k; its
    lower triangle is the Gram, ready for prepare)."""
    torch = _torch()
    batches = list(batches)
    k = batches[0].shape[1]
    dev_ = batches[0].device
    H = out if out is not None else torch.empty((k, k), dtype=torch.float32, device=dev_)
    ws = torch.empty(max(lib().gptq2d_gram_workspace_size(), 256), dtype=torch.uint8, device=dev_)
    total = 0
    for b, X in enumerate(batches):
        gram_accumulate(X, H, accumulate=b > 0, workspace=ws, stream=stream)
        total += X.shape[0]
    return gram_finalize(H, total, damp, workspace=ws, stream=stream)


@_device_scoped
def kron_factor(Ms, *, out=None, stream=None):
    """M_1 kron M_2 kron ... of lower fp64 factors (gptq2d_kron_factor): the reverse Cholesky
    factor of H_1 kron H_2 kron ... when M_j = prepare(H_j).  Entries where some column
    digit exceeds the row digit are exact zeros."""
    torch = _torch()
    if not 1 <= len(Ms) <= MAX_KRON_FACTORS:
        raise ValueError(f"1 to {MAX_KRON_FACTORS} factors")
    _check_device(*Ms, out)
    for M in Ms:
        if M.dtype != torch.float64 or M.dim() != 2 or M.shape[0] != M.shape[1]:
            raise ValueError("factors must be square fp64 matrices")
    n = int(np.prod([M.shape[0] for M in Ms]))
    K = out if out is not None else torch.empty((n, n), dtype=torch.float64, device=Ms[0].device)
    nf = len(Ms)
    ptrs = (ctypes.c_void_p * nf)(*[M.data_ptr() for M in Ms])
    dims = (_c_i64 * nf)(*[M.shape[0] for M in Ms])
    lds = (_c_i64 * nf)(*[_ld(M) for M in Ms])
    rc = lib().gptq2d_kron_factor(nf, ptrs, dims, lds, K.data_ptr(), _ld(K) if n else n,
                                  _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_kron_factor")
    return K


@_device_scoped
def prepare_kron(Hs, *, stream=None, check: bool = True):
    """Factors of a k-factor Kronecker Hessian H_1 kron ... kron H_k (H_j on mode j of a
    k-way tensor) for the 2-D rounding: returns (M_L, M_R) with M_L = prepare(H_1) and
    M_R = kron_factor([prepare(H_2), ..., prepare(H_k)])."""
    if len(Hs) < 2:
        raise ValueError("at least two factors")
    Ms = [prepare(H, stream=stream, check=check) for H in Hs]
    return Ms[0], (Ms[1] if len(Ms) == 2 else kron_factor(Ms[1:], stream=stream))


def kron_inner_size(dims) -> int:
    """m_in of gptq2d_quantize_kron for these trailing modes: the largest product of a
    suffix of ``dims`` dividing 64 when it is at least 8, else 0 (the per-mode path
    does not apply)."""
    p, best = 1, 0
    for d in reversed([int(x) for x in dims]):
        if d < 1 or p * d > 64 or 64 % (p * d) != 0:
            break
        p *= d
        if p >= 8:
            best = p
    return best


def quantize_kron_workspace_size(m: int, dims) -> int:
    nf = len(dims)
    arr = (_c_i64 * nf)(*[int(d) for d in dims])
    return int(lib().gptq2d_quantize_kron_workspace_size(int(m), nf, arr))


@_device_scoped
def quantize_kron(W, M_L, Ms, scales, bits: int = 4, clamp: bool = True, *, group_size: int = 0,
                  zeros=None, packed: bool = False, out=None, stats=None, workspace=None,
                  stream=None):
    """The k-way rounding with the right factor kept per mode (gptq2d_quantize_kron): W is
    the m x (m_2 ... m_k) matrix of the tensor, M_L = prepare(H_1), Ms = [prepare(H_2), ...,
    prepare(H_k)].  group_size / zeros / packed select a grid variant as in quantize_grid
    (gptq2d_quantize_kron_grid).  Returns (Q bytes m x n, or m x ceil(n/2) packed; stats
    on the device)."""
    torch = _torch()
    _check_device(W, M_L, scales, zeros, out, stats, workspace, *Ms)
    m, n = W.shape
    if not 1 <= len(Ms) <= MAX_KRON_FACTORS:
        raise ValueError(f"1 to {MAX_KRON_FACTORS} trailing factors")
    for M in Ms:
        if M.dtype != torch.float64 or M.dim() != 2 or M.shape[0] != M.shape[1]:
            raise ValueError("factors must be square fp64 matrices")
    dims = [int(M.shape[0]) for M in Ms]
    if int(np.prod(dims)) != n:
        raise ValueError("the factors' sizes must multiply to W's column count")
    if M_L.dtype != torch.float64:
        raise ValueError("factors must be fp64")
    if scales.dtype != torch.float32:
        raise ValueError("scales must be fp32")
    grid = group_size != 0 or zeros is not None or packed
    if grid:
        S = scales.reshape(m, -1) if scales.dim() == 1 else scales
        if S.shape[0] != m or S.stride(1) != 1:
            raise ValueError("scales must have m rows with unit column stride")
        if zeros is not None:
            if zeros.dtype != torch.uint8 or tuple(zeros.reshape(m, -1).shape) != tuple(S.shape):
                raise ValueError("zeros must be uint8, shaped like the scales")
            Z = zeros.reshape(m, -1)
            if Z.stride(0) != S.stride(0) or Z.stride(1) != 1:
                raise ValueError("zeros must share the scales' layout")
    elif scales.numel() != m or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous fp32 vector of length m")
    qdt = torch.uint8 if (zeros is not None or packed) else torch.int8
    ncol = (n + 1) // 2 if packed else n
    Q = out if out is not None else torch.empty((m, ncol), dtype=qdt, device=W.device)
    st = stats if stats is not None else torch.empty(STATS_WORDS, dtype=torch.int64, device=W.device)
    ws = _workspace(max(quantize_kron_workspace_size(m, dims), 256), W.device, workspace)
    nf = len(Ms)
    ptrs = (ctypes.c_void_p * nf)(*[M.data_ptr() for M in Ms])
    dimsa = (_c_i64 * nf)(*dims)
    lds = (_c_i64 * nf)(*[_ld(M) for M in Ms])
    if grid:
        gr = _Grid(int(bits), int(clamp), int(group_size), S.data_ptr(), S.stride(0) if m else 1,
                   zeros.data_ptr() if zeros is not None else None, int(bool(packed)))
        rc = lib().gptq2d_quantize_kron_grid(W.data_ptr(), _dtype_code(W), m, _ld(W), M_L.data_ptr(),
                                             _ld(M_L), nf, ptrs, dimsa, lds, ctypes.byref(gr),
                                             Q.data_ptr(), _ld(Q) if Q.numel() else ncol,
                                             st.data_ptr(), ws.data_ptr(), ws.numel(),
                                             _stream(stream))
        name = "gptq2d_quantize_kron_grid"
    else:
        rc = lib().gptq2d_quantize_kron(W.data_ptr(), _dtype_code(W), m, _ld(W), M_L.data_ptr(),
                                        _ld(M_L), nf, ptrs, dimsa, lds, scales.data_ptr(),
                                        int(bits), int(clamp), Q.data_ptr(), _ld(Q),
                                        st.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
        name = "gptq2d_quantize_kron"
    if rc != Status.OK:
        raise GPTQ2DError(rc, name)
    return Q, st


def per_mode_order(dims):
    """An order of the trailing modes for quantize_kron, or None: the subset of modes
    whose sizes multiply to the largest of 64, 32, 16, 8 goes last (the inner group),
    the rest keep their order in front.  The k-way rounding depends only on each
    entry's dominated orthant, so reordering the trailing modes permutes the result
    and nothing else.  The given order is kept when it already reaches that size."""
    dims = [int(d) for d in dims]
    k = len(dims)
    best, best_p = None, 0
    for mask in range(1, 1 << k):
        sel = [i for i in range(k) if (mask >> i) & 1]
        p = int(np.prod([dims[i] for i in sel]))
        if p in (8, 16, 32, 64) and p > best_p:
            best, best_p = sel, p
    if best is None:
        return None
    if kron_inner_size(dims) == best_p:
        return list(range(k))
    return [i for i in range(k) if i not in best] + best


@_device_scoped
def quantize_tensor(W, Hs, scales, bits: int = 4, clamp: bool = True, *, group_size: int = 0,
                    zeros=None, packed: bool = False, per_mode=None, stream=None):
    """GPTQ-2D rounding of a k-way tensor W (m_1 x ... x m_k, C order) under
    H_1 kron ... kron H_k with scales per index of mode 1: the m_1 x (m_2 ... m_k) problem
    with M_L = prepare(H_1) and the right factor M_2 kron ... kron M_k.  per_mode=None picks
    the per-mode right factor (quantize_kron) when some order of the trailing modes allows
    it (per_mode_order: the tensor is rounded with those modes reordered and Q is put back
    in W's order), and the dense Kronecker factor (kron_factor + quantize) otherwise; True
    or False forces one.  group_size / zeros / packed select a grid variant as in
    quantize_grid, with the scale groups along the flattened trailing modes; a grid keeps
    the given mode order (a reorder would break the groups), so the per-mode route then
    needs that order to allow it.  Returns (Q shaped like W, or m_1 x ceil(n/2) bytes
    when packed; stats)."""
    if W.dim() != len(Hs) or W.dim() < 2:
        raise ValueError("one Hessian factor per mode, at least two modes")
    dims = list(W.shape[1:])
    grid = dict(group_size=group_size, zeros=zeros, packed=packed) \
        if (group_size or zeros is not None or packed) else None
    ident = list(range(len(dims)))
    if grid is not None:
        order = ident if kron_inner_size(dims) > 0 else None
    else:
        order = per_mode_order(dims)
    if per_mode is False:
        order = None
    if per_mode and order is None:
        raise ValueError("no usable order of the trailing modes has an inner group of 8 to 64")
    m = W.shape[0]
    if order is not None:
        Ms = [prepare(H, stream=stream) for H in Hs]
        perm = [0] + [1 + i for i in order]
        Wp = W.permute(*perm).contiguous() if order != ident else W
        Q, st = quantize_kron(Wp.reshape(m, -1), Ms[0], [Ms[1 + i] for i in order], scales, bits,
                              clamp, stream=stream, **(grid or {}))
        if grid is not None and packed:
            return Q, st
        Q = Q.reshape(Wp.shape)
        if order != ident:
            inv = [0] * len(perm)
            for a_, b_ in enumerate(perm):
                inv[b_] = a_
            Q = Q.permute(*inv).contiguous()
        return Q, st
    M_L, M_R = prepare_kron(Hs, stream=stream)
    if grid is not None:
        Q, st = quantize_grid(W.reshape(m, -1), M_L, M_R, scales, bits, clamp, stream=stream, **grid)
        return (Q, st) if packed else (Q.reshape(W.shape), st)
    Q, st = quantize(W.reshape(m, -1), M_L, M_R, scales, bits, clamp, stream=stream)
    return Q.reshape(W.shape), st


@_device_scoped
def quantize(W, M_L, M_R, scales, bits: int = 4, clamp: bool = True, *, out=None, stats=None,
             workspace=None, stream=None):
    """GPTQ-2D rounding by gptq2d_quantize.  Returns (Q int8 m x n, stats int64[5] on the
    device; decode with stats_dict)."""
    torch = _torch()
    _check_device(W, M_L, M_R, scales, out, stats, workspace)
    m, n = W.shape
    if scales.dtype != torch.float32 or scales.numel() != m or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous fp32 vector of length m")
    if M_L.dtype != torch.float64 or M_R.dtype != torch.float64:
        raise ValueError("factors must be fp64")
    Q = out if out is not None else torch.empty((m, n), dtype=torch.int8, device=W.device)
    st = stats if stats is not None else torch.empty(STATS_WORDS, dtype=torch.int64, device=W.device)
    ws = _workspace(quantize_workspace_size(m, n), W.device, workspace)
    rc = lib().gptq2d_quantize(W.data_ptr(), _dtype_code(W), m, n, _ld(W), M_L.data_ptr(), _ld(M_L),
                               M_R.data_ptr(), _ld(M_R), scales.data_ptr(), int(bits), int(clamp),
                               Q.data_ptr(), _ld(Q), st.data_ptr(), ws.data_ptr(), ws.numel(),
                               _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_quantize")
    return Q, st


@_device_scoped
def quantize_grid(W, M_L, M_R, scales, bits: int = 4, clamp: bool = True, *, group_size: int = 0,
                  zeros=None, packed: bool = False, out=None, stats=None, workspace=None, stream=None):
    """GPTQ-2D rounding on a grid variant (gptq2d_quantize_grid).  ``scales``: fp32 m x groups
    (or a length-m vector when group_size is 0); ``zeros``: optional uint8 integer zero points
    of the same shape (asymmetric grid, codes in [0, 2^bits - 1]; needs clamp); ``packed``: two 4-bit codes
    per byte (bits <= 4).  Returns (Q bytes: int8 q on the symmetric grid, uint8 codes on the
    asymmetric one, packed codes m x ceil(n/2) when packed; stats on the device)."""
    torch = _torch()
    _check_device(W, M_L, M_R, scales, out, stats, workspace)
    m, n = W.shape
    if scales.dtype != torch.float32:
        raise ValueError("scales must be fp32")
    S = scales.reshape(m, -1) if scales.dim() == 1 else scales
    if S.shape[0] != m or S.stride(1) != 1:
        raise ValueError("scales must have m rows with unit column stride")
    if zeros is not None:
        _check_device(zeros)
        if zeros.dtype != torch.uint8 or tuple(zeros.reshape(m, -1).shape) != tuple(S.shape):
            raise ValueError("zeros must be uint8, shaped like the scales")
        Z = zeros.reshape(m, -1)
        if Z.stride(0) != S.stride(0) or Z.stride(1) != 1:
            raise ValueError("zeros must share the scales' layout")
    if M_L.dtype != torch.float64 or M_R.dtype != torch.float64:
        raise ValueError("factors must be fp64")
    qdt = torch.uint8 if (zeros is not None or packed) else torch.int8
    ncol = (n + 1) // 2 if packed else n
    Q = out if out is not None else torch.empty((m, ncol), dtype=qdt, device=W.device)
    st = stats if stats is not None else torch.empty(STATS_WORDS, dtype=torch.int64, device=W.device)
    ws = _workspace(quantize_workspace_size(m, n), W.device, workspace)
    gr = _Grid(int(bits), int(clamp), int(group_size), S.data_ptr(), S.stride(0) if m else 1,
               zeros.data_ptr() if zeros is not None else None, int(bool(packed)))
    rc = lib().gptq2d_quantize_grid(W.data_ptr(), _dtype_code(W), m, n, _ld(W), M_L.data_ptr(),
                                    _ld(M_L), M_R.data_ptr(), _ld(M_R), ctypes.byref(gr),
                                    Q.data_ptr(), _ld(Q) if Q.numel() else ncol, st.data_ptr(),
                                    ws.data_ptr(), ws.numel(), _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_quantize_grid")
    return Q, st


def _layers(specs, outs, stats):
    torch = _torch()
    arr = (_Layer * len(specs))()
    keep = []
    for i, sp in enumerate(specs):
        W, H_L, H_R, sc = sp["W"], sp["H_L"], sp["H_R"], sp["scales"]
        m, n = W.shape
        S = sc.reshape(m, -1) if sc.dim() == 1 else sc
        Z = sp.get("zeros")
        if Z is not None:
            Z = Z.reshape(m, -1)
        packed = bool(sp.get("packed", False))
        keep += [S, Z]
        gr = _Grid(int(sp.get("bits", 4)), int(sp.get("clamp", True)), int(sp.get("group_size", 0)),
                   S.data_ptr(), S.stride(0) if m else 1, Z.data_ptr() if Z is not None else None,
                   int(packed))
        if H_L.dtype != H_R.dtype:
            raise ValueError("H_L and H_R must share a dtype")
        arr[i] = _Layer(W.data_ptr(), _dtype_code(W), m, n, _ld(W), H_L.data_ptr(), _ld(H_L),
                        H_R.data_ptr(), _ld(H_R), _dtype_code(H_L), gr,
                        outs[i].data_ptr() if outs is not None else None,
                        _ld(outs[i]) if outs is not None and outs[i].numel() else 1,
                        stats[i].data_ptr() if stats is not None else None)
    return arr, keep


def block_workspace_size(specs) -> int:
    """gptq2d_block_workspace_size for layer specs (dicts with W, H_L, H_R, scales, ...)."""
    arr, _ = _layers(specs, None, None)
    return int(lib().gptq2d_block_workspace_size(arr, len(specs)))


@_device_scoped
def quantize_block(specs, *, workspace=None, stream=None):
    """gptq2d_quantize_block: factors and rounds a block of layers, the factor preparation
    of the next layer overlapping the rounding of the current one.  ``specs``: dicts with
    W (m x n), H_L (m x m), H_R (n x n) Grams on the GPU, scales (m or m x groups fp32),
    and optionally bits, clamp, group_size, zeros (uint8), packed.  Returns (list of Q,
    list of stats)."""
    torch = _torch()
    if not specs:
        return [], []
    _check_device(*[sp.get(k) for sp in specs for k in ("W", "H_L", "H_R", "scales", "zeros")],
                  workspace)
    dev_ = specs[0]["W"].device
    outs, stats = [], []
    for sp in specs:
        m, n = sp["W"].shape
        packed = bool(sp.get("packed", False))
        qdt = torch.uint8 if (sp.get("zeros") is not None or packed) else torch.int8
        outs.append(torch.empty((m, (n + 1) // 2 if packed else n), dtype=qdt, device=dev_))
        stats.append(torch.empty(STATS_WORDS, dtype=torch.int64, device=dev_))
    arr, keep = _layers(specs, outs, stats)
    nbytes = int(lib().gptq2d_block_workspace_size(arr, len(specs)))
    ws = _workspace(nbytes, dev_, workspace)
    bl, bp, wf = _c_i64(-1), _c_i64(-1), ctypes.c_int(-1)
    rc = lib().gptq2d_quantize_block(arr, len(specs), ws.data_ptr(), ws.numel(), _stream(stream),
                                     ctypes.byref(bl), ctypes.byref(bp), ctypes.byref(wf))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_quantize_block",
                          f"layer {bl.value} factor {wf.value} pivot {bp.value}"
                          if rc == Status.NOT_SPD else "")
    return outs, stats


@_device_scoped
def quantize_noalloc(W, M_L, M_R, scales, bits: int = 4, clamp: bool = True, *, out=None,
                     stats=None, stream=None):
    """gptq2d_quantize_noalloc: the same rounding with the library's static device scratch
    (no workspace; for callers that cannot allocate).  Problems must fit
    GPTQ2D_NOALLOC_SCRATCH_BYTES; calls that overlap on the GPU race on the shared scratch."""
    torch = _torch()
    _check_device(W, M_L, M_R, scales, out, stats)
    m, n = W.shape
    if scales.dtype != torch.float32 or scales.numel() != m or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous fp32 vector of length m")
    if M_L.dtype != torch.float64 or M_R.dtype != torch.float64:
        raise ValueError("factors must be fp64")
    Q = out if out is not None else torch.empty((m, n), dtype=torch.int8, device=W.device)
    st = stats if stats is not None else torch.empty(STATS_WORDS, dtype=torch.int64, device=W.device)
    rc = lib().gptq2d_quantize_noalloc(W.data_ptr(), _dtype_code(W), m, n, _ld(W), M_L.data_ptr(),
                                       _ld(M_L), M_R.data_ptr(), _ld(M_R), scales.data_ptr(),
                                       int(bits), int(clamp), Q.data_ptr(), _ld(Q), st.data_ptr(),
                                       _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_quantize_noalloc")
    return Q, st


@_device_scoped
def proxy_loss(W, M_L, M_R, scales, Q=None, bits: int = 4, clamp: bool = True, *, out=None,
               workspace=None, stream=None):
    """tr(dW^T H_L dW H_R) = ||M_L dW M_R^T||_F^2 of the integers Q (int8 m x n), or of
    round-to-nearest on the bits / clamp grid when Q is None (gptq2d_proxy_loss).
    Returns a one-element fp64 device tensor."""
    torch = _torch()
    _check_device(W, M_L, M_R, scales, Q, out, workspace)
    m, n = W.shape
    if scales.dtype != torch.float32 or scales.numel() != m or not scales.is_contiguous():
        raise ValueError("scales must be a contiguous fp32 vector of length m")
    if M_L.dtype != torch.float64 or M_R.dtype != torch.float64:
        raise ValueError("factors must be fp64")
    if Q is not None and (Q.dtype != torch.int8 or tuple(Q.shape) != (m, n)):
        raise ValueError("Q must be int8 m x n")
    res = out if out is not None else torch.empty(1, dtype=torch.float64, device=W.device)
    ws = _workspace(int(lib().gptq2d_proxy_loss_workspace_size(m, n)), W.device, workspace)
    rc = lib().gptq2d_proxy_loss(W.data_ptr(), _dtype_code(W), m, n, _ld(W),
                                 Q.data_ptr() if Q is not None else None,
                                 _ld(Q) if Q is not None else n, scales.data_ptr(), int(bits),
                                 int(clamp), M_L.data_ptr(), _ld(M_L), M_R.data_ptr(), _ld(M_R),
                                 res.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    if rc != Status.OK:
        raise GPTQ2DError(rc, "gptq2d_proxy_loss")
    return res


def stats_dict(st) -> dict:
    """Decodes a gptq2d_stats (int64[STATS_WORDS] tensor or array) into a dict."""
    a = np.asarray(st.cpu() if hasattr(st, "cpu") else st, dtype=np.int64).copy()
    return {"proxy_loss": float(a[:1].view(np.float64)[0]), "n_clamped": int(a[1]),
            "n_near_tie": int(a[2]), "n_nonfinite": int(a[3]), "status": int(a[4]),
            "n_out_of_range": int(a[5])}


@_device_scoped
def round_host(W, H_L, H_R, scales, bits: int = 4, clamp: bool = True, *, workspace=None,
               stream=None, Q_out=None, stats_out=None):
    """The whole path from HOST tensors through gptq2d_round_host: copies in, factors both
    Kronecker factors, rounds, copies Q and the statistics out.  Inputs should be pinned CPU
    tensors; ``workspace`` is a device uint8 tensor of round_host_workspace_size bytes."""
    torch = _torch()
    m, n = W.shape
    for t in (W, H_L, H_R, scales):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("round_host takes contiguous host tensors")
    if H_L.dtype != H_R.dtype:
        raise ValueError("H_L and H_R must share a dtype")
    _check_device(workspace)
    wdt, hdt = _dtype_code(W), _dtype_code(H_L)
    need = round_host_workspace_size(m, n, wdt, hdt)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    Q = Q_out if Q_out is not None else torch.empty((m, n), dtype=torch.int8, pin_memory=True)
    st = stats_out if stats_out is not None else torch.empty(STATS_WORDS, dtype=torch.int64,
                                                             pin_memory=True)
    piv, which = _c_i64(-1), ctypes.c_int(-1)
    rc = lib().gptq2d_round_host(W.data_ptr(), wdt, m, n, H_L.data_ptr(), H_R.data_ptr(), hdt,
                                 scales.data_ptr(), int(bits), int(clamp), Q.data_ptr(),
                                 st.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                 _stream(stream), ctypes.byref(piv), ctypes.byref(which))
    if rc not in (Status.OK, Status.NONFINITE, Status.RANGE):
        raise GPTQ2DError(rc, "gptq2d_round_host",
                          f"factor {which.value} pivot {piv.value}" if rc == Status.NOT_SPD else "")
    return Q, st

"""Thin ctypes binding of the C ABI in ``include/sla.h``.

Argument marshalling only: tensors are checked for device, dtype and layout
and passed as raw device pointers together with the current CUDA stream;
every step of the computation runs in the library's kernels.  There is no
fallback: if ``libsla.so`` is missing or no CUDA device is present, the calls
raise.

The same names as the C functions: :func:`sla_route`, :func:`sla_forward`,
:func:`sla_pisa_forward`, :func:`sla_workspace_size`,
:func:`sla_check_device_status`.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsla.so")

SLA_OK = 0
SLA_ERR_INVALID_ARG = 1
SLA_ERR_UNSUPPORTED = 2
SLA_ERR_WORKSPACE = 3
SLA_ERR_CUDA = 4
SLA_ERR_TIMEOUT = 5
SLA_ERR_DEVICE_CHECK = 6

SLA_SPARSE_BF16 = 0
SLA_SPARSE_FP8_E4M3 = 1
SLA_SPARSE_INT8 = 2
SLA_LUT_COMPUTE = 0
SLA_LUT_GIVEN = 1
SLA_OUT_BF16 = 0
SLA_OUT_FP32 = 1

EXPORTED = ("sla_workspace_size", "sla_route", "sla_forward", "sla_pisa_forward",
            "sla_status_string", "sla_check_device_status", "sla_version",
            "sla_profile_enable", "sla_profile_read", "sla_route_noalloc",
            "sla_cocluster", "sla_cocluster_workspace_size", "sla_permute_rows",
            "sla_forward_host", "sla_pisa_forward_host")
KERNEL_KINDS = ("pool", "kv_stats", "h_reduce", "fold_w", "score_topk", "attn", "quant_q", "project",
                "cov", "pre_attn", "cocluster", "permute")
# profile entries that are phases of a call, not kernel launches
PHASE_KINDS = ("pre_attn",)


class SlaParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("Bq", ctypes.c_int32), ("Bk", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("sparse_dtype", ctypes.c_int32), ("lut_mode", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("pisa_first_order", ctypes.c_int32),
                ("pisa_cov_lambda", ctypes.c_float)]


class SlaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s: %s (status %d)" % (where, status_string(code), code))


_lock = threading.Lock()
_lib = None


def load():
    """Load libsla.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError("libsla.so not built: run python -m block_sparse_linear_proj_b200.build")
            lib = ctypes.CDLL(LIB_PATH)
            P = ctypes.c_void_p
            PP = ctypes.POINTER(SlaParams)
            lib.sla_workspace_size.argtypes = [PP]
            lib.sla_workspace_size.restype = ctypes.c_size_t
            lib.sla_route.argtypes = [PP, P, P, P, P, P, P, ctypes.c_size_t, P]
            lib.sla_route.restype = ctypes.c_int
            lib.sla_route_noalloc.argtypes = [PP, P, P, P, P, P, P]
            lib.sla_route_noalloc.restype = ctypes.c_int
            lib.sla_forward.argtypes = [PP, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
            lib.sla_forward.restype = ctypes.c_int
            lib.sla_pisa_forward.argtypes = [PP, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
            lib.sla_pisa_forward.restype = ctypes.c_int
            lib.sla_pisa_cov_norms.argtypes = [PP, P, P, P, P, ctypes.c_size_t, P]
            lib.sla_pisa_cov_norms.restype = ctypes.c_int
            lib.sla_status_string.argtypes = [ctypes.c_int]
            lib.sla_status_string.restype = ctypes.c_char_p
            lib.sla_check_device_status.argtypes = [P]
            lib.sla_check_device_status.restype = ctypes.c_int
            lib.sla_version.argtypes = []
            lib.sla_version.restype = ctypes.c_int32
            lib.sla_profile_enable.argtypes = [ctypes.c_int32]
            lib.sla_profile_enable.restype = ctypes.c_int
            lib.sla_profile_read.argtypes = [P, P]
            lib.sla_profile_read.restype = ctypes.c_int
            lib.sla_cocluster_workspace_size.argtypes = [PP, ctypes.c_int32]
            lib.sla_cocluster_workspace_size.restype = ctypes.c_size_t
            lib.sla_cocluster.argtypes = [PP, P, P, ctypes.c_int32, ctypes.c_int32, P, P, P, ctypes.c_size_t, P]
            lib.sla_cocluster.restype = ctypes.c_int
            lib.sla_permute_rows.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_int32, P]
            lib.sla_permute_rows.restype = ctypes.c_int
            lib.sla_forward_host.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_int32, P,
                                             ctypes.c_size_t, P]
            lib.sla_forward_host.restype = ctypes.c_int
            lib.sla_pisa_forward_host.argtypes = [PP, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_int32, P,
                                                  ctypes.c_size_t, P]
            lib.sla_pisa_forward_host.restype = ctypes.c_int
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load().sla_status_string(int(code)).decode()


def params(B, H, N, d, Bq, Bk, topk, sm_scale=0.0, sparse_dtype=SLA_SPARSE_BF16,
           lut_mode=SLA_LUT_COMPUTE, out_dtype=SLA_OUT_BF16, pisa_first_order=False,
           pisa_cov_lambda=0.0) -> SlaParams:
    return SlaParams(B, H, N, d, Bq, Bk, topk, float(sm_scale), sparse_dtype, lut_mode,
                     out_dtype, 1 if pisa_first_order else 0, float(pisa_cov_lambda))


def out_torch_dtype(p: SlaParams):
    return torch.float32 if p.out_dtype == SLA_OUT_FP32 else torch.bfloat16


def _ptr(t):
    if t is None or t.numel() == 0:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if t.device.index != torch.cuda.current_device():
        # the kernels run on the current device and would dereference another GPU's address
        raise ValueError("tensor is on %s but the current device is cuda:%d"
                         % (t.device, torch.cuda.current_device()))
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _nbytes(t):
    return t.numel() * t.element_size()


def _check(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device.index != torch.cuda.current_device():
        raise ValueError("stream is on %s but the current device is cuda:%d"
                         % (stream.device, torch.cuda.current_device()))
    return ctypes.c_void_p(stream.cuda_stream)


def sla_workspace_size(p: SlaParams) -> int:
    return int(load().sla_workspace_size(ctypes.byref(p)))


def workspace(p: SlaParams, device=None) -> torch.Tensor:
    """A workspace tensor large enough for every call with these parameters."""
    n = sla_workspace_size(p)
    if n == 0:
        raise SlaError(SLA_ERR_INVALID_ARG, "sla_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _raise(code, where):
    if code != SLA_OK:
        raise SlaError(code, where)


def sla_route(p, q, k, w_q, w_k, lut, ws, stream=None):
    """Writes the top-k block LUT [B,H,N/Bq,topk] (int32, ascending) into ``lut``."""
    B, H, N, d = p.B, p.H, p.N, p.d
    _check(q, torch.bfloat16, (B, H, N, d), "q")
    _check(k, torch.bfloat16, (B, H, N, d), "k")
    _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_route(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k), _ptr(lut),
                          _ptr(ws), _nbytes(ws), _stream(stream))
    _raise(rc, "sla_route")
    return lut


def sla_route_noalloc(p, q, k, w_q, w_k, lut, stream=None):
    """sla_route without a workspace: scratch comes from the library's built-in
    32 MiB device array (see include/sla.h)."""
    B, H, N, d = p.B, p.H, p.N, p.d
    _check(q, torch.bfloat16, (B, H, N, d), "q")
    _check(k, torch.bfloat16, (B, H, N, d), "k")
    _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_route_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(w_q), _ptr(w_k),
                                  _ptr(lut), _stream(stream))
    _raise(rc, "sla_route_noalloc")
    return lut


def sla_forward(p, q, k, v, alpha, w_q, w_k, lut, out, ws, stream=None):
    """SLA2 forward into ``out`` [B,H,N,d] bf16.  ``lut`` is written (LUT_COMPUTE,
    may be None) or read (LUT_GIVEN)."""
    B, H, N, d = p.B, p.H, p.N, p.d
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, torch.bfloat16, (B, H, N, d), name)
    _check(out, out_torch_dtype(p), (B, H, N, d), "out")
    _check(alpha, torch.float32, (B, H, N), "alpha")
    if lut is not None:
        _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(w_q),
                            _ptr(w_k), _ptr(lut), _ptr(out), _ptr(ws), _nbytes(ws),
                            _stream(stream))
    _raise(rc, "sla_forward")
    return out


def _hptr(t):
    """A host (CPU) tensor's address; pinned memory lets the copies overlap."""
    if t is None or t.numel() == 0:
        return None
    if t.is_cuda:
        raise ValueError("tensor must be in host memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def sla_forward_host(p, q_h, k_h, v_h, alpha_h, out_h, q, k, v, alpha, out, w_q, w_k, lut, ws,
                     heads_per_chunk=0, stream=None):
    """sla_forward with host inputs and output: chunks of heads are copied into
    the device buffers q, k, v, alpha, computed into ``out`` and copied back into
    ``out_h``, the copies overlapping the computation."""
    B, H, N, d = p.B, p.H, p.N, p.d
    for name, t in (("q_h", q_h), ("k_h", k_h), ("v_h", v_h), ("q", q), ("k", k), ("v", v)):
        _check(t, torch.bfloat16, (B, H, N, d), name)
    for name, t in (("alpha_h", alpha_h), ("alpha", alpha)):
        _check(t, torch.float32, (B, H, N), name)
    for name, t in (("out_h", out_h), ("out", out)):
        _check(t, out_torch_dtype(p), (B, H, N, d), name)
    if lut is not None:
        _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_forward_host(ctypes.byref(p), _hptr(q_h), _hptr(k_h), _hptr(v_h), _hptr(alpha_h),
                                 _hptr(out_h), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(out),
                                 _ptr(w_q), _ptr(w_k), _ptr(lut), int(heads_per_chunk), _ptr(ws),
                                 _nbytes(ws), _stream(stream))
    _raise(rc, "sla_forward_host")
    return out_h


def sla_pisa_forward_host(p, q_h, k_h, v_h, out_h, q, k, v, out, w_q, w_k, lut, ws,
                          heads_per_chunk=0, stream=None):
    """sla_pisa_forward with host inputs and output (see sla_forward_host)."""
    B, H, N, d = p.B, p.H, p.N, p.d
    for name, t in (("q_h", q_h), ("k_h", k_h), ("v_h", v_h), ("q", q), ("k", k), ("v", v)):
        _check(t, torch.bfloat16, (B, H, N, d), name)
    for name, t in (("out_h", out_h), ("out", out)):
        _check(t, out_torch_dtype(p), (B, H, N, d), name)
    if lut is not None:
        _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_pisa_forward_host(ctypes.byref(p), _hptr(q_h), _hptr(k_h), _hptr(v_h), _hptr(out_h),
                                      _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(w_q), _ptr(w_k),
                                      _ptr(lut), int(heads_per_chunk), _ptr(ws), _nbytes(ws),
                                      _stream(stream))
    _raise(rc, "sla_pisa_forward_host")
    return out_h


def sla_pisa_cov_norms(p, k, v, norms, ws, stream=None):
    """Block covariance norms M_j = ||H_j - Hbar||_2 into ``norms`` (fp64
    [B,H,N/Bk]); needs p.pisa_cov_lambda > 0."""
    B, H, N, d = p.B, p.H, p.N, p.d
    for name, t in (("k", k), ("v", v)):
        _check(t, torch.bfloat16, (B, H, N, d), name)
    _check(norms, torch.float64, (B, H, N // p.Bk), "norms")
    rc = load().sla_pisa_cov_norms(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(norms), _ptr(ws),
                                   _nbytes(ws), _stream(stream))
    _raise(rc, "sla_pisa_cov_norms")
    return norms


def sla_pisa_forward(p, q, k, v, w_q, w_k, lut, out, ws, stream=None):
    """PISA zero-order exact-or-approximate forward into ``out``."""
    B, H, N, d = p.B, p.H, p.N, p.d
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check(t, torch.bfloat16, (B, H, N, d), name)
    _check(out, out_torch_dtype(p), (B, H, N, d), "out")
    if lut is not None:
        _check(lut, torch.int32, (B, H, N // p.Bq, p.topk), "lut")
    rc = load().sla_pisa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(w_q),
                                 _ptr(w_k), _ptr(lut), _ptr(out), _ptr(ws), _nbytes(ws),
                                 _stream(stream))
    _raise(rc, "sla_pisa_forward")
    return out


def sla_check_device_status(stream=None) -> int:
    return int(load().sla_check_device_status(_stream(stream)))


def sla_profile_enable(on: bool = True) -> None:
    _raise(load().sla_profile_enable(1 if on else 0), "sla_profile_enable")


def sla_profile_read():
    """{kind: (total ms, count)} since the last read (synchronises).  Kernel kinds
    count launches; the phase kinds (PHASE_KINDS) count calls."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _raise(load().sla_profile_read(ctypes.cast(ms, ctypes.c_void_p), ctypes.cast(cnt, ctypes.c_void_p)),
           "sla_profile_read")
    return {KERNEL_KINDS[i]: (ms[i], cnt[i]) for i in range(n)}


def cocluster_workspace(p: SlaParams, n_clusters: int, device=None) -> torch.Tensor:
    """A workspace tensor for sla_cocluster with these parameters."""
    n = int(load().sla_cocluster_workspace_size(ctypes.byref(p), int(n_clusters)))
    if n == 0:
        raise SlaError(SLA_ERR_INVALID_ARG, "sla_cocluster_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sla_cocluster(p, q, k, n_clusters, iters, q_perm, k_perm, ws, stream=None):
    """SVOO bidirectional co-clustering: writes the stable orders of the queries
    and keys by cluster into q_perm, k_perm (int32 [B,H,N])."""
    B, H, N, d = p.B, p.H, p.N, p.d
    _check(q, torch.bfloat16, (B, H, N, d), "q")
    _check(k, torch.bfloat16, (B, H, N, d), "k")
    _check(q_perm, torch.int32, (B, H, N), "q_perm")
    _check(k_perm, torch.int32, (B, H, N), "k_perm")
    rc = load().sla_cocluster(ctypes.byref(p), _ptr(q), _ptr(k), int(n_clusters), int(iters), _ptr(q_perm),
                              _ptr(k_perm), _ptr(ws), _nbytes(ws), _stream(stream))
    _raise(rc, "sla_cocluster")
    return q_perm, k_perm


def sla_permute_rows(src, perm, dst, inverse=False, stream=None):
    """dst[..., i, :] = src[..., perm[..., i], :] (inverse: the scatter back).
    src, dst: [B, H, N, ...] contiguous (a trailing row of any size, or none);
    perm: int32 [B, H, N]."""
    if src.shape != dst.shape or src.dtype != dst.dtype:
        raise ValueError("src and dst must have one shape and dtype")
    B, H, N = perm.shape
    if tuple(src.shape[:3]) != (B, H, N) or perm.dtype != torch.int32:
        raise ValueError("perm must be int32 [B, H, N] matching src")
    row_bytes = src[0, 0, 0].numel() * src.element_size()
    rc = load().sla_permute_rows(_ptr(src), _ptr(perm), _ptr(dst), B * H, N, row_bytes,
                                 1 if inverse else 0, _stream(stream))
    _raise(rc, "sla_permute_rows")
    return dst


def sla_forward_coclustered(p, q, k, v, alpha, w_q, w_k, q_perm, k_perm, lut, out, ws, scratch=None,
                            stream=None):
    """sla_forward in the co-clustered order: Q and alpha gathered by q_perm, K and
    V by k_perm (into scratch, a dict of tensors shaped like q, k, v, alpha and
    out, allocated here if not given), the forward on them, and the output rows
    scattered back by q_perm.  Every step runs in the library's kernels."""
    if scratch is None:
        scratch = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
                   "alpha": torch.empty_like(alpha), "out": torch.empty_like(out)}
    sla_permute_rows(q, q_perm, scratch["q"], stream=stream)
    sla_permute_rows(alpha, q_perm, scratch["alpha"], stream=stream)
    sla_permute_rows(k, k_perm, scratch["k"], stream=stream)
    sla_permute_rows(v, k_perm, scratch["v"], stream=stream)
    sla_forward(p, scratch["q"], scratch["k"], scratch["v"], scratch["alpha"], w_q, w_k, lut, scratch["out"], ws,
                stream)
    sla_permute_rows(scratch["out"], q_perm, out, inverse=True, stream=stream)
    return out

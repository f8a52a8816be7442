"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, and rejects bad arguments before
anything is enqueued (so no call here touches a device)."""
import ctypes
import os
import re

import pytest

from block_sparse_linear_proj_b200 import build as B
from block_sparse_linear_proj_b200 import sla as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return S.load()


def header_functions():
    txt = open(os.path.join(ROOT, "include", "sla.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sla_[a-z_]+)\s*\(", txt)))


def test_header_declares_the_calls():
    fns = header_functions()
    for name in ("sla_route", "sla_forward", "sla_pisa_forward", "sla_workspace_size",
                 "sla_status_string", "sla_check_device_status"):
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(7):
        assert S.status_string(code)
    assert lib.sla_version() >= 100


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced: validation fails first


def call_route(p, q=FAKE, k=FAKE, lut=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return S.load().sla_route(ctypes.byref(p), q, k, None, None, lut, ws, ws_bytes, None)


def call_forward(p, q=FAKE, k=FAKE, v=FAKE, alpha=FAKE, lut=FAKE, out=FAKE, ws=FAKE,
                 ws_bytes=1 << 40):
    return S.load().sla_forward(ctypes.byref(p), q, k, v, alpha, None, None, lut, out, ws,
                                ws_bytes, None)


def call_pisa(p, ws_bytes=1 << 40, lut=FAKE):
    return S.load().sla_pisa_forward(ctypes.byref(p), FAKE, FAKE, FAKE, None, None, lut, FAKE,
                                     FAKE, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(N=1000), S.SLA_ERR_INVALID_ARG),            # N % Bq != 0
    (dict(topk=17), S.SLA_ERR_INVALID_ARG),           # topk > Nk
    (dict(topk=-1), S.SLA_ERR_INVALID_ARG),
    (dict(B=0), S.SLA_ERR_INVALID_ARG),
    (dict(d=96), S.SLA_ERR_UNSUPPORTED),
    (dict(Bq=32), S.SLA_ERR_UNSUPPORTED),
    (dict(Bk=128, N=1024, topk=2), S.SLA_ERR_UNSUPPORTED),
    (dict(sparse_dtype=7), S.SLA_ERR_INVALID_ARG),
    (dict(sparse_dtype=3), S.SLA_ERR_INVALID_ARG),
    (dict(lut_mode=3), S.SLA_ERR_INVALID_ARG),
])
def test_parameter_validation(lib, kw, code):
    base = dict(B=1, H=2, N=1024, d=64, Bq=64, Bk=64, topk=4)
    base.update(kw)
    extra = {k: base.pop(k) for k in ("sparse_dtype", "lut_mode") if k in base}
    p = S.params(**base, **extra)
    assert call_route(p) == code
    assert call_forward(p) == code
    assert lib.sla_workspace_size(ctypes.byref(p)) == 0


def test_pointer_validation(lib):
    p = S.params(1, 2, 1024, 64, 64, 64, 4)
    assert call_route(p, q=None) == S.SLA_ERR_INVALID_ARG
    assert call_route(p, k=ctypes.c_void_p((1 << 20) + 2)) == S.SLA_ERR_INVALID_ARG
    assert call_forward(p, v=None) == S.SLA_ERR_INVALID_ARG
    assert call_forward(p, alpha=None) == S.SLA_ERR_INVALID_ARG
    assert call_forward(p, out=ctypes.c_void_p((1 << 20) + 8)) == S.SLA_ERR_INVALID_ARG
    pg = S.params(1, 2, 1024, 64, 64, 64, 4, lut_mode=S.SLA_LUT_GIVEN)
    assert call_forward(pg, lut=None) == S.SLA_ERR_INVALID_ARG


def test_workspace_validation(lib):
    p = S.params(1, 2, 1024, 64, 64, 64, 4)
    need = lib.sla_workspace_size(ctypes.byref(p))
    assert need > 0
    assert call_route(p, ws_bytes=need - 1) == S.SLA_ERR_WORKSPACE
    assert call_route(p, ws=None) == S.SLA_ERR_WORKSPACE
    assert call_route(p, ws=ctypes.c_void_p((1 << 20) + 128)) == S.SLA_ERR_WORKSPACE
    assert call_forward(p, ws_bytes=need - 1) == S.SLA_ERR_WORKSPACE


def test_mode_restrictions(lib):
    # PISA needs Bq == Bk and the bf16 sparse branch
    assert call_pisa(S.params(1, 2, 1024, 64, 128, 64, 4)) == S.SLA_ERR_UNSUPPORTED
    assert call_pisa(S.params(1, 2, 1024, 64, 64, 64, 4, sparse_dtype=1)) == S.SLA_ERR_UNSUPPORTED
    assert call_pisa(S.params(1, 2, 1024, 64, 64, 64, 4, sparse_dtype=S.SLA_SPARSE_INT8)) == \
        S.SLA_ERR_UNSUPPORTED
    # the FP8 and INT8 sparse branches need d = 128 and Bq = 128
    for sd in (S.SLA_SPARSE_FP8_E4M3, S.SLA_SPARSE_INT8):
        assert call_forward(S.params(1, 2, 1024, 64, 64, 64, 4, sparse_dtype=sd)) == S.SLA_ERR_UNSUPPORTED
        assert call_forward(S.params(1, 2, 1024, 128, 64, 64, 4, sparse_dtype=sd)) == S.SLA_ERR_UNSUPPORTED


def test_int8_workspace_matches_fp8(lib):
    # both 8-bit branches keep the same code and scale buffers
    sizes = [lib.sla_workspace_size(ctypes.byref(S.params(1, 4, 4096, 128, 128, 64, 8, sparse_dtype=sd)))
             for sd in (S.SLA_SPARSE_BF16, S.SLA_SPARSE_FP8_E4M3, S.SLA_SPARSE_INT8)]
    assert sizes[1] == sizes[2] > sizes[0]


def test_workspace_size_grows_with_problem(lib):
    small = S.params(1, 2, 1024, 64, 64, 64, 4)
    big = S.params(1, 12, 32768, 128, 128, 64, 52)
    assert lib.sla_workspace_size(ctypes.byref(big)) > lib.sla_workspace_size(ctypes.byref(small))


def test_cov_selection_arguments(lib):
    # lambda must be finite and >= 0
    for lam in (-1.0, float("nan"), float("inf")):
        p = S.params(1, 2, 1024, 64, 64, 64, 4, pisa_cov_lambda=lam)
        assert call_route(p) == S.SLA_ERR_INVALID_ARG
        assert lib.sla_workspace_size(ctypes.byref(p)) == 0
    # a PISA selection option: sla_forward and the routing calls reject it
    with_lam = S.params(1, 2, 1024, 64, 64, 64, 4, pisa_cov_lambda=0.5)
    assert call_forward(with_lam) == S.SLA_ERR_INVALID_ARG
    assert call_route(with_lam) == S.SLA_ERR_INVALID_ARG
    assert lib.sla_route_noalloc(ctypes.byref(with_lam), FAKE, FAKE, None, None, FAKE, None) == \
        S.SLA_ERR_INVALID_ARG
    # the norms need lambda > 0 (the workspace holds their scratch then) and 8-byte aligned output
    p0 = S.params(1, 2, 1024, 64, 64, 64, 4)
    assert lib.sla_pisa_cov_norms(ctypes.byref(p0), FAKE, FAKE, FAKE, FAKE, 1 << 40, None) == \
        S.SLA_ERR_INVALID_ARG
    p1 = S.params(1, 2, 1024, 64, 64, 64, 4, pisa_cov_lambda=0.1)
    assert lib.sla_pisa_cov_norms(ctypes.byref(p1), FAKE, FAKE, ctypes.c_void_p((1 << 20) + 4),
                                  FAKE, 1 << 40, None) == S.SLA_ERR_INVALID_ARG
    # the selection term's scratch enlarges the workspace
    with_cov = S.params(1, 24, 32768, 128, 64, 64, 77, pisa_cov_lambda=0.1)
    plain = S.params(1, 24, 32768, 128, 64, 64, 77)
    assert lib.sla_workspace_size(ctypes.byref(with_cov)) > lib.sla_workspace_size(ctypes.byref(plain))


def test_cov_norms_wrapper_checks_arguments():
    import torch
    from block_sparse_linear_proj_b200 import sla as SL
    p = SL.params(1, 1, 1024, 64, 64, 64, 4, pisa_cov_lambda=0.1)
    k = torch.zeros(1, 1, 1024, 64, dtype=torch.bfloat16)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError):          # norms must be fp64
        SL.sla_pisa_cov_norms(p, k, k, torch.zeros(1, 1, 16, dtype=torch.float32), ws)
    with pytest.raises(ValueError):         # one norm per KV block
        SL.sla_pisa_cov_norms(p, k, k, torch.zeros(1, 1, 15, dtype=torch.float64), ws)
    with pytest.raises(TypeError):          # bf16 keys
        SL.sla_pisa_cov_norms(p, k.float(), k, torch.zeros(1, 1, 16, dtype=torch.float64), ws)


def test_cocluster_argument_checks(lib):
    p = S.params(1, 2, 1024, 64, 64, 64, 4)
    need = lib.sla_cocluster_workspace_size(ctypes.byref(p), 16)
    assert need > 0
    assert lib.sla_cocluster_workspace_size(ctypes.byref(p), 3) == 0        # must divide N
    assert lib.sla_cocluster_workspace_size(ctypes.byref(p), 2048) == 0     # more clusters than tokens
    call = lambda C, it, ws_bytes=1 << 40, q=FAKE, qp=FAKE: lib.sla_cocluster(
        ctypes.byref(p), q, FAKE, C, it, qp, FAKE, FAKE, ws_bytes, None)
    assert call(16, 0) == S.SLA_ERR_INVALID_ARG                              # at least one iteration
    assert call(16, 65) == S.SLA_ERR_INVALID_ARG
    assert call(5, 3) == S.SLA_ERR_INVALID_ARG
    assert call(16, 3, q=None) == S.SLA_ERR_INVALID_ARG
    assert call(16, 3, qp=ctypes.c_void_p((1 << 20) + 2)) == S.SLA_ERR_INVALID_ARG
    assert call(16, 3, ws_bytes=need - 1) == S.SLA_ERR_WORKSPACE
    big = S.params(1, 1, 4096, 64, 64, 64, 4)
    assert lib.sla_cocluster_workspace_size(ctypes.byref(big), 2048) == 0   # more than 1024 clusters


def test_permute_rows_argument_checks(lib):
    f = lib.sla_permute_rows
    A, B2 = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    assert f(A, FAKE, A, 2, 64, 256, 0, None) == S.SLA_ERR_INVALID_ARG          # in place
    assert f(A, FAKE, B2, 2, 64, 6, 0, None) == S.SLA_ERR_INVALID_ARG           # not whole words
    assert f(A, FAKE, B2, 2, 64, 256, 2, None) == S.SLA_ERR_INVALID_ARG         # inverse is 0 or 1
    assert f(A, None, B2, 2, 64, 256, 0, None) == S.SLA_ERR_INVALID_ARG
    assert f(ctypes.c_void_p((1 << 20) + 2), FAKE, B2, 2, 64, 4, 0, None) == S.SLA_ERR_INVALID_ARG
    assert f(A, FAKE, B2, 0, 64, 256, 0, None) == S.SLA_ERR_INVALID_ARG
    assert f(A, FAKE, B2, 2, 64, 8192, 0, None) == S.SLA_ERR_INVALID_ARG


@pytest.mark.parametrize("N,d,Bq,topk", [(32768, 128, 128, 52), (8192, 64, 64, 16), (1024, 128, 64, 4)])
def test_workspace_size_never_falls_as_heads_grow(lib, N, d, Bq, topk):
    """A workspace for B*H heads serves a call over a subset of them (the
    host-buffer calls run chunks of heads in the whole problem's workspace).
    The pre-pass's chunks per head shrink as heads are added, so the partial
    sums are sized for the most that any smaller head count uses."""
    prev = 0
    for H in list(range(1, 40)) + [147, 148, 149, 295, 296, 297, 298, 591, 592, 593, 700]:
        need = lib.sla_workspace_size(ctypes.byref(S.params(1, H, N, d, Bq, 64, topk)))
        assert need >= prev, H
        prev = need
    # B and H enter only through B*H
    a = lib.sla_workspace_size(ctypes.byref(S.params(3, 99, N, d, Bq, 64, topk)))
    b = lib.sla_workspace_size(ctypes.byref(S.params(1, 297, N, d, Bq, 64, topk)))
    assert a == b


def call_forward_host(p, hpc=0, q_h=FAKE, alpha_h=FAKE, q=FAKE, lut=FAKE, ws=FAKE, ws_bytes=1 << 40):
    return S.load().sla_forward_host(ctypes.byref(p), q_h, FAKE, FAKE, alpha_h, FAKE, q, FAKE, FAKE, FAKE,
                                     FAKE, None, None, lut, hpc, ws, ws_bytes, None)


def call_pisa_host(p, hpc=0, out_h=FAKE, out=FAKE, ws_bytes=1 << 40):
    return S.load().sla_pisa_forward_host(ctypes.byref(p), FAKE, FAKE, FAKE, out_h, FAKE, FAKE, FAKE, out,
                                          None, None, FAKE, hpc, FAKE, ws_bytes, None)


def test_host_buffer_calls_check_arguments_before_enqueueing(lib):
    """Every rejection here returns before a stream, an event or a copy is
    touched: the whole problem is checked as the device call checks it."""
    p = S.params(1, 2, 1024, 64, 64, 64, 4)
    need = lib.sla_workspace_size(ctypes.byref(p))
    assert call_forward_host(S.params(1, 2, 1000, 64, 64, 64, 4)) == S.SLA_ERR_INVALID_ARG
    assert call_forward_host(p, q=ctypes.c_void_p((1 << 20) + 8)) == S.SLA_ERR_INVALID_ARG
    assert call_forward_host(p, ws_bytes=need - 1) == S.SLA_ERR_WORKSPACE
    assert call_forward_host(p, ws=None) == S.SLA_ERR_WORKSPACE
    assert call_forward_host(p, q_h=None) == S.SLA_ERR_INVALID_ARG
    assert call_forward_host(p, alpha_h=None) == S.SLA_ERR_INVALID_ARG
    assert call_forward_host(p, hpc=-1) == S.SLA_ERR_INVALID_ARG
    pg = S.params(1, 2, 1024, 64, 64, 64, 4, lut_mode=S.SLA_LUT_GIVEN)
    assert call_forward_host(pg, lut=None) == S.SLA_ERR_INVALID_ARG
    assert call_forward_host(S.params(1, 2, 1024, 64, 64, 64, 4, sparse_dtype=1)) == S.SLA_ERR_UNSUPPORTED
    pp = S.params(1, 2, 1024, 64, 64, 64, 4)
    assert call_pisa_host(S.params(1, 2, 1024, 64, 128, 64, 4)) == S.SLA_ERR_UNSUPPORTED
    assert call_pisa_host(pp, out=ctypes.c_void_p((1 << 20) + 4)) == S.SLA_ERR_INVALID_ARG
    assert call_pisa_host(pp, out_h=None) == S.SLA_ERR_INVALID_ARG
    assert call_pisa_host(pp, hpc=-3) == S.SLA_ERR_INVALID_ARG
    assert call_pisa_host(pp, ws_bytes=lib.sla_workspace_size(ctypes.byref(pp)) - 1) == S.SLA_ERR_WORKSPACE

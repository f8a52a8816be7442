"""Failure detection without a GPU fault.  With the test hook SLA_DEBUG_STALL
the attention kernel's loader issues no K/V tile loads (a flag that nothing
sets), so the consumers' bounded waits (limit set to 2 ms here) run out; the
kernel must report SLA_ERR_TIMEOUT through the device status word, drain its
own copies and products, release tensor memory and leave the context usable
for the next call, which must then be correct."""
import os

import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import check, dev, gpu_forward, params

pytestmark = pytest.mark.gpu


HOOK = {"SLA_DEBUG_STALL": "1", "SLA_DEBUG_WAIT_LIMIT_NS": "2000000"}


@pytest.fixture
def stalled_loader():
    old = {k: os.environ.get(k) for k in HOOK}
    os.environ.update(HOOK)
    yield
    for k, v in old.items():
        if v is None:
            del os.environ[k]
        else:
            os.environ[k] = v


def _run(p, g, lut):
    ws = S.workspace(p)
    out = torch.zeros_like(g["q"])
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"],
                  torch.as_tensor(lut).cuda(), out, ws)
    return S.sla_check_device_status(), out


@pytest.mark.parametrize("sd", [S.SLA_SPARSE_BF16, S.SLA_SPARSE_FP8_E4M3, S.SLA_SPARSE_INT8],
                         ids=["bf16", "fp8", "int8"])
def test_wait_expiry_reports_timeout_and_context_survives(sd):
    B, H, N, d, Bq, k = 1, 2, 2048, 128, 128, 6
    inp = W.gaussian_inputs(B, H, N, d, 91)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    g = dev(inp)
    p = params(B, H, N, d, Bq, 64, k, given=True, sparse_dtype=sd)
    old = {k: os.environ.get(k) for k in HOOK}
    os.environ.update(HOOK)
    try:
        status, _ = _run(p, g, lut)
    finally:
        for kk, v in old.items():
            if v is None:
                del os.environ[kk]
            else:
                os.environ[kk] = v
    assert status == S.sla.SLA_ERR_TIMEOUT
    # the context is intact: the same call with the normal limit is correct
    pf = params(B, H, N, d, Bq, 64, k, given=True, sparse_dtype=sd, f32=True)
    out = gpu_forward(pf, g, lut)
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, 64,
                          fp8=sd == S.SLA_SPARSE_FP8_E4M3, int8=sd == S.SLA_SPARSE_INT8)
    check(out, ref, pf, (2e-2, 2e-3) if sd == S.SLA_SPARSE_BF16 else (6e-2, 6e-3))


def test_pisa_wait_expiry(stalled_loader):
    B, H, N, d = 1, 2, 2048, 128
    inp = dev(W.gaussian_inputs(B, H, N, d, 92, use_w=False, with_alpha=False))
    p = params(B, H, N, d, 64, 64, 5)
    ws = S.workspace(p)
    lut = torch.empty((B, H, N // 64, 5), dtype=torch.int32, device="cuda")
    out = torch.zeros_like(inp["q"])
    S.sla_pisa_forward(p, inp["q"], inp["k"], inp["v"], None, None, lut, out, ws)
    assert S.sla_check_device_status() == S.sla.SLA_ERR_TIMEOUT

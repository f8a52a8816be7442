"""SLA2 forward parity on the GPU against the CPU oracle.

The oracle computes from its own LUT; the GPU receives that LUT through
LUT_GIVEN, so no oracle input ever comes from the CUDA path.  LUT_COMPUTE is
checked separately: its LUT against the oracle's and its output against the
LUT_GIVEN output.  Small shapes are compared on every element; the full
workloads on seeded row samples from a few heads (same launch configuration
as the benchmark)."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import (TOL_BF16, check, check_lut, dev, gpu_forward, gpu_route, new_out, params,
                      random_lut, rows_of)

pytestmark = pytest.mark.gpu


def full_lut(B, H, Nq, Nk):
    return np.broadcast_to(np.arange(Nk, dtype=np.int32), (B, H, Nq, Nk)).copy()


@pytest.mark.parametrize("B,H,N,d,Bq,k,alpha", [
    (1, 2, 1024, 64, 64, 4, "rand"),
    (1, 2, 1024, 128, 128, 4, "rand"),
    (2, 1, 2048, 128, 128, 7, "rand"),
    (1, 2, 1088, 64, 64, 3, "rand"),           # odd Nq: last CTA holds one query block
    (1, 2, 1152, 128, 64, 5, "rand"),          # Bq = 64 with d = 128: two row groups per CTA
    (1, 2, 2048, 128, 128, 1, "rand"),
    (1, 2, 2048, 128, 128, 31, "rand"),        # k = Nk - 1
    (1, 1, 2048, 128, 128, 0, "zero"),         # k = 0, alpha = 0: pure linear attention
    (1, 1, 2048, 64, 64, 32, "one"),           # k = Nk, alpha = 1: dense attention
    (1, 1, 1024, 128, 128, 16, "rand"),        # k = Nk with alpha: linear branch empty
])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_forward_small(B, H, N, d, Bq, k, alpha, f32):
    inp = W.gaussian_inputs(B, H, N, d, 200 + N + k + d)
    if alpha == "zero":
        inp["alpha"] = torch.zeros(B, H, N)
    elif alpha == "one":
        inp["alpha"] = torch.ones(B, H, N)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, 64)
    p = params(B, H, N, d, Bq, 64, k, given=True, f32=f32)
    check(gpu_forward(p, dev(inp), lut), ref, p)


def test_forward_random_lut_and_scale():
    B, H, N, d, Bq, k = 1, 2, 2048, 128, 128, 6
    inp = W.gaussian_inputs(B, H, N, d, 31)
    lut = random_lut(B, H, N // Bq, N // 64, k, 3)
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, 64, sm_scale=0.05)
    p = params(B, H, N, d, Bq, 64, k, given=True, sm_scale=0.05, f32=True)
    check(gpu_forward(p, dev(inp), lut), ref, p)


@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_forward_tiny_workload_full(f32):
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], w.Bq, w.Bk, w.topk)
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, w.Bq, w.Bk)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk, given=True, f32=f32)
    print("tiny max/mean err (std units): %.3g %.3g" % check(gpu_forward(p, dev(inp), lut), ref, p))


@pytest.mark.parametrize("name,heads", [("sla2_bf16", [0, 7]), ("sla2_long", [3, 38])])
@pytest.mark.parametrize("f32", [False, True], ids=["out_bf16", "out_fp32"])
def test_forward_workload_sampled(name, heads, f32):
    """Full-size workload in the benchmark's launch configuration (LUT_COMPUTE),
    outputs checked on a seeded sample of rows from two heads."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    lut_ref, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], w.Bq, w.Bk, w.topk)
    g = dev(inp)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk, f32=f32)
    ws = S.workspace(p)
    lut_gpu = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut_gpu, out, ws)
    assert S.sla_check_device_status() == 0
    lg = lut_gpu.cpu().numpy()
    excl = check_lut(lg, lut_ref, gap, w.Nk)
    rows = W.sample_rows(w.B, w.H, w.N, 384, 5, heads=heads).numpy()
    # keep rows whose query block got the oracle's LUT row
    qb = (rows % w.N) // w.Bq
    bh = rows // w.N
    keep = ~excl.reshape(-1, w.Nq)[bh, qb]
    rows = rows[keep]
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut_ref, w.Bq, w.Bk, rows=rows)
    mx, mn = check(rows_of(out, rows), ref, p, TOL_BF16, name)
    print("%s: %d rows, max/mean err (std units) %.3g %.3g" % (name, len(rows), mx, mn))


def test_lut_compute_equals_lut_given():
    B, H, N, d, Bq, k = 1, 3, 4096, 128, 128, 7
    inp = dev(W.gaussian_inputs(B, H, N, d, 41))
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    p = params(B, H, N, d, Bq, 64, k)
    ws = S.workspace(p)
    out1 = torch.empty_like(inp["q"])
    S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["w_q"], inp["w_k"], lut, out1, ws)
    out2 = gpu_forward(params(B, H, N, d, Bq, 64, k, given=True), inp, lut.cpu().numpy())
    assert torch.equal(out1, out2)
    assert np.array_equal(lut.cpu().numpy(), gpu_route(p, inp))


def test_forward_deterministic():
    B, H, N, d, Bq, k = 1, 2, 4096, 128, 128, 9
    inp = dev(W.gaussian_inputs(B, H, N, d, 42))
    p = params(B, H, N, d, Bq, 64, k)
    a = gpu_forward(p, inp)
    b = gpu_forward(p, inp)
    assert torch.equal(a, b)


def test_invalid_lut_entries_are_flagged():
    B, H, N, d, Bq, k = 1, 1, 1024, 128, 128, 3
    inp = dev(W.gaussian_inputs(B, H, N, d, 43))
    lut = random_lut(B, H, N // Bq, N // 64, k, 1)
    lut[0, 0, 2, 1] = 99                      # out of range
    lut[0, 0, 5, 2] = lut[0, 0, 5, 0]         # repeated
    p = params(B, H, N, d, Bq, 64, k, given=True)
    ws = S.workspace(p)
    out = torch.empty_like(inp["q"])
    S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], None, None,
                  torch.as_tensor(lut).cuda(), out, ws)
    assert S.sla_check_device_status() == S.sla.SLA_ERR_DEVICE_CHECK
    assert S.sla_check_device_status() == S.sla.SLA_OK      # the status word is cleared on read

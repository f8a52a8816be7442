"""FP8 e4m3 sparse branch (Q, K, V, P quantised; linear branch and combine in
bf16/fp32).

Three oracles, on the same rows (gpu_util.check_lowbit): the oracle's FP8
forward with the kernel's reading of P's reference (the power of two at or
above the row maximum), against which the stated FP8 tolerance (max-abs 6e-2,
mean-abs 6e-3 in units of the output's standard deviation) applies; the FP8
forward with P against the row maximum itself, against which the tolerance
plus the two oracles' own distance applies; and the exact forward, from which
the GPU may be no further than the ideal quantised computation (mean error at
most 1.05x the second oracle's own plus 2e-3 for the unquantised linear
branch).  Both quantised oracles decide each code on the exact quotient
448 x / absmax, as the kernels do."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import (TOL_FP8, check, check_lowbit, check_lut, dev, err_units, gpu_forward, new_out,
                      params, random_lut, rows_of)

pytestmark = pytest.mark.gpu
FP8 = S.SLA_SPARSE_FP8_E4M3


def fp8_params(B, H, N, d, Bq, k, given=True, f32=True, sm_scale=0.0):
    return params(B, H, N, d, Bq, 64, k, given=given, sparse_dtype=FP8, f32=f32, sm_scale=sm_scale)


def check_fp8(out, inp, lut, Bq, p, sm_scale=0.0, rows=None, what="fp8"):
    """The three-oracle check of gpu_util.check_lowbit (stated tolerance against
    the quantised oracle with the kernel's reading of P's reference; against the
    one with P against the row maximum, plus the two oracles' distance; against
    the exact oracle, no worse than the ideal quantised computation)."""
    return check_lowbit(out, inp, lut, Bq, p, "fp8", sm_scale=sm_scale, rows=rows, what=what)


@pytest.mark.parametrize("B,H,N,k,alpha", [
    (1, 2, 1024, 4, "rand"),
    (2, 1, 2048, 7, "rand"),
    (1, 2, 1152, 5, "rand"),           # odd Nq
    (1, 2, 2048, 1, "rand"),
    (1, 2, 2048, 31, "rand"),          # k = Nk - 1
    (1, 1, 2048, 0, "zero"),           # k = 0, alpha = 0: pure linear attention
    (1, 1, 2048, 32, "one"),           # k = Nk, alpha = 1: dense attention in e4m3
])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_fp8_small(B, H, N, k, alpha, f32):
    d, Bq = 128, 128
    inp = W.gaussian_inputs(B, H, N, d, 500 + N + k)
    if alpha == "zero":
        inp["alpha"] = torch.zeros(B, H, N)
    elif alpha == "one":
        inp["alpha"] = torch.ones(B, H, N)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    p = fp8_params(B, H, N, d, Bq, k, f32=f32)
    check_fp8(gpu_forward(p, dev(inp), lut), inp, lut, Bq, p)


def test_fp8_random_lut_scale_and_zero_blocks():
    """Random LUT, a custom softmax scale, and all-zero K, V and Q blocks (scale 1)."""
    B, H, N, d, Bq, k = 1, 2, 2048, 128, 128, 6
    inp = W.gaussian_inputs(B, H, N, d, 33)
    inp["k"][0, 0, 64:128] = 0
    inp["v"][0, 1, 256:320] = 0
    inp["q"][0, 0, 512:576] = 0
    lut = random_lut(B, H, N // Bq, N // 64, k, 5)
    rng = np.random.default_rng(6)
    for i in range(N // Bq):                 # every row of head 0 selects the zero-K block 1
        others = rng.choice(np.delete(np.arange(N // 64), 1), size=k - 1, replace=False)
        lut[0, 0, i] = np.sort(np.append(others, 1))
    p = fp8_params(B, H, N, d, Bq, k, sm_scale=0.06)
    check_fp8(gpu_forward(p, dev(inp), lut), inp, lut, Bq, p, sm_scale=0.06, what="fp8 zero blocks")


def test_fp8_lut_compute_matches_given_and_is_deterministic():
    B, H, N, d, Bq, k = 1, 2, 4096, 128, 128, 9
    inp = dev(W.gaussian_inputs(B, H, N, d, 44))
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    p = fp8_params(B, H, N, d, Bq, k, given=False, f32=False)
    ws = S.workspace(p)
    out1 = new_out(p, inp["q"])
    S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["w_q"], inp["w_k"], lut, out1, ws)
    assert S.sla_check_device_status() == 0
    out2 = gpu_forward(fp8_params(B, H, N, d, Bq, k, f32=False), inp, lut.cpu().numpy())
    assert torch.equal(out1, out2)
    out3 = gpu_forward(fp8_params(B, H, N, d, Bq, k, f32=False), inp, lut.cpu().numpy())
    assert torch.equal(out2, out3)


def test_fp8_differs_from_bf16_path():
    """The FP8 call really runs the quantised branch (its error is not the bf16 one)."""
    B, H, N, d, Bq, k = 1, 1, 2048, 128, 128, 8
    inp = W.gaussian_inputs(B, H, N, d, 45)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    g = dev(inp)
    o8 = gpu_forward(fp8_params(B, H, N, d, Bq, k), g, lut)
    o16 = gpu_forward(params(B, H, N, d, Bq, 64, k, given=True, f32=True), g, lut)
    assert not torch.equal(o8, o16)


@pytest.mark.parametrize("d,Bq", [(64, 64), (128, 64)])
def test_fp8_unsupported_shapes(d, Bq):
    B, H, N, k = 1, 1, 1024, 2
    inp = dev(W.gaussian_inputs(B, H, N, d, 46))
    p = fp8_params(B, H, N, d, Bq, k, given=False)
    ws = S.workspace(p)
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    out = new_out(p, inp["q"])
    with pytest.raises(S.SlaError) as ei:
        S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["w_q"], inp["w_k"], lut, out, ws)
    assert ei.value.code == S.sla.SLA_ERR_UNSUPPORTED


@pytest.mark.parametrize("f32", [False, True], ids=["out_bf16", "out_fp32"])
def test_fp8_workload_sampled(f32):
    """The FP8 video workload in the benchmark's launch configuration, sampled rows."""
    w = W.WORKLOADS["sla2_fp8"]
    inp = W.make_inputs(w)
    lut_ref, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], w.Bq, w.Bk, w.topk)
    g = dev(inp)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk, sparse_dtype=FP8, f32=f32)
    ws = S.workspace(p)
    lut_gpu = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut_gpu, out, ws)
    assert S.sla_check_device_status() == 0
    excl = check_lut(lut_gpu.cpu().numpy(), lut_ref, gap, w.Nk)
    rows = W.sample_rows(w.B, w.H, w.N, 384, 7, heads=[2, 9]).numpy()
    keep = ~excl.reshape(-1, w.Nq)[rows // w.N, (rows % w.N) // w.Bq]
    rows = rows[keep]
    print("sla2_fp8: %d rows" % len(rows))
    check_fp8(out, inp, lut_ref, w.Bq, p, rows=rows, what="sla2_fp8")

"""INT8 sparse branch: symmetric 8-bit integer Q and K codes (exact s32 scores),
e4m3 P and V; the linear branch and the combine stay bf16/fp32.

Three oracles, on the same rows (gpu_util.check_lowbit), as for the FP8
branch: the oracle's INT8 forward with the kernel's reading of P's reference
(stated FP8 tolerance, max-abs 6e-2 and mean-abs 6e-3 in units of the output's
standard deviation), the INT8 forward with P against the row maximum itself
(the tolerance plus the two oracles' distance), and the exact forward (mean
error at most 1.05x the second oracle's own plus 2e-3).  Q and K codes round
the exact quotient 127 x / absmax on both sides."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import (TOL_FP8, check, check_lowbit, check_lut, dev, err_units, gpu_forward, new_out,
                      params, random_lut, rows_of)

pytestmark = pytest.mark.gpu
INT8 = S.SLA_SPARSE_INT8


def int8_params(B, H, N, d, Bq, k, given=True, f32=True, sm_scale=0.0):
    return params(B, H, N, d, Bq, 64, k, given=given, sparse_dtype=INT8, f32=f32, sm_scale=sm_scale)


def check_int8(out, inp, lut, Bq, p, sm_scale=0.0, rows=None, what="int8"):
    """The three-oracle check of gpu_util.check_lowbit (stated tolerance against
    the quantised oracle with the kernel's reading of P's reference; against the
    one with P against the row maximum, plus the two oracles' distance; against
    the exact oracle, no worse than the ideal quantised computation)."""
    return check_lowbit(out, inp, lut, Bq, p, "int8", sm_scale=sm_scale, rows=rows, what=what)


@pytest.mark.parametrize("B,H,N,k,alpha", [
    (1, 2, 1024, 4, "rand"),
    (2, 1, 2048, 7, "rand"),
    (1, 2, 1152, 5, "rand"),           # odd Nq
    (1, 2, 2048, 1, "rand"),
    (1, 2, 2048, 31, "rand"),          # k = Nk - 1
    (1, 1, 2048, 0, "zero"),           # k = 0, alpha = 0: pure linear attention
    (1, 1, 2048, 32, "one"),           # k = Nk, alpha = 1: dense attention, 8-bit
])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_int8_small(B, H, N, k, alpha, f32):
    d, Bq = 128, 128
    inp = W.gaussian_inputs(B, H, N, d, 700 + N + k)
    if alpha == "zero":
        inp["alpha"] = torch.zeros(B, H, N)
    elif alpha == "one":
        inp["alpha"] = torch.ones(B, H, N)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    p = int8_params(B, H, N, d, Bq, k, f32=f32)
    check_int8(gpu_forward(p, dev(inp), lut), inp, lut, Bq, p)


def test_int8_exact_integer_inputs():
    """Q and K whose blocks hold integers of absmax 127 (scale exactly 1, codes
    the values themselves), so S is the exact integer product: the GPU's error
    is then only the e4m3 P, V and the output rounding, as the oracle's."""
    B, H, N, d, Bq, k = 1, 2, 2048, 128, 128, 8
    inp = W.gaussian_inputs(B, H, N, d, 71)
    g = torch.Generator().manual_seed(72)
    for name in ("q", "k"):
        x = torch.randint(-127, 128, (B, H, N, d), generator=g).float()
        x[..., 0] = 127.0                                   # every 64-token block: absmax 127
        inp[name] = x.to(torch.bfloat16)                    # integers up to 256 are exact in bf16
    lut = random_lut(B, H, N // Bq, N // 64, k, 73)
    # logits of a few units, never whole numbers: a whole-number log2 logit makes
    # its P an exact power of two, and P * 448 s_v,j / s_v,max can then sit exactly
    # on an e4m3 rounding midpoint (bf16 absmax ratios such as 25/28 are common),
    # a tie that fp32 and fp64 arithmetic may break either way
    sm = 1.3 / 127.0 ** 2
    p = int8_params(B, H, N, d, Bq, k, sm_scale=sm)
    check_int8(gpu_forward(p, dev(inp), lut), inp, lut, Bq, p, sm_scale=sm, what="int8 integer inputs")


def test_int8_random_lut_scale_and_zero_blocks():
    """Random LUT, a custom softmax scale, and all-zero K, V and Q blocks (scale 1)."""
    B, H, N, d, Bq, k = 1, 2, 2048, 128, 128, 6
    inp = W.gaussian_inputs(B, H, N, d, 74)
    inp["k"][0, 0, 64:128] = 0
    inp["v"][0, 1, 256:320] = 0
    inp["q"][0, 0, 512:576] = 0
    lut = random_lut(B, H, N // Bq, N // 64, k, 75)
    rng = np.random.default_rng(76)
    for i in range(N // Bq):                 # every row of head 0 selects the zero-K block 1
        others = rng.choice(np.delete(np.arange(N // 64), 1), size=k - 1, replace=False)
        lut[0, 0, i] = np.sort(np.append(others, 1))
    p = int8_params(B, H, N, d, Bq, k, sm_scale=0.06)
    check_int8(gpu_forward(p, dev(inp), lut), inp, lut, Bq, p, sm_scale=0.06, what="int8 zero blocks")


def test_int8_lut_compute_matches_given_and_is_deterministic():
    B, H, N, d, Bq, k = 1, 2, 4096, 128, 128, 9
    inp = dev(W.gaussian_inputs(B, H, N, d, 77))
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    p = int8_params(B, H, N, d, Bq, k, given=False, f32=False)
    ws = S.workspace(p)
    out1 = new_out(p, inp["q"])
    S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["w_q"], inp["w_k"], lut, out1, ws)
    assert S.sla_check_device_status() == 0
    out2 = gpu_forward(int8_params(B, H, N, d, Bq, k, f32=False), inp, lut.cpu().numpy())
    assert torch.equal(out1, out2)
    out3 = gpu_forward(int8_params(B, H, N, d, Bq, k, f32=False), inp, lut.cpu().numpy())
    assert torch.equal(out2, out3)


def test_int8_differs_from_fp8_path():
    """The INT8 call really runs the integer product: its output is not the FP8 one,
    and it is closer to the exact forward (8-bit integers carry 3 more bits than
    the e4m3 mantissa over a block's range)."""
    B, H, N, d, Bq, k = 1, 1, 2048, 128, 128, 8
    inp = W.gaussian_inputs(B, H, N, d, 78)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    g = dev(inp)
    oi = gpu_forward(int8_params(B, H, N, d, Bq, k), g, lut)
    of = gpu_forward(params(B, H, N, d, Bq, 64, k, given=True, sparse_dtype=S.SLA_SPARSE_FP8_E4M3,
                            f32=True), g, lut)
    assert not torch.equal(oi, of)
    exact = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, 64)
    ei = err_units(oi.double().cpu().numpy(), exact)
    ef = err_units(of.double().cpu().numpy(), exact)
    print("vs exact: int8 %.3g/%.3g, fp8 %.3g/%.3g" % (ei + ef))
    assert ei[1] <= ef[1]


@pytest.mark.parametrize("d,Bq", [(64, 64), (128, 64)])
def test_int8_unsupported_shapes(d, Bq):
    B, H, N, k = 1, 1, 1024, 2
    inp = dev(W.gaussian_inputs(B, H, N, d, 79))
    p = int8_params(B, H, N, d, Bq, k, given=False)
    ws = S.workspace(p)
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    out = new_out(p, inp["q"])
    with pytest.raises(S.SlaError) as ei:
        S.sla_forward(p, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["w_q"], inp["w_k"], lut, out, ws)
    assert ei.value.code == S.sla.SLA_ERR_UNSUPPORTED


@pytest.mark.parametrize("f32", [False, True], ids=["out_bf16", "out_fp32"])
def test_int8_workload_sampled(f32):
    """The INT8 video workload in the benchmark's launch configuration, sampled rows."""
    w = W.WORKLOADS["sla2_int8"]
    inp = W.make_inputs(w)
    lut_ref, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], w.Bq, w.Bk, w.topk)
    g = dev(inp)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk, sparse_dtype=INT8, f32=f32)
    ws = S.workspace(p)
    lut_gpu = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut_gpu, out, ws)
    assert S.sla_check_device_status() == 0
    excl = check_lut(lut_gpu.cpu().numpy(), lut_ref, gap, w.Nk)
    rows = W.sample_rows(w.B, w.H, w.N, 384, 8, heads=[3, 10]).numpy()
    keep = ~excl.reshape(-1, w.Nq)[rows // w.N, (rows % w.N) // w.Bq]
    rows = rows[keep]
    print("sla2_int8: %d rows" % len(rows))
    check_int8(out, inp, lut_ref, w.Bq, p, rows=rows, what="sla2_int8")

"""PISA zero-order exact-or-approximate forward: GPU against the oracle, and
the mathematical special cases run through the real kernels."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc

from gpu_util import TOL_BF16, check, check_lut, dev, gpu_pisa, new_out, params, rows_of
import block_sparse_linear_proj_b200 as S

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,k", [
    (1, 2, 1024, 64, 4),
    (1, 2, 2048, 128, 5),
    (2, 1, 1088, 128, 3),       # odd Nq
    (1, 2, 2048, 128, 0),       # only centroids
    (1, 1, 1024, 128, 16),      # every block exact: dense attention
    (1, 1, 4160, 128, 9),       # Nk = 65: ragged centroid pseudo-tile
])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_pisa_small(B, H, N, d, k, f32):
    inp = W.gaussian_inputs(B, H, N, d, 300 + N + k, use_w=False, with_alpha=False)
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    ref = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut, 64, 64)
    p = params(B, H, N, d, 64, 64, k, given=True, f32=f32)
    check(gpu_pisa(p, dev(inp), lut), ref, p)


def test_pisa_block_constant_keys_is_dense_attention():
    """Zero-order exactness through the kernels: block-constant keys."""
    B, H, N, d, k = 1, 2, 2048, 128, 3
    inp = W.gaussian_inputs(B, H, N, d, 61, use_w=False, with_alpha=False)
    g = torch.Generator().manual_seed(2)
    kb = torch.randn(B, H, N // 64, 1, d, generator=g).to(torch.bfloat16)
    inp["k"] = kb.expand(B, H, N // 64, 64, d).reshape(B, H, N, d).contiguous()
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    dense = torch.nn.functional.scaled_dot_product_attention(
        inp["q"].double(), inp["k"].double(), inp["v"].double()).numpy()
    p = params(B, H, N, d, 64, 64, k, given=True, f32=True)
    check(gpu_pisa(p, dev(inp), lut), dense, p)


@pytest.mark.parametrize("f32", [False, True], ids=["out_bf16", "out_fp32"])
def test_pisa_workload_sampled(f32):
    w = W.WORKLOADS["pisa"]
    inp = W.make_inputs(w)
    lut_ref, gap = orc.route(inp["q"], inp["k"], None, None, w.Bq, w.Bk, w.topk)
    g = dev(inp)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk, f32=f32)
    ws = S.workspace(p)
    lut = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, ws)
    assert S.sla_check_device_status() == 0
    excl = check_lut(lut.cpu().numpy(), lut_ref, gap, w.Nk)
    rows = W.sample_rows(w.B, w.H, w.N, 384, 6, heads=[1, 17]).numpy()
    keep = ~excl.reshape(-1, w.Nq)[rows // w.N, (rows % w.N) // w.Bq]
    rows = rows[keep]
    ref = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut_ref, w.Bq, w.Bk, rows=rows)
    mx, mn = check(rows_of(out, rows), ref, p, TOL_BF16, "pisa")
    print("pisa: %d rows, max/mean err (std units) %.3g %.3g" % (len(rows), mx, mn))


# ---------------------------------------------------------------- global first-order term

def fo_params(B, H, N, d, k, given=True, f32=True):
    return S.params(B, H, N, d, 64, 64, k, lut_mode=S.SLA_LUT_GIVEN if given else S.SLA_LUT_COMPUTE,
                    out_dtype=S.SLA_OUT_FP32 if f32 else S.SLA_OUT_BF16, pisa_first_order=True)


@pytest.mark.parametrize("B,H,N,d,k", [
    (1, 2, 1024, 64, 4),
    (1, 2, 2048, 128, 5),
    (2, 1, 1088, 128, 3),       # odd Nq
    (1, 2, 2048, 128, 0),       # only centroids
    (1, 1, 4160, 128, 9),       # Nk = 65: ragged centroid pseudo-tile
])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_pisa_first_order_small(B, H, N, d, k, f32):
    inp = W.gaussian_inputs(B, H, N, d, 700 + N + k, use_w=False, with_alpha=False)
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    ref = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut, 64, 64, first_order=True)
    p = fo_params(B, H, N, d, k, f32=f32)
    out = gpu_pisa(p, dev(inp), lut)
    check(out, ref, p)
    # and it is not the zero-order result
    zero = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut, 64, 64)
    assert np.abs(out.double().cpu().numpy() - zero).max() > 1e-4 * zero.std()


def test_pisa_first_order_block_constant_keys_is_dense_attention():
    B, H, N, d, k = 1, 2, 2048, 128, 3
    inp = W.gaussian_inputs(B, H, N, d, 71, use_w=False, with_alpha=False)
    g = torch.Generator().manual_seed(3)
    kb = torch.randn(B, H, N // 64, 1, d, generator=g).to(torch.bfloat16)
    inp["k"] = kb.expand(B, H, N // 64, 64, d).reshape(B, H, N, d).contiguous()
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    dense = torch.nn.functional.scaled_dot_product_attention(
        inp["q"].double(), inp["k"].double(), inp["v"].double()).numpy()
    p = fo_params(B, H, N, d, k)
    check(gpu_pisa(p, dev(inp), lut), dense, p)


@pytest.mark.parametrize("f32", [False, True], ids=["out_bf16", "out_fp32"])
def test_pisa_first_order_workload_sampled(f32):
    w = W.WORKLOADS["pisa"]
    inp = W.make_inputs(w)
    lut_ref, gap = orc.route(inp["q"], inp["k"], None, None, w.Bq, w.Bk, w.topk)
    g = dev(inp)
    p = fo_params(w.B, w.H, w.N, w.d, w.topk, given=False, f32=f32)
    ws = S.workspace(p)
    lut = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, ws)
    assert S.sla_check_device_status() == 0
    excl = check_lut(lut.cpu().numpy(), lut_ref, gap, w.Nk)
    rows = W.sample_rows(w.B, w.H, w.N, 384, 8, heads=[4, 20]).numpy()
    keep = ~excl.reshape(-1, w.Nq)[rows // w.N, (rows % w.N) // w.Bq]
    rows = rows[keep]
    ref = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut_ref, w.Bq, w.Bk, rows=rows, first_order=True)
    mx, mn = check(rows_of(out, rows), ref, p, TOL_BF16, "pisa first order")
    print("pisa first order: %d rows, max/mean err (std units) %.3g %.3g" % (len(rows), mx, mn))

"""The host-buffer calls sla_forward_host and sla_pisa_forward_host: chunks of
heads copied in, computed and copied back on overlapping streams.  Their LUT
equals the device call's (the router is per head), their output meets the
oracle's tolerance, and they agree with the device call to within the
rounding of a different summation order (the pre-pass chunking depends on
the number of heads in a call)."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import check, check_lut, dev, params

pytestmark = pytest.mark.gpu


def _pinned(inp):
    return {k: (v.contiguous().pin_memory() if v is not None else None) for k, v in inp.items()}


@pytest.mark.parametrize("hpc", [0, 1, 3, 64])
@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
def test_forward_host_matches_device_and_oracle(hpc, f32):
    B, H, N, d, Bq, k = 2, 3, 2048, 128, 128, 6
    inp = W.gaussian_inputs(B, H, N, d, 77)
    g = dev(inp)
    p = params(B, H, N, d, Bq, 64, k, f32=f32)
    ws = S.workspace(p)
    # the device call
    lut_d = torch.full((B, H, N // Bq, k), -1, dtype=torch.int32, device="cuda")
    out_d = torch.empty(g["q"].shape, dtype=S.sla.out_torch_dtype(p), device="cuda")
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut_d, out_d, ws)
    # the host call into fresh device buffers
    h = _pinned(inp)
    out_h = torch.full(inp["q"].shape, float("nan"), dtype=S.sla.out_torch_dtype(p)).pin_memory()
    bufs = {n: torch.empty_like(g[n]) for n in ("q", "k", "v", "alpha")}
    out = torch.empty_like(out_d)
    lut = torch.full_like(lut_d, -1)
    S.sla_forward_host(p, h["q"], h["k"], h["v"], h["alpha"], out_h, bufs["q"], bufs["k"], bufs["v"],
                       bufs["alpha"], out, g["w_q"], g["w_k"], lut, S.workspace(p), heads_per_chunk=hpc)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    assert torch.equal(lut, lut_d)
    ref_lut, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, 64, k)
    check_lut(lut.cpu().numpy(), ref_lut, gap, N // 64)
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut.cpu().numpy(), Bq, 64)
    check(out_h, ref, p)
    o_h = out_h.double().numpy()
    o_d = out_d.double().cpu().numpy()
    assert np.abs(o_h - o_d).max() <= 1e-3 * np.abs(o_d).max()


@pytest.mark.parametrize("hpc", [0, 5])
def test_pisa_forward_host_matches_oracle(hpc):
    B, H, N, d, k = 1, 4, 2048, 128, 5
    inp = W.gaussian_inputs(B, H, N, d, 78, use_w=False, with_alpha=False)
    g = dev(inp)
    p = S.params(B, H, N, d, 64, 64, k, out_dtype=S.SLA_OUT_FP32, pisa_first_order=True)
    h = _pinned(inp)
    out_h = torch.full(inp["q"].shape, float("nan"), dtype=torch.float32).pin_memory()
    bufs = {n: torch.empty_like(g[n]) for n in ("q", "k", "v")}
    out = torch.empty(g["q"].shape, dtype=torch.float32, device="cuda")
    lut = torch.full((B, H, N // 64, k), -1, dtype=torch.int32, device="cuda")
    S.sla_pisa_forward_host(p, h["q"], h["k"], h["v"], out_h, bufs["q"], bufs["k"], bufs["v"], out,
                            None, None, lut, S.workspace(p), heads_per_chunk=hpc)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    ref_lut, gap = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    check_lut(lut.cpu().numpy(), ref_lut, gap, N // 64)
    ref = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut.cpu().numpy(), 64, 64, first_order=True)
    check(out_h, ref, p)


def test_forward_host_pageable_memory_and_arguments():
    """Pageable host memory gives the same result; a device tensor where a host
    buffer belongs, and a negative chunk size, are refused."""
    B, H, N, d, Bq, k = 1, 2, 1024, 64, 64, 4
    inp = W.gaussian_inputs(B, H, N, d, 79)
    g = dev(inp)
    p = params(B, H, N, d, Bq, 64, k, f32=True)
    outs = []
    for pin in (True, False):
        h = _pinned(inp) if pin else {k_: (v.contiguous() if v is not None else None) for k_, v in inp.items()}
        out_h = torch.empty(inp["q"].shape, dtype=torch.float32)
        out_h = out_h.pin_memory() if pin else out_h
        bufs = {n: torch.empty_like(g[n]) for n in ("q", "k", "v", "alpha")}
        out = torch.empty(g["q"].shape, dtype=torch.float32, device="cuda")
        S.sla_forward_host(p, h["q"], h["k"], h["v"], h["alpha"], out_h, bufs["q"], bufs["k"], bufs["v"],
                           bufs["alpha"], out, g["w_q"], g["w_k"], None, S.workspace(p))
        torch.cuda.synchronize()
        outs.append(out_h.clone())
    assert torch.equal(outs[0], outs[1])
    with pytest.raises(ValueError):
        S.sla_forward_host(p, g["q"], g["k"], g["v"], g["alpha"], outs[0], g["q"], g["k"], g["v"],
                           g["alpha"], out, g["w_q"], g["w_k"], None, S.workspace(p))
    with pytest.raises(S.SlaError) as ei:
        S.sla_forward_host(p, _pinned(inp)["q"], inp["k"], inp["v"], inp["alpha"], outs[0], g["q"], g["k"],
                           g["v"], g["alpha"], out, g["w_q"], g["w_k"], None, S.workspace(p), heads_per_chunk=-1)
    assert ei.value.code == S.sla.SLA_ERR_INVALID_ARG


def test_forward_host_given_lut():
    """LUT_GIVEN: each chunk reads its own rows of the caller's LUT."""
    B, H, N, d, Bq, k = 1, 5, 2048, 128, 128, 7
    inp = W.gaussian_inputs(B, H, N, d, 80)
    g = dev(inp)
    rng = np.random.default_rng(3)
    lut_np = np.sort(np.stack([[[rng.choice(N // 64, k, replace=False) for _ in range(N // Bq)]
                                for _ in range(H)] for _ in range(B)]), axis=-1).astype(np.int32)
    p = params(B, H, N, d, Bq, 64, k, given=True, f32=True)
    h = _pinned(inp)
    out_h = torch.full(inp["q"].shape, float("nan"), dtype=torch.float32).pin_memory()
    bufs = {n: torch.empty_like(g[n]) for n in ("q", "k", "v", "alpha")}
    out = torch.empty(g["q"].shape, dtype=torch.float32, device="cuda")
    lut = torch.as_tensor(lut_np).cuda()
    S.sla_forward_host(p, h["q"], h["k"], h["v"], h["alpha"], out_h, bufs["q"], bufs["k"], bufs["v"],
                       bufs["alpha"], out, g["w_q"], g["w_k"], lut, S.workspace(p), heads_per_chunk=2)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut_np, Bq, 64)
    check(out_h, ref, p)


def test_forward_host_many_heads_in_the_whole_problems_workspace():
    """297 heads of 64 KV blocks in chunks of 296 and 1: the whole problem's
    pre-pass keeps a head in one chunk (297 partial sums), while the 296-head
    chunk splits each head in two (592).  The workspace sized for the whole
    problem must still serve that chunk."""
    B, H, N, d, Bq, k = 1, 297, 4096, 64, 64, 4
    inp = W.gaussian_inputs(B, H, N, d, 81)
    g = dev(inp)
    p = params(B, H, N, d, Bq, 64, k, f32=False)
    ws = S.workspace(p)
    lut_d = torch.full((B, H, N // Bq, k), -1, dtype=torch.int32, device="cuda")
    out_d = torch.empty(g["q"].shape, dtype=S.sla.out_torch_dtype(p), device="cuda")
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut_d, out_d, ws)
    h = _pinned(inp)
    out_h = torch.full(inp["q"].shape, float("nan"), dtype=S.sla.out_torch_dtype(p)).pin_memory()
    bufs = {n: torch.empty_like(g[n]) for n in ("q", "k", "v", "alpha")}
    out = torch.empty_like(out_d)
    lut = torch.full_like(lut_d, -1)
    S.sla_forward_host(p, h["q"], h["k"], h["v"], h["alpha"], out_h, bufs["q"], bufs["k"], bufs["v"],
                       bufs["alpha"], out, g["w_q"], g["w_k"], lut, ws, heads_per_chunk=296)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    assert torch.equal(lut, lut_d)
    o_h = out_h.float()
    o_d = out_d.float().cpu()
    assert torch.isfinite(o_h).all()
    assert (o_h - o_d).abs().max() <= 1e-3 * o_d.abs().max()

"""PISA covariance-aware selection on the GPU: the block norms
M_j = ||H_j - Hbar||_2 against the oracle (numpy SVD in fp64), and the LUT of
a covariance-aware sla_pisa_forward against the oracle's routing with the
bias lambda M_j.  GPU norms carry a relative error of a few 1e-7 (the tensor
core's fp32 sums of exact products, fp32 Lanczos), so LUT rows whose k-th and
(k+1)-th biased scores lie closer than 1e-5 + 4e-6 lambda max M may differ."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import check, dev, new_out

pytestmark = pytest.mark.gpu


def cov_params(B, H, N, d, k, lam, given=False):
    return S.params(B, H, N, d, 64, 64, k, pisa_cov_lambda=lam,
                    lut_mode=S.SLA_LUT_GIVEN if given else S.SLA_LUT_COMPUTE,
                    out_dtype=S.SLA_OUT_FP32)


def gpu_norms(p, g):
    ws = S.workspace(p)
    norms = torch.full((p.B, p.H, p.N // p.Bk), float("nan"), dtype=torch.float64, device="cuda")
    S.sla_pisa_cov_norms(p, g["k"], g["v"], norms, ws)
    assert S.sla_check_device_status() == 0
    return norms.cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
def test_cov_norms_match_oracle(d):
    B, H, N = 1, 2, 4096
    inp = W.gaussian_inputs(B, H, N, d, 40 + d)
    m = gpu_norms(cov_params(B, H, N, d, 8, 0.1), dev(inp))
    ref = orc.block_cov_norms(inp["k"], inp["v"], 64)
    rel = np.abs(m - ref) / ref
    print("d=%d: max rel %.2e, median %.2e" % (d, rel.max(), np.median(rel)))
    assert rel.max() < 2e-6


def test_cov_norms_video_workload_heads():
    w = W.WORKLOADS["pisa_cov"]
    inp = W.make_inputs(w)
    m = gpu_norms(cov_params(w.B, w.H, w.N, w.d, w.topk, w.cov_lambda), dev(inp))
    hs = [0, 7, 23]
    ref = orc.block_cov_norms(inp["k"][:, hs], inp["v"][:, hs], 64)
    rel = np.abs(m[:, hs] - ref) / ref
    print("pisa_cov heads %s: max rel %.2e" % (hs, rel.max()))
    assert rel.max() < 2e-6


def test_cov_norms_closed_form():
    """H_0 = diag(48, 24) = -H_1, blocks 2 and 3 with constant keys: M = 48, 48, 0, 0
    (the spectral norm; the Frobenius norm would be 53.67)."""
    d, Bk = 64, 64
    rng = np.random.default_rng(31)
    k = np.repeat(rng.integers(-8, 9, size=(4, 1, d)) / 4.0, Bk, axis=1)
    v = rng.integers(-8, 9, size=(4, Bk, d)) / 4.0
    s = np.ones(Bk)
    s[1::2] = -1.0
    for j, sign in ((0, 1.0), (1, -1.0)):
        v[j] = 0.0
        k[j, :32, 0] += 1.5 * s[:32]
        k[j, 32:, 1] += 0.75 * s[32:]
        v[j, :32, 0] = sign * s[:32]
        v[j, 32:, 1] = sign * s[32:]
    g = {"k": torch.as_tensor(k.reshape(1, 1, -1, d), dtype=torch.float32).to(torch.bfloat16).cuda(),
         "v": torch.as_tensor(v.reshape(1, 1, -1, d), dtype=torch.float32).to(torch.bfloat16).cuda()}
    m = gpu_norms(cov_params(1, 1, 4 * Bk, d, 2, 1.0), g)[0, 0]
    np.testing.assert_allclose(m, [48.0, 48.0, 0.0, 0.0], rtol=1e-6, atol=0)


def _check_cov_lut(lut, ref, gap, m, lam):
    tol = 1e-5 + 4e-6 * lam * float(m.max())
    excl = gap < tol
    ok = (lut == ref).all(axis=-1) | excl
    assert ok.all(), np.argwhere(~ok)[:5]
    assert excl.mean() < 0.05, excl.mean()
    return excl


@pytest.mark.parametrize("N,k,lam", [(4096, 8, 0.5), (2048, 31, 2.0)])
def test_cov_routing_matches_oracle(N, k, lam):
    B, H, d = 1, 2, 128
    inp = W.gaussian_inputs(B, H, N, d, 50 + k)
    g = dev(inp)
    p = cov_params(B, H, N, d, k, lam)
    ws = S.workspace(p)
    lut = torch.full((B, H, N // 64, k), -1, dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, ws)
    assert S.sla_check_device_status() == 0
    m = orc.block_cov_norms(inp["k"], inp["v"], 64)
    ref, gap = orc.route_cov(inp["q"], inp["k"], inp["v"], 64, 64, k, lam)
    plain, _ = orc.route(inp["q"], inp["k"], None, None, 64, 64, k)
    assert not np.array_equal(ref, plain)            # the term changes the selection
    _check_cov_lut(lut.cpu().numpy(), ref, gap, m, lam)
    # the forward on its own LUT equals the forward on that LUT given
    out2 = new_out(p, g["q"])
    pg = cov_params(B, H, N, d, k, lam, given=True)
    S.sla_pisa_forward(pg, g["q"], g["k"], g["v"], None, None, lut.clone(), out2, S.workspace(pg))
    assert S.sla_check_device_status() == 0
    assert torch.equal(out, out2)


def test_cov_workload_lut():
    """The benchmark's covariance-aware PISA workload: every head's LUT."""
    w = W.WORKLOADS["pisa_cov"]
    inp = W.make_inputs(w)
    g = dev(inp)
    p = cov_params(w.B, w.H, w.N, w.d, w.topk, w.cov_lambda)
    ws = S.workspace(p)
    lut = torch.empty((w.B, w.H, w.Nq, w.topk), dtype=torch.int32, device="cuda")
    out = torch.empty(g["q"].shape, dtype=torch.float32, device="cuda")
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, ws)
    assert S.sla_check_device_status() == 0
    m = orc.block_cov_norms(inp["k"], inp["v"], 64)
    ref, gap = orc.route(inp["q"], inp["k"], None, None, w.Bq, w.Bk, w.topk, bias=w.cov_lambda * m)
    excl = _check_cov_lut(lut.cpu().numpy(), ref, gap, m, w.cov_lambda)
    print("pisa_cov: %d of %d rows excluded by the gap rule" % (excl.sum(), excl.size))


def test_cov_routing_with_first_order_term():
    """Both PISA options at once: the covariance-aware LUT (the pre-pass then
    forms the blocks' H_j sums exactly, for Hbar and for the first-order term)
    and the first-order output on that LUT, against the oracle."""
    B, H, N, d, k, lam = 1, 2, 4096, 128, 8, 0.5
    inp = W.gaussian_inputs(B, H, N, d, 91, use_w=False, with_alpha=False)
    g = dev(inp)
    p = S.params(B, H, N, d, 64, 64, k, pisa_cov_lambda=lam, pisa_first_order=True,
                 out_dtype=S.SLA_OUT_FP32)
    lut = torch.full((B, H, N // 64, k), -1, dtype=torch.int32, device="cuda")
    out = new_out(p, g["q"])
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, S.workspace(p))
    assert S.sla_check_device_status() == 0
    m = orc.block_cov_norms(inp["k"], inp["v"], 64)
    ref, gap = orc.route_cov(inp["q"], inp["k"], inp["v"], 64, 64, k, lam)
    _check_cov_lut(lut.cpu().numpy(), ref, gap, m, lam)
    lut_np = lut.cpu().numpy()
    want = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut_np, 64, 64, first_order=True)
    check(out, want, p)

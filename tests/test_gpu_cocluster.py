"""SVOO online bidirectional Q-K co-clustering on the GPU against the oracle,
the row permutation, and the block-sparse forward in the co-clustered order.

The co-clustering is a discrete result (two permutations per head): it must
equal the oracle's exactly.  Both sides work in fp64 from the bf16 inputs; the
centroid sums are exact, so only a near-tie of two affinities (within a few
ulps of fp64) could split them, and the inputs here have none."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W
from oracle import oracle as orc

from gpu_util import TOL_BF16, check, dev, gpu_forward, params, rows_of

pytestmark = pytest.mark.gpu


def gpu_cocluster(p, g, C, iters):
    ws = S.cocluster_workspace(p, C)
    qp = torch.full((p.B, p.H, p.N), -1, dtype=torch.int32, device="cuda")
    kp = torch.full_like(qp, -1)
    S.sla_cocluster(p, g["q"], g["k"], C, iters, qp, kp, ws)
    assert S.sla_check_device_status() == 0
    return qp, kp


def planted(N, d, C, seed, bias=0.5):
    rng = np.random.default_rng(seed)
    u, _ = np.linalg.qr(rng.standard_normal((d, C)))
    u = u.T
    chunk = N // C
    group = np.zeros(N, dtype=np.int64)
    for c in range(C):
        own = int(round(bias * chunk))
        lab = np.concatenate([np.full(own, c), rng.choice([x for x in range(C) if x != c], chunk - own)])
        rng.shuffle(lab)
        group[c * chunk:(c + 1) * chunk] = lab
    q = 4 * u[group] + 0.05 * rng.standard_normal((N, d))
    k = 4 * u[group] + 0.05 * rng.standard_normal((N, d))
    to = lambda x: torch.from_numpy(x.reshape(1, 1, N, d)).float().to(torch.bfloat16)
    return {"q": to(q), "k": to(k)}, group


def test_cocluster_planted_groups():
    inp, group = planted(2048, 128, 8, 91)
    p = params(1, 1, 2048, 128, 128, 64, 4)
    qp, kp = gpu_cocluster(p, dev(inp), 8, 3)
    want = np.argsort(group, kind="stable")
    assert np.array_equal(qp.cpu().numpy()[0, 0], want)
    assert np.array_equal(kp.cpu().numpy()[0, 0], want)


@pytest.mark.parametrize("B,H,N,d,C,iters,gen", [
    (1, 2, 2048, 128, 16, 3, "video"),
    (2, 1, 2048, 64, 32, 2, "gaussian"),
    (1, 3, 4096, 128, 64, 4, "video"),
    (1, 2, 1024, 64, 1, 1, "gaussian"),       # one cluster: the identity
    (1, 1, 2048, 128, 512, 2, "video"),       # many clusters (several centroid tiles), some empty
])
def test_cocluster_matches_oracle(B, H, N, d, C, iters, gen):
    if gen == "video":
        inp = W.video_inputs(B, H, N, d, (6, 16, 21) if N == 2048 else (8, 20, 25), 92 + N + C)
    else:
        inp = W.gaussian_inputs(B, H, N, d, 92 + N + C)
    p = params(B, H, N, d, 64, 64, 4)
    qp, kp = gpu_cocluster(p, dev(inp), C, iters)
    rq, rk, _, _ = orc.cocluster(inp["q"], inp["k"], C, iters)
    assert np.array_equal(qp.cpu().numpy(), rq) and np.array_equal(kp.cpu().numpy(), rk)


def test_cocluster_video_workload():
    """The 32K-token video workload, all 12 heads, 64 clusters, 3 iterations."""
    w = W.WORKLOADS["sla2_svoo"]
    inp = W.make_inputs(w)
    p = params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk)
    qp, kp = gpu_cocluster(p, dev(inp), w.clusters, w.cluster_iters)
    rq, rk, _, _ = orc.cocluster(inp["q"], inp["k"], w.clusters, w.cluster_iters)
    assert np.array_equal(qp.cpu().numpy(), rq) and np.array_equal(kp.cpu().numpy(), rk)


@pytest.mark.parametrize("shape,dtype", [((2, 3, 512, 128), torch.bfloat16), ((1, 2, 256, 64), torch.bfloat16),
                                         ((2, 3, 512), torch.float32), ((1, 2, 128, 128), torch.float32),
                                         ((1, 3, 1000, 64), torch.bfloat16),       # rows not a multiple of a pass
                                         ((1, 4, 32768, 128), torch.bfloat16),     # several grid strides a thread
                                         ((4, 8, 65536), torch.float32)])
def test_permute_rows_gather_and_scatter(shape, dtype):
    g = torch.Generator().manual_seed(93)
    x = torch.randn(shape, generator=g).to(dtype).cuda()
    B, H, N = shape[:3]
    perm = torch.stack([torch.randperm(N, generator=g) for _ in range(B * H)]).reshape(B, H, N).int().cuda()
    y = torch.empty_like(x)
    S.sla_permute_rows(x, perm, y)
    idx = perm.long().reshape(B, H, N, *([1] * (x.dim() - 3))).expand_as(x)
    assert torch.equal(y, torch.gather(x, 2, idx))
    z = torch.empty_like(x)
    S.sla_permute_rows(y, perm, z, inverse=True)
    assert torch.equal(z, x)
    assert S.sla_check_device_status() == 0


def _permuted(inp, qp, kp):
    g = lambda x, p: torch.gather(x, 2, torch.as_tensor(p).long().unsqueeze(-1).expand(-1, -1, -1, x.shape[-1]))
    out = dict(inp)
    out["q"], out["k"], out["v"] = g(inp["q"], qp), g(inp["k"], kp), g(inp["v"], kp)
    out["alpha"] = torch.gather(inp["alpha"], 2, torch.as_tensor(qp).long())
    return out


@pytest.mark.parametrize("f32", [True, False], ids=["out_fp32", "out_bf16"])
@pytest.mark.parametrize("B,H,N,d,Bq,k,C", [(1, 2, 2048, 128, 128, 5, 16), (1, 2, 2048, 64, 64, 6, 32)])
def test_coclustered_forward_matches_oracle(B, H, N, d, Bq, k, C, f32):
    """Gather by the GPU's permutations, route and attend, scatter back: equal to
    the oracle's forward on the oracle-permuted inputs, put back in place."""
    inp = W.video_inputs(B, H, N, d, (6, 16, 21), 94 + d)
    g = dev(inp)
    p = params(B, H, N, d, Bq, 64, k, f32=f32)
    qp, kp = gpu_cocluster(p, g, C, 3)
    rq, rk, _, _ = orc.cocluster(inp["q"], inp["k"], C, 3)
    assert np.array_equal(qp.cpu().numpy(), rq) and np.array_equal(kp.cpu().numpy(), rk)
    ws = S.workspace(p)
    out = torch.empty(B, H, N, d, dtype=S.sla.out_torch_dtype(p), device="cuda")
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    S.sla_forward_coclustered(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], qp, kp, lut, out, ws)
    assert S.sla_check_device_status() == 0
    pin = _permuted(inp, rq, rk)
    lut_ref, gap = orc.route(pin["q"], pin["k"], pin["w_q"], pin["w_k"], Bq, 64, k)
    assert np.array_equal(lut.cpu().numpy()[gap >= 1e-5], lut_ref[gap >= 1e-5])
    ref_p = orc.sla_forward(pin["q"], pin["k"], pin["v"], pin["alpha"], lut_ref, Bq, 64)
    ref = np.zeros_like(ref_p)
    for b in range(B):
        for h in range(H):
            ref[b, h, rq[b, h]] = ref_p[b, h]
    check(out, ref, p, TOL_BF16, "coclustered")


def test_coclustered_dense_attention_is_order_free():
    """All blocks selected, alpha = 1: dense attention, whatever the order; the
    co-clustered call meets the stated tolerance against the oracle's dense
    attention in the original order (two GPU runs in different block orders
    differ by their own fp16 P rounding, so they are each compared with the
    oracle, not with one another)."""
    B, H, N, d, Bq = 1, 2, 2048, 128, 128
    inp = W.video_inputs(B, H, N, d, (6, 16, 21), 95)
    inp["alpha"] = torch.ones(B, H, N)
    g = dev(inp)
    Nk = N // 64
    p = params(B, H, N, d, Bq, 64, Nk, f32=True)
    qp, kp = gpu_cocluster(p, g, 16, 3)
    out = torch.empty(B, H, N, d, dtype=torch.float32, device="cuda")
    S.sla_forward_coclustered(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], qp, kp, None, out,
                              S.workspace(p))
    lut_all = np.broadcast_to(np.arange(Nk, dtype=np.int32), (B, H, N // Bq, Nk)).copy()
    ref = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut_all, Bq, 64)
    check(out, ref, p, TOL_BF16, "coclustered dense")
    check(gpu_forward(p, g), ref, p, TOL_BF16, "plain dense")

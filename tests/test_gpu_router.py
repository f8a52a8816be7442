"""Router parity on the GPU: the top-k block LUT from sla_route equals the
oracle's bit for bit (except rows whose k-th/(k+1)-th pooled-score gap is
below 1e-5), on small shapes with ragged tails and on the full workloads."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc

from gpu_util import check_lut, dev, gpu_route, params

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,Bq,Bk,k,use_w", [
    (1, 2, 1024, 64, 64, 64, 4, True),
    (2, 3, 1088, 64, 64, 64, 5, True),        # Nq = 17: a partial row group; Nk = 17 < d
    (1, 2, 4096, 128, 128, 64, 13, True),     # Nk = 64
    (1, 1, 8320, 128, 128, 64, 30, False),    # Nk = 130: ragged 64-column chunk
    (1, 2, 2048, 128, 64, 64, 0, True),       # k = 0
    (1, 2, 2048, 128, 64, 64, 32, True),      # k = Nk
    (1, 2, 2048, 128, 64, 64, 31, True),      # k = Nk - 1
    (1, 1, 1024, 128, 128, 64, 1, True),      # k = 1
    # long rows: fewer query blocks per CTA (8, 4, 2; the MMA's 8-row tile padded)
    (1, 1, 131072, 64, 128, 64, 37, True),    # Nk = 2048
    (1, 1, 262144, 64, 128, 64, 100, True),   # Nk = 4096
    (1, 1, 524288, 64, 128, 64, 300, False),  # Nk = 8192, the largest supported
    (1, 1, 524288, 128, 128, 64, 77, True),   # the same with d = 128
])
def test_route_small(B, H, N, d, Bq, Bk, k, use_w):
    inp = W.gaussian_inputs(B, H, N, d, 100 + N + k, use_w=use_w)
    ref, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, Bk, k)
    lut = gpu_route(params(B, H, N, d, Bq, Bk, k), dev(inp))
    check_lut(lut, ref, gap, N // Bk)


@pytest.mark.parametrize("name", ["tiny", "sla2_bf16", "sla2_long", "pisa"])
def test_route_workloads(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    ref, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], w.Bq, w.Bk, w.topk)
    lut = gpu_route(params(w.B, w.H, w.N, w.d, w.Bq, w.Bk, w.topk), dev(inp))
    excl = check_lut(lut, ref, gap, w.Nk)
    print("%s: %d of %d rows excluded by the gap rule" % (name, excl.sum(), excl.size))


def test_route_deterministic():
    inp = dev(W.gaussian_inputs(1, 4, 4096, 128, 7))
    p = params(1, 4, 4096, 128, 128, 64, 9)
    a = gpu_route(p, inp)
    b = gpu_route(p, inp)
    assert np.array_equal(a, b)


def test_route_projection_matches_identity():
    inp = W.gaussian_inputs(1, 2, 2048, 64, 8, use_w=False)
    g = dev(inp)
    p = params(1, 2, 2048, 64, 64, 64, 6)
    a = gpu_route(p, g)
    g2 = dict(g, w_q=torch.eye(64, device="cuda"), w_k=torch.eye(64, device="cuda"))
    b = gpu_route(p, g2)
    assert np.array_equal(a, b)

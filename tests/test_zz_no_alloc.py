"""sla_route_noalloc: routing for callers that cannot allocate device memory
(a plugin under a host engine that owns the device-memory budget, a serving
loop that must not enter an allocator).  Its scratch is the library's
built-in device array, so it takes no workspace.  This file sorts last so that
a run stopping at the first failure has run every other test first."""
import numpy as np
import pytest
import torch

import block_sparse_linear_proj_b200 as S
from block_sparse_linear_proj_b200 import sla as B
import workloads as W

pytestmark = pytest.mark.gpu


def _route_with_workspace(p, g):
    lut = torch.full((p.B, p.H, p.N // p.Bq, p.topk), -1, dtype=torch.int32, device="cuda")
    S.sla_route(p, g["q"], g["k"], g["w_q"], g["w_k"], lut, S.workspace(p))
    return lut


def _route_noalloc(p, g):
    lut = torch.full((p.B, p.H, p.N // p.Bq, p.topk), -1, dtype=torch.int32, device="cuda")
    B.sla_route_noalloc(p, g["q"], g["k"], g["w_q"], g["w_k"], lut)
    return lut


def test_noalloc_route_matches_workspace_route_twice():
    """Calls in a row, each equal to sla_route with a fresh caller workspace
    (the LUT is integer output, compared exactly): a small call, a larger one,
    then a small one without projections, after the larger call has filled
    more of the shared array and its W_q W_k^T region, so that nothing left in
    the array from an earlier call can reach the LUT."""
    cases = [(1, 2, 1024, 64, 64, 4, 501, True), (1, 12, 32768, 128, 128, 52, 502, True),
             (1, 2, 2048, 128, 64, 5, 503, False)]
    for (Bb, H, N, d, Bq, k, seed, with_w) in cases:
        g = {kk: (v.cuda() if v is not None else None)
             for kk, v in W.gaussian_inputs(Bb, H, N, d, seed).items()}
        if not with_w:
            g["w_q"] = g["w_k"] = None
        p = S.params(Bb, H, N, d, Bq, 64, k)
        ref = _route_with_workspace(p, g)
        got = _route_noalloc(p, g)
        assert B.sla_check_device_status() == B.SLA_OK
        assert torch.equal(ref, got)
        assert (got >= 0).all()


def test_noalloc_route_rejects_oversized_problem():
    # 40 heads x 75776 tokens needs ~72 MiB of scratch, above the built-in 32 MiB
    p = S.params(1, 40, 75776, 128, 128, 64, 59)
    q = torch.empty((1, 40, 75776, 128), dtype=torch.bfloat16, device="cuda")
    lut = torch.empty((1, 40, 592, 59), dtype=torch.int32, device="cuda")
    with pytest.raises(S.SlaError) as ei:
        B.sla_route_noalloc(p, q, q, None, None, lut)
    assert ei.value.code == B.SLA_ERR_WORKSPACE

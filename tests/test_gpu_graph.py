"""Stream capture: a forward call captured into a CUDA graph (its side-stream
K/V pre-pass included, through the fork and join events) replays to the same
result as the eager call, and picks up new input values on replay."""
import pytest
import torch

import block_sparse_linear_proj_b200 as S
import workloads as W

from gpu_util import dev, new_out, params

pytestmark = pytest.mark.gpu


def _setup(mode, sd=S.SLA_SPARSE_BF16, first_order=False):
    B, H, N, d, k = 1, 2, 4096, 128, 9
    Bq = 64 if mode == "pisa" else 128
    inp = dev(W.gaussian_inputs(B, H, N, d, 61))
    p = S.params(B, H, N, d, Bq, 64, k, sparse_dtype=sd, pisa_first_order=first_order,
                 out_dtype=S.SLA_OUT_FP32)
    ws = S.workspace(p)
    lut = torch.empty((B, H, N // Bq, k), dtype=torch.int32, device="cuda")
    out = new_out(p, inp["q"])
    return inp, p, ws, lut, out


def _call(mode, p, g, lut, out, ws, stream=None):
    if mode == "pisa":
        S.sla_pisa_forward(p, g["q"], g["k"], g["v"], None, None, lut, out, ws, stream)
    else:
        S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lut, out, ws, stream)


@pytest.mark.parametrize("mode,sd,fo", [
    ("sla", S.SLA_SPARSE_BF16, False),
    ("sla", S.SLA_SPARSE_FP8_E4M3, False),
    ("pisa", S.SLA_SPARSE_BF16, True),
], ids=["sla_bf16", "sla_fp8", "pisa_first_order"])
def test_captured_forward_replays_like_eager(mode, sd, fo):
    g, p, ws, lut, out = _setup(mode, sd, fo)
    # eager reference (also creates the library's side stream before the capture)
    _call(mode, p, g, lut, out, ws)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    ref, ref_lut = out.clone(), lut.clone()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    out.fill_(float("nan"))
    lut.fill_(-1)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            _call(mode, p, g, lut, out, ws, side)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    assert torch.equal(lut, ref_lut)
    assert torch.equal(out, ref)

    # new input values in the same buffers: the replay sees them
    g["q"].mul_(-1.0)
    g["v"].mul_(0.5)
    graph.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    _call(mode, p, g, lut, out, ws)
    torch.cuda.synchronize()
    assert S.sla_check_device_status() == 0
    assert torch.equal(replayed, out)
    assert not torch.equal(replayed, ref)

"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
call the library through its C ABI binding, compare with the CPU oracle.

Tolerances (errors in units of the oracle output's standard deviation):
bf16 sparse branch: max-abs <= 2e-2, mean-abs <= 2e-3; FP8: 6e-2 / 6e-3.
They are applied as stated to fp32 outputs.  For bf16 outputs the mean-abs
bound is applied as stated and the max-abs bound to the error beyond the
output format's own rounding, |out - ref| <= tol * std + |bf16(ref) - ref|:
on heavy-tailed outputs (max|O| of 13.7 std at the 32K-token video
workload) rounding the exact result to bf16 alone exceeds 2e-2 std.
The LUT must match the oracle's exactly except on rows whose k-th and
(k+1)-th pooled scores are closer than 1e-5; those rows must still hold topk
distinct, ascending, in-range block indices."""
import numpy as np
import torch

import block_sparse_linear_proj_b200 as S
from oracle import oracle as orc

TOL_BF16 = (2e-2, 2e-3)
TOL_FP8 = (6e-2, 6e-3)
GAP_EXCLUDE = 1e-5


def dev(inp):
    return {k: (v.cuda() if v is not None else None) for k, v in inp.items()}


def params(B, H, N, d, Bq, Bk, topk, given=False, sparse_dtype=S.SLA_SPARSE_BF16, sm_scale=0.0,
           f32=False):
    return S.params(B, H, N, d, Bq, Bk, topk, sm_scale=sm_scale, sparse_dtype=sparse_dtype,
                    lut_mode=S.SLA_LUT_GIVEN if given else S.SLA_LUT_COMPUTE,
                    out_dtype=S.SLA_OUT_FP32 if f32 else S.SLA_OUT_BF16)


def new_out(p, like):
    return torch.full(tuple(like.shape), float("nan"), dtype=S.sla.out_torch_dtype(p),
                      device=like.device)


def gpu_route(p, g):
    ws = S.workspace(p)
    lut = torch.full((p.B, p.H, p.N // p.Bq, p.topk), -1, dtype=torch.int32, device="cuda")
    S.sla_route(p, g["q"], g["k"], g["w_q"], g["w_k"], lut, ws)
    assert S.sla_check_device_status() == S.sla.SLA_OK
    return lut.cpu().numpy()


def gpu_forward(p, g, lut=None):
    ws = S.workspace(p)
    out = new_out(p, g["q"])
    lt = None if lut is None else torch.as_tensor(lut, dtype=torch.int32).cuda()
    S.sla_forward(p, g["q"], g["k"], g["v"], g["alpha"], g["w_q"], g["w_k"], lt, out, ws)
    assert S.sla_check_device_status() == S.sla.SLA_OK
    return out


def gpu_pisa(p, g, lut=None):
    ws = S.workspace(p)
    out = new_out(p, g["q"])
    lt = None if lut is None else torch.as_tensor(lut, dtype=torch.int32).cuda()
    S.sla_pisa_forward(p, g["q"], g["k"], g["v"], g["w_q"], g["w_k"], lt, out, ws)
    assert S.sla_check_device_status() == S.sla.SLA_OK
    return out


def check_lut(lut_gpu, lut_ref, gap, Nk):
    """Bit-exact except rows with gap < GAP_EXCLUDE; returns the excluded-row mask."""
    assert lut_gpu.shape == lut_ref.shape
    excl = gap < GAP_EXCLUDE
    same = np.all(lut_gpu == lut_ref, axis=-1)
    bad = ~same & ~excl
    assert not bad.any(), "LUT mismatch on %d rows (first %s)" % (bad.sum(), np.argwhere(bad)[:3])
    if lut_gpu.shape[-1]:
        assert (lut_gpu >= 0).all() and (lut_gpu < Nk).all()
        assert (np.diff(lut_gpu, axis=-1) > 0).all()
    return excl


def err_units(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(out).all(), "non-finite output"
    std = ref.std()
    err = np.abs(out - ref)
    return err.max() / std, err.mean() / std


def assert_close(out, ref, tol=TOL_BF16, what=""):
    """Stated tolerance, for fp32 outputs."""
    mx, mn = err_units(out, ref)
    assert mx <= tol[0] and mn <= tol[1], "%s max %.3g mean %.3g (units of std; tol %s)" % (
        what, mx, mn, tol)
    return mx, mn


def bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def assert_close_bf16out(out, ref, tol=TOL_BF16, what=""):
    """bf16 outputs: mean-abs as stated; max-abs beyond the format's rounding."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(out).all(), "non-finite output"
    std = ref.std()
    err = np.abs(out - ref)
    excess = (err - np.abs(bf16_round(ref) - ref)).max() / std
    mn = err.mean() / std
    assert excess <= tol[0] and mn <= tol[1], "%s max-beyond-rounding %.3g mean %.3g (tol %s)" % (
        what, excess, mn, tol)
    return excess, mn


def check(out_t, ref, p, tol=TOL_BF16, what=""):
    o = out_t.double().cpu().numpy() if hasattr(out_t, "cpu") else out_t
    if p.out_dtype == S.SLA_OUT_FP32:
        return assert_close(o, ref, tol, what)
    return assert_close_bf16out(o, ref, tol, what)


def rows_of(out_gpu, rows):
    """GPU output [B,H,N,d] -> float64 numpy [len(rows), d] at flat row indices."""
    flat = out_gpu.reshape(-1, out_gpu.shape[-1])
    idx = torch.as_tensor(rows, dtype=torch.int64, device=flat.device)
    return flat.index_select(0, idx).double().cpu().numpy()


def random_lut(B, H, Nq, Nk, k, seed):
    rng = np.random.default_rng(seed)
    lut = np.zeros((B, H, Nq, k), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                lut[b, h, i] = np.sort(rng.choice(Nk, size=k, replace=False))
    return lut


def check_lowbit(out, inp, lut, Bq, p, mode, sm_scale=0.0, rows=None, what=""):
    """The 8-bit sparse branches (mode "fp8" or "int8") against three oracles on
    the same rows:
      * the quantised oracle with the kernel's reading of P's reference (the power
        of two at or above the row maximum): the stated FP8 tolerance;
      * the quantised oracle with P against the row maximum itself: the stated
        tolerance plus the two oracles' own distance from each other (triangle
        inequality: the readings round P at different points, so element by
        element they differ by about a P-rounding error);
      * the exact oracle: the mean error at most 1.05x the second oracle's own
        (the CPU pins show the two readings' errors agree within 5%) plus the
        bf16 path's mean tolerance (2e-3, for the unquantised linear branch).
    Returns (vs pow2 oracle, vs plain oracle, gpu vs exact, plain vs exact)."""
    o = rows_of(out, rows) if rows is not None else out.double().cpu().numpy()
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, 64)
    kw = {mode: True}
    ref2 = orc.sla_forward(*args, sm_scale=sm_scale, rows=rows, **kw)
    refp = orc.sla_forward(*args, sm_scale=sm_scale, rows=rows, p_plain=True, **kw)
    exact = orc.sla_forward(*args, sm_scale=sm_scale, rows=rows)
    ref2, refp, exact = ref2.reshape(o.shape), refp.reshape(o.shape), exact.reshape(o.shape)
    e2 = check(o, ref2, p, TOL_FP8, what + " vs pow2-reference oracle")
    # triangle inequality in absolute terms: |o - refp| <= |o - ref2| + |ref2 - refp|,
    # with |o - ref2| bounded as check() just verified (bf16 outputs: plus the
    # format's own rounding of ref2)
    s2 = ref2.std()
    rnd = np.abs(bf16_round(ref2) - ref2).max() if p.out_dtype != S.SLA_OUT_FP32 else 0.0
    d_o, d_r = np.abs(o - refp), np.abs(ref2 - refp)
    assert d_o.max() <= TOL_FP8[0] * s2 + rnd + d_r.max(), (what, d_o.max(), d_r.max(), s2)
    assert d_o.mean() <= TOL_FP8[1] * s2 + d_r.mean(), (what, d_o.mean(), d_r.mean(), s2)
    dist, ep = err_units(ref2, refp), err_units(o, refp)
    gpu_x, plain_x = err_units(o, exact), err_units(refp, exact)
    assert gpu_x[1] <= 1.05 * plain_x[1] + 2e-3, (what, gpu_x, plain_x)
    print("%s: vs pow2 oracle %.3g/%.3g; vs plain oracle %.3g/%.3g (oracles apart %.3g/%.3g); "
          "vs exact: gpu %.3g/%.3g, plain oracle %.3g/%.3g" % (
              (what,) + tuple(e2) + tuple(ep) + tuple(dist) + tuple(gpu_x) + tuple(plain_x)))
    return e2, ep, gpu_x, plain_x

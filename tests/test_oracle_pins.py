"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each pin uses something other than the oracle itself: a library routine for
a special case (torch's scaled-dot-product attention in fp64, torch.topk),
the pairwise O(N^2) form of linear attention (a different association from
the oracle's per-block sums), brute force on tiny inputs (full sort of an
explicit score matrix), closed forms and invariants.  Chosen so that a
dropped term, a wrong sign or index, a transposed operand, a wrong block
multiplicity or a mean-for-sum slip fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore")


def f64(x):
    return x.to(torch.float64)


def dense_sdpa(q, k, v, mask=None, scale=None):
    """Textbook softmax attention (torch library routine, fp64)."""
    d = q.shape[-1]
    return torch.nn.functional.scaled_dot_product_attention(
        f64(q), f64(k), f64(v), attn_mask=mask,
        scale=scale if scale else 1.0 / math.sqrt(d)).numpy()


def block_mask(lut, N, Bq, Bk):
    """Token-level boolean mask [B,H,N,N] (True = attend) from a block LUT."""
    B, H, Nq, k = lut.shape
    Nk = N // Bk
    m = np.zeros((B, H, Nq, Nk), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                m[b, h, i, lut[b, h, i]] = True
    m = np.repeat(np.repeat(m, Bq, axis=2), Bk, axis=3)
    return torch.from_numpy(m)


def random_lut(B, H, Nq, Nk, k, seed):
    rng = np.random.default_rng(seed)
    lut = np.zeros((B, H, Nq, k), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                lut[b, h, i] = np.sort(rng.choice(Nk, size=k, replace=False))
    return lut


def full_lut(B, H, Nq, Nk):
    return np.broadcast_to(np.arange(Nk, dtype=np.int32), (B, H, Nq, Nk)).copy()


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("N,d,Bq,Bk,k,use_w,seed", [
    (256, 64, 64, 64, 2, True, 1),
    (256, 32, 32, 16, 5, True, 2),
    (192, 16, 64, 32, 3, False, 3),
    (256, 64, 128, 64, 1, True, 4),
    (128, 8, 16, 16, 7, True, 5),
])
def test_router_brute_force(N, d, Bq, Bk, k, use_w, seed):
    """Brute force on tiny inputs: explicit pooled score matrix, full sort."""
    inp = W.gaussian_inputs(2, 2, N, d, seed, use_w=use_w)
    lut, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, Bk, k)
    q = f64(inp["q"]).numpy()
    kk = f64(inp["k"]).numpy()
    Nq, Nk = N // Bq, N // Bk
    qbar = q.reshape(2, 2, Nq, Bq, d).mean(axis=3)
    kbar = kk.reshape(2, 2, Nk, Bk, d).mean(axis=3)
    if use_w:
        qbar = qbar @ f64(inp["w_q"]).numpy()
        kbar = kbar @ f64(inp["w_k"]).numpy()
    s = qbar @ np.swapaxes(kbar, -1, -2)
    for b in range(2):
        for h in range(2):
            for i in range(Nq):
                order = np.lexsort((np.arange(Nk), -s[b, h, i]))
                assert np.array_equal(lut[b, h, i], np.sort(order[:k]))
                srt = s[b, h, i][order]
                assert gap[b, h, i] == pytest.approx(srt[k - 1] - srt[k], rel=1e-9, abs=1e-12)


def test_router_textbook_topk():
    """Bq = Bk = 1 and no projection: per-row top-k of Q K^T (torch.topk)."""
    inp = W.gaussian_inputs(1, 3, 64, 16, 11, use_w=False)
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 1, 1, 9)
    s = f64(inp["q"]) @ f64(inp["k"]).transpose(-1, -2)
    ref = torch.topk(s, 9, dim=-1).indices.sort(dim=-1).values.numpy()
    assert np.array_equal(lut, ref)


def test_router_block_permutation():
    """Permuting the KV blocks permutes the selected set."""
    N, d, Bq, Bk, k = 256, 32, 32, 32, 3
    inp = W.gaussian_inputs(1, 2, N, d, 12)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, Bk, k)
    Nk = N // Bk
    perm = np.random.default_rng(0).permutation(Nk)           # new block j' = old block perm[j']
    kp = inp["k"].reshape(1, 2, Nk, Bk, d)[:, :, torch.from_numpy(perm)].reshape(1, 2, N, d)
    lutp, _ = orc.route(inp["q"], kp.contiguous(), inp["w_q"], inp["w_k"], Bq, Bk, k)
    inv = np.argsort(perm)
    for h in range(2):
        for i in range(N // Bq):
            assert np.array_equal(lutp[0, h, i], np.sort(inv[lut[0, h, i]]))


def test_router_projection_identity_and_scale():
    N, d, Bq, Bk, k = 256, 32, 64, 32, 3
    inp = W.gaussian_inputs(1, 2, N, d, 13)
    eye = torch.eye(d)
    a, ga = orc.route(inp["q"], inp["k"], None, None, Bq, Bk, k)
    b, gb = orc.route(inp["q"], inp["k"], eye, eye, Bq, Bk, k)
    assert np.array_equal(a, b)
    np.testing.assert_allclose(ga, gb, rtol=1e-12)
    c, gc = orc.route(inp["q"], inp["k"], 2.0 * inp["w_q"], 0.5 * inp["w_k"], Bq, Bk, k)
    d_, gd = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], Bq, Bk, k)
    assert np.array_equal(c, d_)
    np.testing.assert_allclose(gc, gd, rtol=1e-12)
    e, ge = orc.route(inp["q"], inp["k"], 4.0 * inp["w_q"], inp["w_k"], Bq, Bk, k)
    assert np.array_equal(e, d_)
    np.testing.assert_allclose(ge, 4.0 * gd, rtol=1e-12)


def test_router_extreme_k():
    N, d = 256, 16
    inp = W.gaussian_inputs(1, 1, N, d, 14)
    lut0, g0 = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 64, 32, 0)
    assert lut0.shape == (1, 1, 4, 0) and np.all(np.isinf(g0))
    lutn, gn = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 64, 32, 8)
    assert np.array_equal(lutn, full_lut(1, 1, 4, 8)) and np.all(np.isinf(gn))


def test_router_rejects_bad_shapes():
    inp = W.gaussian_inputs(1, 1, 256, 16, 15)
    with pytest.raises(ValueError):
        orc.route(inp["q"], inp["k"], None, None, 96, 32, 1)      # N % Bq != 0
    with pytest.raises(ValueError):
        orc.route(inp["q"], inp["k"], None, None, 64, 32, 9)      # k > Nk


# --------------------------------------------------------- sparse branch

@pytest.mark.parametrize("N,d,Bq,Bk", [(256, 64, 64, 64), (256, 32, 128, 32), (192, 16, 32, 64)])
def test_sparse_all_selected_is_dense_attention(N, d, Bq, Bk):
    """k = Nk, alpha = 1: the sparse branch is full softmax attention."""
    inp = W.gaussian_inputs(1, 2, N, d, 21)
    alpha = torch.ones(1, 2, N)
    lut = full_lut(1, 2, N // Bq, N // Bk)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], alpha, lut, Bq, Bk)
    ref = dense_sdpa(inp["q"], inp["k"], inp["v"])
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("scale", [0.0, 0.37])
def test_sparse_partial_is_masked_attention(scale):
    """alpha = 1: block-masked softmax attention, renormalised over the kept
    blocks (torch SDPA with a boolean mask)."""
    N, d, Bq, Bk, k = 256, 32, 64, 32, 3
    inp = W.gaussian_inputs(2, 2, N, d, 22)
    alpha = torch.ones(2, 2, N)
    lut = random_lut(2, 2, N // Bq, N // Bk, k, 5)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], alpha, lut, Bq, Bk, sm_scale=scale)
    ref = dense_sdpa(inp["q"], inp["k"], inp["v"], block_mask(lut, N, Bq, Bk),
                     scale=scale if scale else None)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)


def test_sparse_empty_selection_is_zero():
    N, d = 128, 16
    inp = W.gaussian_inputs(1, 1, N, d, 23)
    lut = np.zeros((1, 1, 2, 0), dtype=np.int32)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], torch.ones(1, 1, N), lut, 64, 32)
    assert np.all(out == 0.0)


def test_sparse_shift_invariance():
    """Adding one vector u to every key shifts each row's logits by q.u: the
    sparse branch is unchanged.  Keys and u are multiples of 1/8 so k + u is
    exact in bf16."""
    N, d, Bq, Bk, k = 128, 16, 32, 32, 2
    g = torch.Generator().manual_seed(3)
    q = (torch.randint(-8, 9, (1, 1, N, d), generator=g) / 8).to(torch.bfloat16)
    kk = (torch.randint(-8, 9, (1, 1, N, d), generator=g) / 8).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    u = (torch.randint(-8, 9, (d,), generator=g) / 8)
    ku = (kk.float() + u).to(torch.bfloat16)
    assert torch.equal(ku.float(), kk.float() + u)
    lut = random_lut(1, 1, N // Bq, N // Bk, k, 7)
    ones = torch.ones(1, 1, N)
    a = orc.sla_forward(q, kk, v, ones, lut, Bq, Bk)
    b = orc.sla_forward(q, ku, v, ones, lut, Bq, Bk)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


# --------------------------------------------------------- linear branch

def pairwise_linear(q, k, v, keep=None):
    """Textbook ReLU linear attention in its O(N^2) pairwise form:
    sum_n (phi(q).phi(k_n)) v_n / sum_n phi(q).phi(k_n); 0 if the denominator
    is not positive.  keep: boolean [.., N, N] of pairs that take part."""
    a = np.maximum(f64(q).numpy(), 0) @ np.swapaxes(np.maximum(f64(k).numpy(), 0), -1, -2)
    if keep is not None:
        a = a * keep
    num = a @ f64(v).numpy()
    den = a.sum(-1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(den > 0, num / np.where(den > 0, den, 1), 0.0)


def test_linear_no_selection_is_pairwise_linear_attention():
    N, d, Bq, Bk = 256, 32, 64, 32
    inp = W.gaussian_inputs(1, 2, N, d, 31)
    lut = np.zeros((1, 2, N // Bq, 0), dtype=np.int32)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], torch.zeros(1, 2, N), lut, Bq, Bk)
    ref = pairwise_linear(inp["q"], inp["k"], inp["v"])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_linear_covers_only_unselected_blocks():
    N, d, Bq, Bk, k = 256, 32, 64, 32, 3
    inp = W.gaussian_inputs(1, 2, N, d, 32)
    lut = random_lut(1, 2, N // Bq, N // Bk, k, 9)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], torch.zeros(1, 2, N), lut, Bq, Bk)
    keep = ~block_mask(lut, N, Bq, Bk).numpy()
    ref = pairwise_linear(inp["q"], inp["k"], inp["v"], keep)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_linear_scale_invariance():
    """phi = ReLU is positively homogeneous: scaling q or k by 2^e > 0 leaves
    the linear branch unchanged (power-of-two scales are exact in bf16)."""
    N, d, Bq, Bk, k = 256, 32, 64, 32, 2
    inp = W.gaussian_inputs(1, 1, N, d, 33)
    lut = random_lut(1, 1, N // Bq, N // Bk, k, 3)
    zero = torch.zeros(1, 1, N)
    a = orc.sla_forward(inp["q"], inp["k"], inp["v"], zero, lut, Bq, Bk)
    b = orc.sla_forward(inp["q"] * 4, inp["k"] * 0.5, inp["v"], zero, lut, Bq, Bk)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_linear_nonpositive_denominator_gives_zero():
    N, d, Bq, Bk = 128, 16, 64, 32
    inp = W.gaussian_inputs(1, 1, N, d, 34)
    qneg = -inp["q"].abs()
    lut = random_lut(1, 1, N // Bq, N // Bk, 1, 1)
    out = orc.sla_forward(qneg, inp["k"], inp["v"], torch.zeros(1, 1, N), lut, Bq, Bk)
    assert np.all(out == 0.0)


# ---------------------------------------------------------------- combine

def test_combine_is_affine_in_alpha():
    N, d, Bq, Bk, k = 256, 32, 64, 32, 3
    inp = W.gaussian_inputs(1, 2, N, d, 41)
    lut = random_lut(1, 2, N // Bq, N // Bk, k, 4)
    out, os_, ol = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, Bk,
                                   branches=True)
    one = orc.sla_forward(inp["q"], inp["k"], inp["v"], torch.ones(1, 2, N), lut, Bq, Bk)
    zero = orc.sla_forward(inp["q"], inp["k"], inp["v"], torch.zeros(1, 2, N), lut, Bq, Bk)
    np.testing.assert_allclose(os_, one, rtol=0, atol=1e-13)
    np.testing.assert_allclose(ol, zero, rtol=0, atol=1e-13)
    a = inp["alpha"].double().numpy()[..., None]
    np.testing.assert_allclose(out, a * one + (1 - a) * zero, rtol=0, atol=1e-12)


def test_sla_brute_force_matrix_form():
    """The whole forward in explicit N x N matrix form on a tiny case."""
    N, d, Bq, Bk, k = 256, 16, 64, 32, 3
    inp = W.gaussian_inputs(1, 2, N, d, 42)
    lut = random_lut(1, 2, N // Bq, N // Bk, k, 8)
    out = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, Bk)
    m = block_mask(lut, N, Bq, Bk).numpy()
    q, kk, v = (f64(inp[x]).numpy() for x in "qkv")
    logits = (q @ np.swapaxes(kk, -1, -2)) / math.sqrt(d)
    logits = np.where(m, logits, -np.inf)
    p = np.exp(logits - logits.max(-1, keepdims=True))
    os_ = (p / p.sum(-1, keepdims=True)) @ v
    a = np.maximum(q, 0) @ np.swapaxes(np.maximum(kk, 0), -1, -2) * (~m)
    ol = (a @ v) / a.sum(-1, keepdims=True)
    al = inp["alpha"].double().numpy()[..., None]
    np.testing.assert_allclose(out, al * os_ + (1 - al) * ol, rtol=0, atol=1e-11)


def test_row_sampling_matches_full_output():
    N, d, Bq, Bk, k = 256, 32, 128, 64, 2
    inp = W.gaussian_inputs(2, 2, N, d, 43)
    lut = random_lut(2, 2, N // Bq, N // Bk, k, 2)
    full = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, Bk)
    rows = np.array([1000, 3, 517, 1023, 64, 65])
    part = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, Bq, Bk, rows=rows)
    np.testing.assert_array_equal(part, full.reshape(-1, d)[rows])
    pp = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut, Bq, Bk, rows=rows)
    pf = orc.pisa_forward(inp["q"], inp["k"], inp["v"], lut, Bq, Bk)
    np.testing.assert_array_equal(pp, pf.reshape(-1, d)[rows])


def test_oracle_rejects_invalid_lut():
    N, d = 128, 16
    inp = W.gaussian_inputs(1, 1, N, d, 44)
    bad = np.array([[[[0, 0], [1, 2]]]], dtype=np.int32)            # duplicate
    with pytest.raises(ValueError):
        orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], bad, 64, 32)
    bad = np.array([[[[0, 4], [1, 2]]]], dtype=np.int32)            # out of range
    with pytest.raises(ValueError):
        orc.pisa_forward(inp["q"], inp["k"], inp["v"], bad, 64, 32)


# ------------------------------------------------------------------- PISA

def test_pisa_all_exact_is_dense_attention():
    N, d, B_ = 256, 32, 64
    inp = W.gaussian_inputs(1, 2, N, d, 51)
    out = orc.pisa_forward(inp["q"], inp["k"], inp["v"], full_lut(1, 2, N // B_, N // B_), B_, B_)
    np.testing.assert_allclose(out, dense_sdpa(inp["q"], inp["k"], inp["v"]), rtol=0, atol=1e-11)


def block_constant_keys(B, H, N, d, Bk, seed):
    g = torch.Generator().manual_seed(seed)
    kb = torch.randn(B, H, N // Bk, 1, d, generator=g).to(torch.bfloat16)
    return kb.expand(B, H, N // Bk, Bk, d).reshape(B, H, N, d).contiguous()


@pytest.mark.parametrize("k", [0, 1, 3, 4])
def test_pisa_zero_order_exact_for_block_constant_keys(k):
    """If every key of a block equals its centroid, the zero-order term is
    the exact block contribution: PISA equals dense attention for any k."""
    N, d, B_ = 256, 32, 32
    inp = W.gaussian_inputs(1, 2, N, d, 52)
    kc = block_constant_keys(1, 2, N, d, B_, 9)
    lut = random_lut(1, 2, N // B_, N // B_, k, 10 + k)
    out = orc.pisa_forward(inp["q"], kc, inp["v"], lut, B_, B_)
    np.testing.assert_allclose(out, dense_sdpa(inp["q"], kc, inp["v"]), rtol=0, atol=1e-11)


def test_pisa_no_exact_block_closed_form():
    """k = 0 with block-constant keys: softmax over the centroids, each with
    multiplicity Bk, applied to the block mean values."""
    N, d, B_ = 256, 16, 64
    inp = W.gaussian_inputs(1, 1, N, d, 53)
    kc = block_constant_keys(1, 1, N, d, B_, 11)
    lut = np.zeros((1, 1, N // B_, 0), dtype=np.int32)
    out = orc.pisa_forward(inp["q"], kc, inp["v"], lut, B_, B_)
    q = f64(inp["q"]).numpy()[0, 0]
    cent = f64(kc).numpy()[0, 0, ::B_]                           # [Nk, d]
    vmean = f64(inp["v"]).numpy()[0, 0].reshape(N // B_, B_, d).mean(1)
    c = q @ cent.T / math.sqrt(d)
    w = np.exp(c - c.max(-1, keepdims=True))
    ref = (w @ vmean) / w.sum(-1, keepdims=True)
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-12)


def test_pisa_zero_order_error_is_first_order():
    """Keys = centroid + eps * delta (delta zero-mean within each block): the
    zero-order approximation error against dense attention is O(eps), so
    halving eps halves it.  All values are exact in bf16."""
    N, d, B_, k = 256, 16, 32, 2
    g = torch.Generator().manual_seed(5)
    base = (torch.randint(-6, 7, (1, 1, N // B_, 1, d), generator=g) / 8.0)
    base = base.expand(1, 1, N // B_, B_, d).reshape(1, 1, N, d)
    sign = torch.randint(0, 2, (1, 1, N // B_, B_ // 2, d), generator=g) * 2.0 - 1.0
    delta = torch.cat([sign, -sign], 3).reshape(1, 1, N, d)      # zero mean per block
    q = (torch.randint(-8, 9, (1, 1, N, d), generator=g) / 4.0).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    lut = random_lut(1, 1, N // B_, N // B_, k, 12)
    errs = []
    for e in (2.0 ** -4, 2.0 ** -5, 2.0 ** -6):
        kk = (base + e * delta).to(torch.bfloat16)
        assert torch.equal(kk.double(), (base + e * delta).double())
        out = orc.pisa_forward(q, kk, v, lut, B_, B_)
        errs.append(np.abs(out - dense_sdpa(q, kk, v)).max())
    assert errs[0] > errs[1] > errs[2] > 0
    for a, b in zip(errs, errs[1:]):
        assert 1.6 < a / b < 2.5, errs


# ---------------------------------------------------------------- E4M3 and the FP8 mode

def e4m3_decode(code):
    """Value of one 8-bit E4M3 code, from the format's definition: sign bit,
    4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal;
    exponent 15 with mantissa 7 is NaN (no infinities)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table():
    """Non-negative finite values in code order, with their mantissa parity."""
    vals = [e4m3_decode(c) for c in range(0x7F)]
    return np.array(vals), np.array([c & 1 for c in range(0x7F)])


def test_e4m3_codes_are_fixed_points_and_ties_go_to_even():
    vals, odd = e4m3_table()
    assert vals[-1] == 448.0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6
    assert np.all(np.diff(vals) > 0)
    both = np.concatenate([vals, -vals[1:]])
    assert np.array_equal(orc.e4m3(both), both)
    mids = (vals[:-1] + vals[1:]) / 2
    want = np.where(odd[:-1] == 0, vals[:-1], vals[1:])
    assert np.array_equal(orc.e4m3(mids), want)
    assert np.array_equal(orc.e4m3(-mids), -want)
    # just off the midpoints: plain nearest
    assert np.array_equal(orc.e4m3(mids * (1 - 1e-9)), vals[:-1])
    assert np.array_equal(orc.e4m3(mids * (1 + 1e-9)), vals[1:])


def test_e4m3_saturates_and_underflows():
    big = np.array([448.0, 449.0, 463.99, 464.0, 480.0, 1e6, np.inf])
    assert np.array_equal(orc.e4m3(big), np.full(7, 448.0))
    assert np.array_equal(orc.e4m3(-big), np.full(7, -448.0))
    assert np.array_equal(orc.e4m3(np.array([2.0 ** -10, 1e-30, 0.0])), np.zeros(3))
    assert orc.e4m3(np.array([2.0 ** -10 * 1.0001]))[0] == 2.0 ** -9
    assert np.isnan(orc.e4m3(np.array([np.nan]))[0])


def test_e4m3_matches_library_conversion():
    """torch's float8_e4m3fn cast (round to nearest even) on values within range."""
    rng = np.random.default_rng(7)
    mag = 2.0 ** rng.uniform(-11, math.log2(448), 200000)
    x = mag * rng.choice([-1.0, 1.0], mag.size)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(orc.e4m3(x), lib)


def exact_fp8_inputs(seed, v_fifths=False):
    """Inputs on which every FP8 quantisation step is exact: block absmaxes are
    448 * 2^-r (so each scale is a power of two), every entry divided by its
    block scale is an E4M3 value, and with sm_scale = ln 2 the logits in log2
    units are small integers, so each P = 2^(integer) times a power-of-two
    factor is an E4M3 value too.  Q, K and V use different scales per
    64-token block (two Q scale blocks inside one 128-token query block).
    v_fifths: V blocks take absmax 448 * f * 2^-r with f in {1, 5/8}; every
    step except the rounding of P stays exact, and P * 448 s_v,j / s_v,max
    is then a power of two times 448 f_j / f_max, never an E4M3 tie."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 2, 512, 128
    q = np.zeros((B, H, N, d))
    k = np.zeros((B, H, N, d))
    v = np.zeros((B, H, N, d))
    vals, _ = e4m3_table()
    for b in range(B):
        for h in range(H):
            for blk in range(N // 64):
                rq, rk, rv = rng.integers(7, 9), rng.integers(7, 9), rng.integers(6, 10)
                fv = rng.choice([1.0, 0.625]) if v_fifths else 1.0
                for t in range(blk * 64, blk * 64 + 64):
                    cq = rng.choice(np.arange(2, 10), 2, replace=False)
                    q[b, h, t, cq] = rng.choice([-1.0, 1.0], 2) * (rng.choice([1.0, 2.0], 2) if rq == 7 else 1.0)
                    ck = rng.choice(np.arange(2, 10), 3, replace=False)
                    k[b, h, t, ck] = rng.choice([-1.0, 1.0], 3)
                    v[b, h, t] = rng.choice(vals[1:], d) * rng.choice([-1.0, 1.0], d) * fv * 2.0 ** -rv
                # block absmax: column 0 of Q and column 1 of K never meet a nonzero
                q[b, h, blk * 64, 0] = 448.0 * 2.0 ** -rq
                k[b, h, blk * 64, 1] = 448.0 * 2.0 ** -rk
                v[b, h, blk * 64, 5] = 448.0 * fv * 2.0 ** -rv
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16)
    qt, kt, vt = to(q), to(k), to(v)
    for a, x in ((qt, q), (kt, k), (vt, v)):
        assert np.array_equal(a.double().numpy(), x), "construction must be exact in bf16"
    alpha = torch.from_numpy(rng.uniform(0, 1, (B, H, N))).float()
    return qt, kt, vt, alpha


@pytest.mark.parametrize("p_plain", [False, True], ids=["p_pow2", "p_max"])
@pytest.mark.parametrize("topk", [1, 3, 8])
def test_fp8_mode_is_exact_when_every_quantisation_is_exact(topk, p_plain):
    q, k, v, alpha = exact_fp8_inputs(11 + topk)
    Bq, Bk = 128, 64
    lut, _ = orc.route(q, k, None, None, Bq, Bk, topk)
    ln2 = math.log(2.0)
    o8, s8, l8 = orc.sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=ln2, branches=True, fp8=True,
                                 p_plain=p_plain)
    o, s, l = orc.sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=ln2, branches=True)
    scale = np.abs(s).max()
    assert scale > 0
    assert np.abs(s8 - s).max() <= 1e-12 * scale
    assert np.array_equal(l8, l)
    assert np.abs(o8 - o).max() <= 1e-12 * scale
    # the case is not degenerate: within a query block's selected keys the
    # logits (log2 units) span several powers of two
    qd, kd = q.double().numpy()[0, 0], k.double().numpy()[0, 0]
    keys = np.concatenate([np.arange(j * Bk, (j + 1) * Bk) for j in lut[0, 0, 1]])
    spread = np.ptp(qd[Bq:2 * Bq] @ kd[keys].T, axis=1)
    assert spread.max() >= 3


@pytest.mark.parametrize("p_plain", [False, True], ids=["p_pow2", "p_max"])
@pytest.mark.parametrize("topk", [2, 5])
def test_fp8_p_rounding_matches_library_codec_on_known_weights(topk, p_plain):
    """Only the rounding of P is inexact here: every P is a power of two, so
    block j's quantised weights are its exact weights times
    gamma_j = e4m3(448 rho_j) / (448 rho_j), rho_j = s_v,j / s_v,max, with the
    row sum taken over the unquantised P.  The sparse branch must equal fp64
    softmax attention over the selected blocks with V_j scaled by gamma_j
    (E4M3 rounding from torch's float8_e4m3fn cast)."""
    q, k, v, alpha = exact_fp8_inputs(40 + topk, v_fifths=True)
    Bq, Bk = 128, 64
    B, H, N, d = q.shape
    lut, _ = orc.route(q, k, None, None, Bq, Bk, topk)
    ln2 = math.log(2.0)
    _, s8, _ = orc.sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=ln2, branches=True, fp8=True,
                               p_plain=p_plain)
    qd, kd, vd = f64(q), f64(k), f64(v)
    s_v = vd.reshape(B, H, N // 64, 64 * d).abs().amax(-1) / 448.0
    want = torch.zeros(B, H, N, d, dtype=torch.float64)
    nontrivial = 0
    for b in range(B):
        for h in range(H):
            for i in range(N // Bq):
                sel = torch.as_tensor(lut[b, h, i], dtype=torch.long)
                rho = s_v[b, h, sel] / s_v[b, h, sel].max()
                gamma = (448.0 * rho).to(torch.float8_e4m3fn).double() / (448.0 * rho)
                nontrivial += int((gamma != 1).sum())
                keys = torch.cat([torch.arange(j * Bk, (j + 1) * Bk) for j in sel.tolist()])
                vj = vd[b, h, keys] * gamma.repeat_interleave(Bk)[:, None]
                rows = slice(i * Bq, (i + 1) * Bq)
                w = torch.softmax(ln2 * qd[b, h, rows] @ kd[b, h, keys].T, dim=-1)
                want[b, h, rows] = w @ vj
    assert nontrivial > 0
    want = want.numpy()
    assert np.abs(s8 - want).max() <= 1e-12 * np.abs(want).max()


def test_fp8_mode_error_has_the_size_the_format_implies():
    """On Gaussian inputs the quantised branch differs from the exact one by
    a few percent (E4M3 keeps 3 mantissa bits): nonzero, and far from gross."""
    inp = W.gaussian_inputs(1, 2, 1024, 128, 77)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 128, 64, 6)
    _, s8, l8 = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, 128, 64,
                                branches=True, fp8=True)
    _, s, l = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, 128, 64, branches=True)
    assert np.array_equal(l8, l)
    rel = np.abs(s8 - s).mean() / np.abs(s).mean()
    assert 0.005 < rel < 0.1, rel
    cos = (s8 * s).sum() / np.sqrt((s8 * s8).sum() * (s * s).sum())
    assert cos > 0.99


def test_fp8_mode_requires_64_token_blocks():
    inp = W.gaussian_inputs(1, 1, 256, 64, 5)
    lut, _ = orc.route(inp["q"], inp["k"], None, None, 64, 32, 2)
    with pytest.raises(ValueError):
        orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut, 64, 32, fp8=True)


# ------------------------------------------- 8-bit codes: the exact quotient rule
# A code rounds the exact quotient top * x / max|x| of its 64-token block
# (top = 448 for E4M3, 127 for the integer code).

def _exact_code(r, int8):
    """Rounding of the exact rational r: to the nearest E4M3 value (ties to the
    even mantissa, from the format table) or to the nearest integer within
    +-127 (ties to even)."""
    from fractions import Fraction
    if int8:
        lo = math.floor(r)
        frac = r - lo
        n = lo + (1 if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2) else 0)
        return float(max(-127, min(127, n)))
    vals, odd = e4m3_table()
    a = abs(r)
    fv = [Fraction(float(x)) for x in vals]
    j = max(i for i in range(len(fv)) if fv[i] <= a)
    if j == len(fv) - 1:
        c = fv[j]
    else:
        lo, hi = fv[j], fv[j + 1]
        if a - lo < hi - a or (a - lo == hi - a and odd[j] == 0):
            c = lo
        else:
            c = hi
    return float(c) if r >= 0 else -float(c)


def _midpoint_blocks(int8, seed):
    """bf16 blocks [64 * nb, 64] whose entries include exact rounding midpoints
    of top * x / max|x| for block maxima that are not powers of two, plus random
    entries; the block maximum sits in column 63 of the block's first row."""
    rng = np.random.default_rng(seed)
    top = 127.0 if int8 else 448.0
    amaxes = [448.0, 7.0, 5.0, 3.0, 13.0, 0.75, 127.0, 100.0, 254.0, 1.25, 135.0, 149.0]
    in_bf16 = lambda t: float(torch.tensor(t).to(torch.bfloat16)) == t
    x = np.zeros((64 * len(amaxes), 64))
    n_mid = 0
    for b, A in enumerate(amaxes):
        blk = rng.uniform(-A, A, (64, 64))
        mids = []
        if int8:
            mids.append(A / 2)                                   # 63.5 exactly
            if A == 127.0 or A == 254.0:                         # power-of-two scales
                mids += [(k + 0.5) * A / 127 for k in range(-20, 20)]
        else:
            for f in range(-8, 4):
                for M in (7, 21):
                    mids.append(A * (M / 7) * 2.0 ** f / 64)     # top x / A = M 2^(f-1)
                    if A == 448.0:
                        mids += [(2 * c + 1) * 2.0 ** (f - 1) for c in range(8, 16)]
            mids.append(A * 2.0 ** -16)                          # the subnormal midpoint 7 2^-10
        mids = [m for m in mids if in_bf16(m)]
        mids = [m for m in mids if abs(m) < A]
        flat = blk.reshape(-1)
        flat[:len(mids)] = mids
        flat[len(mids):2 * len(mids)] = -np.array(mids)
        blk[0, 63] = A
        x[64 * b:64 * b + 64] = blk
        n_mid += len(mids)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    return xt, amaxes, top, n_mid


@pytest.mark.parametrize("int8", [False, True], ids=["e4m3", "int8"])
def test_codes_round_the_exact_quotient(int8):
    from fractions import Fraction
    xt, amaxes, top, n_mid = _midpoint_blocks(int8, 3 + int8)
    xd = xt.double().numpy()
    codes, scales = orc.quantise(xt, int8=int8)
    assert np.allclose(scales, np.array(amaxes) / top, rtol=0, atol=0)
    ties = 0
    for b, A in enumerate(amaxes):
        for t in range(64 * b, 64 * b + 64):
            for c in range(0, 64, 1 if t < 64 * b + 8 else 7):
                r = Fraction(top) * Fraction(float(xd[t, c])) / Fraction(A)
                want = _exact_code(r, int8)
                assert codes[t, c] == want, (A, xd[t, c], codes[t, c], want)
                half = r * 2 if int8 else None
                ties += int(int8 and half.denominator == 1 and half.numerator % 2 == 1)
    assert n_mid > 20 and (ties > 0 or not int8)


@pytest.mark.parametrize("int8", [False, True], ids=["e4m3", "int8"])
def test_fp32_quotient_decides_the_same_codes(int8):
    """Every bf16 x with |x| <= A, for block maxima A: the code of the fp32
    quotient fl32(fl32(top * x) / A) (top * x is exact in fp32) equals the code
    of the exact quotient, so a kernel can decide codes in fp32 without
    changing one.  Dividing by a rounded scale fl32(A / top) first does not:
    near exact midpoints it breaks ties by rounding noise."""
    top = 127.0 if int8 else 448.0
    code = orc.int8 if int8 else orc.e4m3
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    allx = (bits << 16).view(np.float32)
    allx = allx[np.isfinite(allx)]
    rng = np.random.default_rng(12)
    amaxes = [5.0, 7.0, 13.0, 3.0, 448.0, 127.0, 1.0, 0.75, 254.0, 6.0e-39]
    amaxes += [float(torch.tensor(a).to(torch.bfloat16)) for a in 2.0 ** rng.uniform(-20, 20, 20)]
    flips_scale_first = 0
    for A in amaxes:
        x = allx[np.abs(allx) <= A].astype(np.float64)
        exact = code((top * x) / A)
        q32 = (np.float32(top) * x.astype(np.float32)) / np.float32(A)
        assert np.array_equal(code(q32.astype(np.float64)), exact), A
        s32 = np.float32(A) / np.float32(top)
        flips_scale_first += int((code((x.astype(np.float32) / s32).astype(np.float64)) != exact).sum())
    assert flips_scale_first > 0


def _fp8_errors(inp, k, mode):
    """Mean and max distance (std units of the exact output) from the exact
    forward of the quantised branch with P against the power of two at or
    above the row maximum and against the row maximum itself, and between the two."""
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 128, 64, k)
    a = (inp["q"], inp["k"], inp["v"], inp["alpha"], lut, 128, 64)
    ex = orc.sla_forward(*a)
    std = ex.std()
    p2 = orc.sla_forward(*a, **{mode: True})
    pl = orc.sla_forward(*a, p_plain=True, **{mode: True})
    f = lambda x, y: (np.abs(x - y).mean() / std, np.abs(x - y).max() / std)
    return f(p2, ex), f(pl, ex), f(p2, pl)


@pytest.mark.parametrize("mode", ["fp8", "int8"])
@pytest.mark.parametrize("family", ["gaussian", "video"])
def test_power_of_two_p_reference_is_not_load_bearing(mode, family):
    """The two readings of P's reference quantise different values (their
    outputs differ by about as much as either differs from the exact branch's
    P-rounding share), but their errors against the exact forward agree: mean
    within 5%, max within 40%, on both input families."""
    if family == "gaussian":
        inp = W.gaussian_inputs(1, 2, 2048, 128, 901)
    else:
        inp = W.video_inputs(1, 2, 2048, 128, (6, 16, 21), 902)
    (m2, x2), (mp, xp), (md, _) = _fp8_errors(inp, 6, mode)
    assert abs(m2 - mp) <= 0.05 * mp, (m2, mp)
    assert abs(x2 - xp) <= 0.4 * max(x2, xp), (x2, xp)
    assert 0.3 * mp < md < 1.2 * mp, (md, mp)


# ---------------------------------------------------------------- PISA first-order term

def test_pisa_first_order_vanishes_for_block_constant_keys():
    """Block-constant keys give H_j = 0, hence Hbar = 0: the first-order mode
    equals the zero-order mode, which is exact (dense attention)."""
    N, d, Bq, k = 512, 32, 64, 3
    g = torch.Generator().manual_seed(17)
    kb = torch.randn(1, 2, N // 64, 1, d, generator=g)
    kk = kb.expand(1, 2, N // 64, 64, d).reshape(1, 2, N, d).to(torch.bfloat16)
    q = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    lut = random_lut(1, 2, N // Bq, N // 64, k, 4)
    a = orc.pisa_forward(q, kk, v, lut, Bq, 64, first_order=True)
    b = orc.pisa_forward(q, kk, v, lut, Bq, 64)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()
    assert np.abs(a - dense_sdpa(q, kk, v)).max() <= 1e-10


def test_pisa_first_order_error_is_second_order():
    """Keys = centroid + eps * delta with the same zero-mean delta pattern and the
    same values in every block, so every block's first-order matrix H_j equals
    Hbar.  Against dense attention the zero-order error is O(eps) (halving eps
    halves it) and the first-order-corrected error is O(eps^2) (halving eps
    quarters it), and smaller.  All inputs are exact in bf16."""
    N, d, B_, k = 256, 16, 32, 2
    g = torch.Generator().manual_seed(6)
    base = (torch.randint(-6, 7, (1, 1, N // B_, 1, d), generator=g) / 8.0)
    base = base.expand(1, 1, N // B_, B_, d).reshape(1, 1, N, d)
    sign = torch.randint(0, 2, (1, 1, 1, B_ // 2, d), generator=g) * 2.0 - 1.0
    delta = torch.cat([sign, -sign], 3).expand(1, 1, N // B_, B_, d).reshape(1, 1, N, d)
    q = (torch.randint(-8, 9, (1, 1, N, d), generator=g) / 4.0).to(torch.bfloat16)
    vb = torch.randn(1, 1, 1, B_, d, generator=g)
    v = vb.expand(1, 1, N // B_, B_, d).reshape(1, 1, N, d).to(torch.bfloat16)
    lut = random_lut(1, 1, N // B_, N // B_, k, 13)
    e0, e1 = [], []
    for e in (2.0 ** -4, 2.0 ** -5, 2.0 ** -6):
        kk = (base + e * delta).to(torch.bfloat16)
        assert torch.equal(kk.double(), (base + e * delta).double())
        dense = dense_sdpa(q, kk, v)
        e0.append(np.abs(orc.pisa_forward(q, kk, v, lut, B_, B_) - dense).max())
        e1.append(np.abs(orc.pisa_forward(q, kk, v, lut, B_, B_, first_order=True) - dense).max())
    for a, b in zip(e0, e0[1:]):
        assert 1.6 < a / b < 2.5, e0
    for a, b in zip(e1, e1[1:]):
        assert 3.2 < a / b < 5.0, e1
    assert all(x1 < 0.5 * x0 for x0, x1 in zip(e0, e1)), (e0, e1)


# ---------------------------------------------------------------- INT8 Q/K codes

def test_int8_codes_match_library_rounding():
    """Nearest integer with ties to even (numpy's rint), clamped to +-127."""
    rng = np.random.default_rng(9)
    x = np.concatenate([rng.uniform(-140, 140, 100000), np.arange(-130, 131) + 0.5,
                        np.array([127.4999, 127.5, -127.5, 0.0, -0.5])])
    assert np.array_equal(orc.int8(x), np.clip(np.rint(x), -127, 127))


def exact_int8_inputs(seed):
    """Q entries are integers times 1/2 with a block absmax of 127/2 (scale 1/2),
    K entries integers with a block absmax of 127 (scale 1): every code is exact,
    q . k is an integer times 1/2, and with sm_scale = 2 ln 2 the logits in log2
    units are integers.  V follows the exact E4M3 construction."""
    q, k, v, alpha = exact_fp8_inputs(seed)
    rng = np.random.default_rng(seed + 1000)
    B, H, N, d = q.shape
    qn = np.zeros((B, H, N, d))
    kn = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            for blk in range(N // 64):
                for t in range(blk * 64, blk * 64 + 64):
                    cq = rng.choice(np.arange(2, 10), 2, replace=False)
                    qn[b, h, t, cq] = rng.choice([-1.0, 1.0, -2.0, 2.0], 2) * 0.5
                    ck = rng.choice(np.arange(2, 10), 3, replace=False)
                    kn[b, h, t, ck] = rng.choice([-1.0, 1.0], 3)
                qn[b, h, blk * 64, 0] = 63.5
                kn[b, h, blk * 64, 1] = 127.0
    to = lambda x: torch.from_numpy(x).to(torch.bfloat16)
    return to(qn), to(kn), v, alpha


@pytest.mark.parametrize("p_plain", [False, True], ids=["p_pow2", "p_max"])
@pytest.mark.parametrize("topk", [1, 3, 8])
def test_int8_mode_is_exact_when_every_quantisation_is_exact(topk, p_plain):
    q, k, v, alpha = exact_int8_inputs(21 + topk)
    Bq, Bk = 128, 64
    lut, _ = orc.route(q, k, None, None, Bq, Bk, topk)
    sc = 2.0 * math.log(2.0)
    o8, s8, l8 = orc.sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=sc, branches=True, int8=True,
                                 p_plain=p_plain)
    o, s, l = orc.sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=sc, branches=True)
    scale = np.abs(s).max()
    assert np.abs(s8 - s).max() <= 1e-12 * scale
    assert np.abs(o8 - o).max() <= 1e-12 * scale
    # not degenerate: the logits of a query block's selected keys span several units
    qd, kd = q.double().numpy()[0, 0], k.double().numpy()[0, 0]
    keys = np.concatenate([np.arange(j * Bk, (j + 1) * Bk) for j in lut[0, 0, 1]])
    assert np.ptp(qd[Bq:2 * Bq] @ kd[keys].T, axis=1).max() >= 2


def test_int8_mode_error_is_below_fp8():
    """Q, K as 8-bit integers keep more precision than E4M3, so on Gaussian inputs
    the INT8 mode's distance from the exact branch is nonzero and below FP8's."""
    inp = W.gaussian_inputs(1, 2, 1024, 128, 78)
    lut, _ = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 128, 64, 6)
    args = (inp["q"], inp["k"], inp["v"], inp["alpha"], lut, 128, 64)
    _, s, _ = orc.sla_forward(*args, branches=True)
    _, s8, _ = orc.sla_forward(*args, branches=True, fp8=True)
    _, si, _ = orc.sla_forward(*args, branches=True, int8=True)
    e8, ei = np.abs(s8 - s).mean(), np.abs(si - s).mean()
    assert 0 < ei < 0.8 * e8, (ei, e8)
    assert not np.array_equal(si, s8)


# ------------------------------------------------ PISA covariance-aware routing
# [PISA] sec. 2 "Routing Consapevole della Covarianza": M_j = ||H_j - Hbar||_2.

def _cov_blocks(Nk, d, Bk=64):
    """Keys and values (float32, exact in bf16) of Nk blocks with block-constant
    keys: every first-order matrix H_j is zero."""
    rng = np.random.default_rng(31)
    k = np.repeat(rng.integers(-8, 9, size=(Nk, 1, d)) / 4.0, Bk, axis=1)
    v = rng.integers(-8, 9, size=(Nk, Bk, d)) / 4.0
    return k, v


def _signed_pairs(Bk):
    s = np.ones(Bk)
    s[1::2] = -1.0                      # +1, -1, ...: zero sum in every half
    return s


def _as_input(x):
    return torch.as_tensor(x.reshape(1, 1, -1, x.shape[-1]), dtype=torch.float32).to(torch.bfloat16)


def test_cov_norms_vanish_for_block_constant_keys():
    k, v = _cov_blocks(6, 64)
    m = orc.block_cov_norms(_as_input(k), _as_input(v), 64)
    assert np.array_equal(m, np.zeros((1, 1, 6)))


def test_cov_norms_are_spectral_about_the_mean():
    """Block 0: centred keys +-a e1 (tokens 0-31) and +-b e2 (tokens 32-63) with
    values of the same signs along e1, e2, so H_0 = diag(32 a, 32 b); block 1
    the same keys with negated values (H_1 = -H_0); blocks 2, 3 constant keys.
    Hbar = 0, so M_0 = M_1 = 32 max(a, b) (the Frobenius norm would give
    32 sqrt(a^2 + b^2)) and M_2 = M_3 = 0."""
    d, Bk, a, b = 64, 64, 1.5, 0.75
    k, v = _cov_blocks(4, d)
    s = _signed_pairs(Bk)
    for j, sign in ((0, 1.0), (1, -1.0)):
        v[j] = 0.0
        k[j, :32, 0] += a * s[:32]
        k[j, 32:, 1] += b * s[32:]
        v[j, :32, 0] = sign * s[:32]
        v[j, 32:, 1] = sign * s[32:]
    m = orc.block_cov_norms(_as_input(k), _as_input(v), Bk)[0, 0]
    np.testing.assert_allclose(m, [32 * a, 32 * a, 0.0, 0.0], rtol=0, atol=1e-12)


def test_cov_norms_subtract_the_mean_matrix():
    """Only block 0 has a first-order matrix: its 64 centred keys are +-a e1 with
    values of the same sign along e1, so H_0 = 64 a E_11.  Hbar = H_0 / Nk, so
    M_0 = (1 - 1/Nk) 64 a and every other block has M = 64 a / Nk."""
    d, Bk, a, Nk = 64, 64, 1.25, 4
    k, v = _cov_blocks(Nk, d)
    s = _signed_pairs(Bk)
    k[0, :, 0] += a * s
    v[0] = 0.0
    v[0, :, 0] = s
    m = orc.block_cov_norms(_as_input(k), _as_input(v), Bk)[0, 0]
    np.testing.assert_allclose(m, [(1 - 1 / Nk) * 64 * a] + [64 * a / Nk] * (Nk - 1), rtol=0, atol=1e-12)


def test_cov_norms_ignore_a_shift_of_a_blocks_keys():
    rng = np.random.default_rng(32)
    k = rng.integers(-16, 17, size=(8, 64, 64)) / 8.0
    v = rng.integers(-16, 17, size=(8, 64, 64)) / 8.0
    m0 = orc.block_cov_norms(_as_input(k), _as_input(v), 64)
    k[3] += rng.integers(-8, 9, size=(1, 64)) / 8.0          # exact in bf16
    m1 = orc.block_cov_norms(_as_input(k), _as_input(v), 64)
    np.testing.assert_allclose(m1, m0, rtol=1e-12, atol=0)
    assert np.all(m0 > 0)


def test_cov_routing_lambda_zero_is_plain_routing():
    inp = W.gaussian_inputs(1, 2, 2048, 64, 33)
    plain, gap = orc.route(inp["q"], inp["k"], None, None, 64, 64, 7)
    cov, gap0 = orc.route_cov(inp["q"], inp["k"], inp["v"], 64, 64, 7, 0.0)
    assert np.array_equal(plain, cov) and np.array_equal(gap, gap0)


def test_cov_routing_large_lambda_ranks_blocks_by_norm():
    """With a huge weight every query block selects the top-k blocks of M (the
    same set for all rows), written in ascending order; a moderate weight
    changes some rows relative to plain routing."""
    B, H, N, d, Bq, Bk, k = 1, 2, 2048, 64, 64, 64, 5
    inp = W.gaussian_inputs(B, H, N, d, 34)
    m = orc.block_cov_norms(inp["k"], inp["v"], Bk)
    lut, _ = orc.route_cov(inp["q"], inp["k"], inp["v"], Bq, Bk, k, 1e12)
    for h in range(H):
        top = np.sort(np.argsort(-m[0, h], kind="stable")[:k])
        assert np.array_equal(lut[0, h], np.broadcast_to(top, lut[0, h].shape))
    plain, _ = orc.route(inp["q"], inp["k"], None, None, Bq, Bk, k)
    some, _ = orc.route_cov(inp["q"], inp["k"], inp["v"], Bq, Bk, k, 0.5)
    assert not np.array_equal(plain, some)


def test_route_with_zero_bias_is_plain_routing():
    """The router's per-block bias path adds nothing when the bias is zero."""
    inp = W.gaussian_inputs(1, 2, 2048, 64, 36)
    plain, gap = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 64, 64, 9)
    zero, gap0 = orc.route(inp["q"], inp["k"], inp["w_q"], inp["w_k"], 64, 64, 9, bias=np.zeros((1, 2, 32)))
    assert np.array_equal(plain, zero) and np.array_equal(gap, gap0)


# ------------------------------------------- SVOO online bidirectional co-clustering
# [SVOO] sec. 2.B: keys assigned by their affinity to the query centroids, then
# queries by their affinity to the updated key centroids, alternately; the
# tokens are then ordered by cluster so that contiguous blocks share a cluster.

def _planted(N, d, C, seed, bias=0.5, shuffle=True, scale=4.0):
    """Tokens of C planted groups (group g: q, k near scale * u_g, with u_g
    orthonormal).  Chunk c of the raster order (N/C tokens) holds a share `bias`
    of group c and the rest spread over the other groups, so the initial query
    centroid of chunk c leans toward u_c.  Returns (q, k bf16 [1,1,N,d], group)."""
    rng = np.random.default_rng(seed)
    u, _ = np.linalg.qr(rng.standard_normal((d, C)))
    u = u.T                                              # [C, d] orthonormal rows
    chunk = N // C
    group = np.zeros(N, dtype=np.int64)
    for c in range(C):
        own = int(round(bias * chunk))
        others = [g for g in range(C) if g != c]
        lab = np.concatenate([np.full(own, c), rng.choice(others, chunk - own)])
        if shuffle:
            rng.shuffle(lab)
        group[c * chunk:(c + 1) * chunk] = lab
    q = scale * u[group] + 0.05 * rng.standard_normal((N, d))
    k = scale * u[group] + 0.05 * rng.standard_normal((N, d))
    to = lambda x: torch.from_numpy(x.reshape(1, 1, N, d)).float().to(torch.bfloat16)
    return to(q), to(k), group


def test_cocluster_single_cluster_is_identity():
    inp = W.gaussian_inputs(1, 2, 512, 64, 81)
    qp, kp, ql, kl = orc.cocluster(inp["q"], inp["k"], 1, 3)
    ident = np.broadcast_to(np.arange(512), qp.shape)
    assert np.array_equal(qp, ident) and np.array_equal(kp, ident)
    assert (ql == 0).all() and (kl == 0).all()


def test_cocluster_recovers_planted_groups():
    """Every key and query of planted group g ends in cluster g, and the orders
    are the stable sorts of the planted groups (one wrong affinity direction,
    swapped roles of queries and keys or a missing mean breaks this)."""
    N, d, C = 1024, 64, 4
    q, k, group = _planted(N, d, C, 82)
    qp, kp, ql, kl = orc.cocluster(q, k, C, 3)
    assert np.array_equal(ql[0, 0], group) and np.array_equal(kl[0, 0], group)
    want = np.argsort(group, kind="stable")
    assert np.array_equal(qp[0, 0], want) and np.array_equal(kp[0, 0], want)


def test_cocluster_block_sorted_input_is_left_in_place():
    """Tokens already grouped in the raster chunks the iteration starts from: the
    order does not change."""
    N, d, C = 1024, 64, 8
    q, k, group = _planted(N, d, C, 83, bias=1.0)
    assert np.array_equal(group, np.repeat(np.arange(C), N // C))
    qp, kp, ql, kl = orc.cocluster(q, k, C, 3)
    assert np.array_equal(qp[0, 0], np.arange(N)) and np.array_equal(kp[0, 0], np.arange(N))


def test_cocluster_labels_are_the_alternating_argmax():
    """On video-shaped inputs: the final query labels maximise the affinity to the
    means of the final key clusters, and the final key labels maximise it to the
    means of the query clusters of the iteration before (empty clusters excluded,
    ties to the lower index), computed here from the labels alone."""
    inp = W.video_inputs(1, 2, 2048, 128, (6, 16, 21), 84)
    C, T = 16, 3
    _, _, ql, kl = orc.cocluster(inp["q"], inp["k"], C, T)
    _, _, ql_prev, _ = orc.cocluster(inp["q"], inp["k"], C, T - 1)
    Qd, Kd = f64(inp["q"]).numpy(), f64(inp["k"]).numpy()

    def centroids(x, lab):
        cnt = np.bincount(lab, minlength=C)
        cent = np.stack([x[lab == c].mean(axis=0) if cnt[c] else np.zeros(x.shape[1]) for c in range(C)])
        return cent, cnt > 0

    for h in range(2):
        kc, kv = centroids(Kd[0, h], kl[0, h])
        aff = Qd[0, h] @ kc.T
        aff[:, ~kv] = -np.inf
        assert np.array_equal(np.argmax(aff, axis=1), ql[0, h])
        qc, qv = centroids(Qd[0, h], ql_prev[0, h])
        aff = Kd[0, h] @ qc.T
        aff[:, ~qv] = -np.inf
        assert np.array_equal(np.argmax(aff, axis=1), kl[0, h])
        # the orders are stable sorts by label
        assert np.array_equal(np.argsort(ql[0, h], kind="stable"), np.argsort(ql[0, h], kind="stable"))


def test_cocluster_planted_groups_are_a_fixed_point():
    q, k, group = _planted(1024, 64, 4, 85)
    a = orc.cocluster(q, k, 4, 2)
    b = orc.cocluster(q, k, 4, 5)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def _permute(inp, qp, kp):
    """Inputs reordered by the co-clustering: queries (and alpha) by q_perm, keys
    and values by k_perm."""
    g = lambda x, p: torch.gather(x, 2, torch.as_tensor(p).unsqueeze(-1).expand(-1, -1, -1, x.shape[-1]))
    out = dict(inp)
    out["q"] = g(inp["q"], qp)
    out["k"] = g(inp["k"], kp)
    out["v"] = g(inp["v"], kp)
    out["alpha"] = torch.gather(inp["alpha"], 2, torch.as_tensor(qp))
    return out


def test_coclustered_dense_attention_equals_unpermuted():
    """All blocks selected with alpha = 1 is dense attention, which does not depend
    on the order of queries or keys: routing and attending in the co-clustered
    order, then putting the rows back, gives the unpermuted result."""
    B, H, N, d, Bq, Bk = 1, 2, 512, 64, 64, 64
    inp = W.gaussian_inputs(B, H, N, d, 86)
    inp["alpha"] = torch.ones(B, H, N)
    qp, kp, _, _ = orc.cocluster(inp["q"], inp["k"], 8, 3)
    assert not np.array_equal(qp, np.broadcast_to(np.arange(N), qp.shape))
    pin = _permute(inp, qp, kp)
    Nk = N // Bk
    lut, _ = orc.route(pin["q"], pin["k"], None, None, Bq, Bk, Nk)
    o_perm = orc.sla_forward(pin["q"], pin["k"], pin["v"], pin["alpha"], lut, Bq, Bk)
    back = np.zeros_like(o_perm)
    for h in range(H):
        back[0, h, qp[0, h]] = o_perm[0, h]
    lut0, _ = orc.route(inp["q"], inp["k"], None, None, Bq, Bk, Nk)
    o = orc.sla_forward(inp["q"], inp["k"], inp["v"], inp["alpha"], lut0, Bq, Bk)
    assert np.abs(back - o).max() <= 1e-12 * np.abs(o).max()


def test_cocluster_empty_cluster_is_no_candidate():
    """Queries of the two raster chunks point along +u and -u, every key along +u:
    all keys join cluster 0, cluster 1 gets no key and so no key centroid, and
    every query must then join cluster 0 (a stale or zero centroid for cluster 1
    would attract the -u queries)."""
    N, d = 256, 64
    u = np.zeros(d)
    u[3] = 1.0
    q = np.concatenate([np.tile(u, (N // 2, 1)), np.tile(-u, (N // 2, 1))])
    k = np.tile(u, (N, 1)) * 0.5
    to = lambda x: torch.from_numpy(x.reshape(1, 1, N, d)).float().to(torch.bfloat16)
    _, _, ql, kl = orc.cocluster(to(q), to(k), 2, 2)
    assert (kl == 0).all() and (ql == 0).all()

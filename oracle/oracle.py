"""Python front end of the CPU oracle (``sla_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only users.  The product path never imports this.

The C file is compiled here with gcc (``-O2 -fopenmp``, IEEE double, no
fast-math) into ``oracle/liboracle.so``; numpy marshals the buffers.
Functions:

* :func:`route`        -- pooled, projected top-k block routing (SLA2 router),
  optionally with a per-block score bias
* :func:`block_cov_norms`, :func:`route_cov` -- PISA covariance-aware routing
  (spectral norms of the blocks' first-order matrices about their mean)
* :func:`sla_forward`  -- sparse branch + ReLU linear branch + alpha combine
  (``fp8=True``: the sparse branch on E4M3-quantised Q, K, P, V)
* :func:`quantise`     -- the per-block codes and scales of the 8-bit branches
* :func:`e4m3`         -- the E4M3 conversion (round to nearest even, saturating)
* :func:`int8`         -- the symmetric 8-bit integer code (nearest, ties to even)
* :func:`pisa_forward` -- PISA exact-or-approximate forward (zero-order terms,
  optionally the global first-order correction)
* :func:`cocluster`    -- SVOO online bidirectional Q-K co-clustering (token
  permutations that group tokens of one co-cluster into contiguous blocks)

Inputs may be torch tensors (bf16 / fp32 / int32, on the CPU) or numpy arrays
(bf16 given as uint16 bit patterns).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wno-unknown-pragmas", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_int64
            D = ctypes.c_double
            lib.oracle_route.argtypes = [I] * 7 + [P] * 7 + [I]
            lib.oracle_route.restype = I
            lib.oracle_sla_forward.argtypes = [I] * 7 + [D] + [P] * 5 + [L, P, P, P, P, I, I, I]
            lib.oracle_sla_forward.restype = I
            lib.oracle_pisa_forward.argtypes = [I] * 7 + [D] + [P] * 4 + [L, P, P, I, I]
            lib.oracle_pisa_forward.restype = I
            lib.oracle_e4m3_array.argtypes = [P, P, L]
            lib.oracle_e4m3_array.restype = None
            lib.oracle_int8_array.argtypes = [P, P, L]
            lib.oracle_int8_array.restype = None
            lib.oracle_quantise.argtypes = [P, I, I, I, P, P]
            lib.oracle_quantise.restype = I
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = I
            _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def _bf16_bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch  # noqa: F401  (only for the dtype view)
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                    .view(np.uint16))
    a = np.asarray(x)
    assert a.dtype == np.uint16, "bf16 inputs must be torch.bfloat16 or uint16 bit patterns"
    return np.ascontiguousarray(a)


def _np(x, dtype):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, name):
    if rc != 0:
        raise ValueError("%s: oracle rejected the arguments (code %d)" % (name, rc))


def route(q, k, w_q, w_k, Bq, Bk, topk, threads=0, bias=None):
    """Returns (lut int32 [B,H,N/Bq,topk] ascending, gap float64 [B,H,N/Bq]).
    bias (float64 [B,H,N/Bk], optional) is added to every score of KV block j."""
    qb, kb = _bf16_bits(q), _bf16_bits(k)
    B, H, N, d = qb.shape
    wq, wk = _np(w_q, np.float32), _np(w_k, np.float32)
    bs = None if bias is None else np.ascontiguousarray(np.asarray(bias, dtype=np.float64).reshape(B * H, N // Bk))
    lut = np.zeros((B, H, N // Bq, topk), dtype=np.int32)
    gap = np.zeros((B, H, N // Bq), dtype=np.float64)
    rc = _load().oracle_route(B, H, N, d, Bq, Bk, topk, _ptr(qb), _ptr(kb), _ptr(wq), _ptr(wk),
                              _ptr(bs), _ptr(lut), _ptr(gap), threads)
    _check(rc, "route")
    return lut, gap


def block_cov_norms(k, v, Bk):
    """PISA block covariance norms ([PISA] sec. 2, "Routing Consapevole della
    Covarianza"): M_j = ||H_j - Hbar||_2, the largest singular value of the
    block's first-order matrix H_j = sum_{n in j} (k_n - kbar_j)^T v_n minus
    their mean over the head's blocks, Hbar = (1/Nk) sum_j H_j.  fp64 from the
    bf16 inputs; the singular values come from numpy's SVD.  Returns [B,H,N/Bk]."""
    kb = _bf16_bits(k)
    B, H, N, d = kb.shape
    Nk = N // Bk
    kd = kb.astype(np.uint32).__lshift__(16).view(np.float32).astype(np.float64)
    vd = _bf16_bits(v).astype(np.uint32).__lshift__(16).view(np.float32).astype(np.float64)
    out = np.zeros((B, H, Nk), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kk = kd[b, h].reshape(Nk, Bk, d)
            vv = vd[b, h].reshape(Nk, Bk, d)
            kc = kk - kk.mean(axis=1, keepdims=True)
            hj = np.einsum('jnc,jne->jce', kc, vv)          # [Nk, d, d]
            dev = hj - hj.mean(axis=0, keepdims=True)
            out[b, h] = np.linalg.norm(dev, ord=2, axis=(1, 2))
    return out


def route_cov(q, k, v, Bq, Bk, topk, lam, threads=0):
    """PISA covariance-aware routing: the top-k of s_ij + lam * M_j, with s_ij
    the plain pooled score (no projections) and M_j from block_cov_norms."""
    bias = lam * block_cov_norms(k, v, Bk) if lam else None
    return route(q, k, None, None, Bq, Bk, topk, threads=threads, bias=bias)


def cocluster(q, k, n_clusters, iters):
    """SVOO online bidirectional Q-K co-clustering ([SVOO] sec. 2.B, "Co-Clustering
    Bidirezionale Online"), in fp64 from the bf16 inputs.  The page gives the two
    alternating steps; the readings taken where it is silent:
      * C = n_clusters co-clusters; the initial query centroids are the means of
        C contiguous chunks of N/C queries (the raster partition);
      * step 1, keys guided by the queries: key n goes to the cluster c whose query
        centroid has the largest affinity qbar_c . k_n (the attention score), ties
        to the lower c; key centroids kbar_c = mean of the keys in cluster c;
      * step 2, queries guided by the keys: query n goes to argmax_c kbar_c . q_n
        (ties to the lower c); query centroids = means of their queries;
      * a cluster left without tokens has no centroid and is no candidate of the
        next assignment;
      * iters repetitions of (step 1, step 2); the tokens are then ordered stably
        by cluster label, so that the block-sparse path's contiguous blocks hold
        tokens of one cluster (a block may straddle two).
    Returns (q_perm, k_perm, q_label, k_label), int64 [B,H,N]: q_perm[b,h,i] is
    the original index of the query at sorted position i."""
    qb, kb = _bf16_bits(q), _bf16_bits(k)
    B, H, N, d = qb.shape
    C = int(n_clusters)
    if C < 1 or N % C:
        raise ValueError("cocluster: n_clusters must divide N")
    to64 = lambda x: (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    qd, kd = to64(qb), to64(kb)
    q_perm = np.zeros((B, H, N), dtype=np.int64)
    k_perm = np.zeros((B, H, N), dtype=np.int64)
    q_lab = np.zeros((B, H, N), dtype=np.int64)
    k_lab = np.zeros((B, H, N), dtype=np.int64)

    def assign(x, cent, valid):
        aff = x @ cent.T                                  # [N, C] affinities
        aff[:, ~valid] = -np.inf
        return np.argmax(aff, axis=1)                     # first maximum: ties to the lower c

    def means(x, lab, prev, prev_valid):
        cnt = np.bincount(lab, minlength=C)
        sums = np.zeros((C, x.shape[1]))
        np.add.at(sums, lab, x)
        valid = cnt > 0
        cent = np.where(valid[:, None], sums / np.maximum(cnt, 1)[:, None], prev)
        return cent, valid

    for b in range(B):
        for h in range(H):
            Q, K = qd[b, h], kd[b, h]
            qc = Q.reshape(C, N // C, d).mean(axis=1)
            qv = np.ones(C, dtype=bool)
            kc, kv = np.zeros((C, d)), np.zeros(C, dtype=bool)
            ql = kl = None
            for _ in range(iters):
                kl = assign(K, qc, qv)
                kc, kv = means(K, kl, kc, kv)
                ql = assign(Q, kc, kv)
                qc, qv = means(Q, ql, qc, qv)
            if iters == 0:
                ql = np.repeat(np.arange(C), N // C)
                kl = ql.copy()
            q_lab[b, h], k_lab[b, h] = ql, kl
            q_perm[b, h] = np.argsort(ql, kind="stable")
            k_perm[b, h] = np.argsort(kl, kind="stable")
    return q_perm, k_perm, q_lab, k_lab


def _rows(rows, B, H, N):
    if rows is None:
        return None, -1
    r = _np(rows, np.int64).reshape(-1)
    return r, r.size


def e4m3(x) -> np.ndarray:
    """E4M3 conversion of float64 values (round to nearest even, saturating)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(a)
    _load().oracle_e4m3_array(_ptr(a), _ptr(out), a.size)
    return out


def int8(x) -> np.ndarray:
    """8-bit integer codes of float64 values (nearest, ties to even, within +-127)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(a)
    _load().oracle_int8_array(_ptr(a), _ptr(out), a.size)
    return out


def quantise(x, int8=False):
    """Codes and per-64-token-block scales of the FP8 (E4M3, top 448) or INT8
    (top 127) sparse branch for one bf16 tensor [N, d]: each code rounds the
    exact quotient top * x / max|x| of its block; scale = max|x| / top (1 for
    an all-zero block).  Returns (codes float64 [N, d], scales float64 [N/64])."""
    xb = _bf16_bits(x)
    N, d = xb.shape
    codes = np.zeros((N, d), dtype=np.float64)
    scales = np.zeros(N // 64, dtype=np.float64)
    _check(_load().oracle_quantise(_ptr(xb), N, d, 1 if int8 else 0, _ptr(codes), _ptr(scales)),
           "quantise")
    return codes, scales


def sla_forward(q, k, v, alpha, lut, Bq, Bk, sm_scale=0.0, rows=None, branches=False,
                threads=0, fp8=False, int8=False, p_plain=False):
    """SLA2 forward on a given LUT.  rows=None: every row, returns [B,H,N,d];
    else flat row indices, returns [len(rows), d].  branches=True also returns
    the sparse-branch and linear-branch outputs.  fp8=True: the sparse branch
    on E4M3-quantised Q, K, P, V with per-64-token-block scales (Bk = 64).
    int8=True: the same with 8-bit integer Q and K codes (P and V E4M3).
    p_plain (fp8 / int8): P is taken against the row maximum itself instead of
    the power of two at or above it before its E4M3 rounding."""
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, H, N, d = qb.shape
    al = _np(alpha, np.float32)
    lt = _np(lut, np.int32)
    topk = lt.shape[-1]
    r, nr = _rows(rows, B, H, N)
    n = B * H * N if r is None else nr
    out = np.zeros((n, d), dtype=np.float64)
    os_ = np.zeros((n, d), dtype=np.float64) if branches else None
    ol_ = np.zeros((n, d), dtype=np.float64) if branches else None
    rc = _load().oracle_sla_forward(B, H, N, d, Bq, Bk, topk, float(sm_scale), _ptr(qb), _ptr(kb),
                                    _ptr(vb), _ptr(al), _ptr(lt), nr, _ptr(r), _ptr(out),
                                    _ptr(os_), _ptr(ol_), 2 if int8 else (1 if fp8 else 0),
                                    1 if p_plain else 0, threads)
    _check(rc, "sla_forward")
    shape = (B, H, N, d) if r is None else (n, d)
    if branches:
        return out.reshape(shape), os_.reshape(shape), ol_.reshape(shape)
    return out.reshape(shape)


def pisa_forward(q, k, v, lut, Bq, Bk, sm_scale=0.0, rows=None, threads=0, first_order=False):
    """PISA exact-or-approximate forward on a given LUT: zero-order terms for the
    unselected blocks, plus (first_order=True) the global first-order term."""
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, H, N, d = qb.shape
    lt = _np(lut, np.int32)
    topk = lt.shape[-1]
    r, nr = _rows(rows, B, H, N)
    n = B * H * N if r is None else nr
    out = np.zeros((n, d), dtype=np.float64)
    rc = _load().oracle_pisa_forward(B, H, N, d, Bq, Bk, topk, float(sm_scale), _ptr(qb),
                                     _ptr(kb), _ptr(vb), _ptr(lt), nr, _ptr(r), _ptr(out),
                                     1 if first_order else 0, threads)
    _check(rc, "pisa_forward")
    return out.reshape((B, H, N, d) if r is None else (n, d))

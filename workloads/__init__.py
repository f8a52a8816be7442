"""Seeded synthetic inputs for hybrid sparse-linear attention.

This module holds the workload definitions (shapes, block sizes, keep counts)
and the deterministic input generators that both the CUDA path and the CPU
oracle read.  It contains none of the method's arithmetic: no pooling, no
scoring, no softmax, no feature map.  It only draws random numbers.

Two generators:

* ``gaussian``: Q, K, V ~ N(0, 1), alpha ~ U(lo, hi) per (head, token),
  W_q, W_k ~ N(0, 1/d).  Used for the tiny workload and for randomised test
  shapes.
* ``video``: a stand-in for video-DiT activations (Wan2.1 / HunyuanVideo
  latents are not available).  Tokens are raster-ordered over a (T, Y, X)
  latent grid, pad tokens last.  Per head, 16 frequencies
  w_f ~ N(0, diag(0.35^2, 0.25^2, 0.25^2)) rad/step give features
  Phi(p) = [cos(w_f . p), sin(w_f . p)] in R^32 (zero for pad tokens);
  A_h in R^{d x 32} is Gaussian, orthonormalised by QR;
  q = g A_h Phi(p) + eps, k = g A_h Phi(p) + eps', g^2 = sqrt(d)/2, so that the
  positional part of the softmax-scaled logit is 1/2 sum_f cos(w_f . dp), in
  [-8, 8].  eps, eps' ~ N(0, 0.25) (variance 0.25), V ~ N(0, 1).

All draws use torch's CPU generator in fp32 and are rounded to bf16 once
(round-to-nearest-even); the consumers read those bf16 values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

SPARSE_BF16 = 0
SPARSE_FP8_E4M3 = 1
SPARSE_INT8 = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    Bq: int
    Bk: int
    topk: int
    mode: str                 # "sla" or "pisa"
    sparse_dtype: int         # SPARSE_BF16, SPARSE_FP8_E4M3 or SPARSE_INT8
    generator: str            # "gaussian" or "video"
    seed: int
    grid: Optional[tuple] = None   # (T, Y, X) latent grid for the video generator
    alpha_range: Optional[tuple] = (0.0, 1.0)
    use_w: bool = True
    first_order: bool = False     # PISA: add the global first-order term
    cov_lambda: float = 0.0       # PISA: weight of the covariance-aware selection term
    clusters: int = 0             # SVOO co-clustering: co-clusters (0 = raster order)
    cluster_iters: int = 0        # SVOO co-clustering: alternating iterations
    cluster_every: int = 0        # SVOO co-clustering: recomputed every this many steps

    @property
    def Nq(self) -> int:
        return self.N // self.Bq

    @property
    def Nk(self) -> int:
        return self.N // self.Bk

    def dense_equiv_flops(self) -> float:
        """4*B*H*N^2*d: two N x N x d contractions of full attention."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d

    def executed_sparse_flops(self) -> float:
        """4*Bq*Bk*d per (query block, selected KV block) pair."""
        pairs = self.B * self.H * self.Nq * self.topk
        return 4.0 * pairs * self.Bq * self.Bk * self.d


# The workloads: tiny, SLA2 bf16 (21x30x52 grid + 8 pad tokens), long (21x45x80
# grid + 176 pad tokens), the FP8 and INT8 sparse branches (the inputs of the FP8
# one), PISA and PISA with the first-order term (the inputs of the PISA one).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 1024, 64, 64, 64, 4, "sla", SPARSE_BF16,
                     "gaussian", 1001, None, (0.2, 0.8), True),
    "sla2_bf16": Workload("sla2_bf16", 1, 12, 32768, 128, 128, 64, 52, "sla",
                          SPARSE_BF16, "video", 1002, (21, 30, 52), (0.0, 1.0), True),
    "sla2_long": Workload("sla2_long", 1, 40, 75776, 128, 128, 64, 59, "sla",
                          SPARSE_BF16, "video", 1003, (21, 45, 80), (0.0, 1.0), True),
    "sla2_fp8": Workload("sla2_fp8", 1, 12, 32768, 128, 128, 64, 52, "sla",
                         SPARSE_FP8_E4M3, "video", 1004, (21, 30, 52), (0.0, 1.0), True),
    "sla2_int8": Workload("sla2_int8", 1, 12, 32768, 128, 128, 64, 52, "sla",
                          SPARSE_INT8, "video", 1004, (21, 30, 52), (0.0, 1.0), True),
    "pisa": Workload("pisa", 1, 24, 32768, 128, 64, 64, 77, "pisa", SPARSE_BF16,
                     "video", 1005, (21, 30, 52), None, False),
    # the PISA workload with the global first-order correction
    "pisa_fo": Workload("pisa_fo", 1, 24, 32768, 128, 64, 64, 77, "pisa", SPARSE_BF16,
                        "video", 1005, (21, 30, 52), None, False, True),
    # the PISA workload with the covariance-aware selection (lambda = 0.1 moves
    # about 28% of the selected blocks on these inputs)
    "pisa_cov": Workload("pisa_cov", 1, 24, 32768, 128, 64, 64, 77, "pisa", SPARSE_BF16,
                         "video", 1005, (21, 30, 52), None, False, False, 0.1),
    # the SLA2 bf16 workload in the order of SVOO's online bidirectional co-clustering
    # (64 co-clusters, 3 iterations, recomputed every 20 steps)
    "sla2_svoo": Workload("sla2_svoo", 1, 12, 32768, 128, 128, 64, 52, "sla", SPARSE_BF16,
                          "video", 1002, (21, 30, 52), (0.0, 1.0), True, clusters=64, cluster_iters=3,
                          cluster_every=20),
}
ORDER = ["tiny", "sla2_bf16", "sla2_long", "sla2_fp8", "sla2_int8", "pisa", "pisa_fo", "pisa_cov",
         "sla2_svoo"]


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def gaussian_inputs(B, H, N, d, seed, alpha_range=(0.2, 0.8), use_w=True,
                    with_alpha=True):
    """Q, K, V ~ N(0,1) bf16 [B,H,N,d]; alpha ~ U(lo,hi) fp32 [B,H,N];
    W_q, W_k ~ N(0, 1/d) fp32 [d,d] (or None)."""
    g = torch.Generator().manual_seed(seed)
    q = _bf16(torch.randn(B, H, N, d, generator=g))
    k = _bf16(torch.randn(B, H, N, d, generator=g))
    v = _bf16(torch.randn(B, H, N, d, generator=g))
    alpha = None
    if with_alpha:
        lo, hi = alpha_range
        alpha = lo + (hi - lo) * torch.rand(B, H, N, generator=g)
    wq = wk = None
    if use_w:
        wq = torch.randn(d, d, generator=g) / math.sqrt(d)
        wk = torch.randn(d, d, generator=g) / math.sqrt(d)
    return dict(q=q, k=k, v=v, alpha=alpha, w_q=wq, w_k=wk)


def video_inputs(B, H, N, d, grid, seed, alpha_range=(0.0, 1.0), use_w=True,
                 with_alpha=True):
    """The raster-ordered latent-grid generator described in the module doc."""
    T, Y, X = grid
    n_real = T * Y * X
    assert n_real <= N, "grid larger than the token count"
    g = torch.Generator().manual_seed(seed)
    tt, yy, xx = torch.meshgrid(torch.arange(T), torch.arange(Y), torch.arange(X),
                                indexing="ij")
    pos = torch.stack([tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)], 1).float()
    gain = math.sqrt(math.sqrt(d) / 2.0)
    sig = torch.tensor([0.35, 0.25, 0.25])
    q = torch.empty(B, H, N, d, dtype=torch.bfloat16)
    k = torch.empty(B, H, N, d, dtype=torch.bfloat16)
    v = torch.empty(B, H, N, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            omega = torch.randn(16, 3, generator=g) * sig          # rad / step
            a = torch.randn(d, 32, generator=g)
            a, _ = torch.linalg.qr(a)                              # d x 32, orthonormal cols
            ang = pos @ omega.t()                                  # [n_real, 16]
            feat = torch.zeros(N, 32)
            feat[:n_real] = torch.cat([torch.cos(ang), torch.sin(ang)], 1)
            sig_part = gain * (feat @ a.t())                       # [N, d]
            eq = 0.5 * torch.randn(N, d, generator=g)
            ek = 0.5 * torch.randn(N, d, generator=g)
            q[b, h] = _bf16(sig_part + eq)
            k[b, h] = _bf16(sig_part + ek)
            v[b, h] = _bf16(torch.randn(N, d, generator=g))
    alpha = None
    if with_alpha:
        lo, hi = alpha_range
        alpha = lo + (hi - lo) * torch.rand(B, H, N, generator=g)
    wq = wk = None
    if use_w:
        wq = torch.randn(d, d, generator=g) / math.sqrt(d)
        wk = torch.randn(d, d, generator=g) / math.sqrt(d)
    return dict(q=q, k=k, v=v, alpha=alpha, w_q=wq, w_k=wk)


def make_inputs(w: Workload):
    """Inputs of a named workload (CPU tensors)."""
    with_alpha = w.mode == "sla"
    if w.generator == "gaussian":
        return gaussian_inputs(w.B, w.H, w.N, w.d, w.seed, w.alpha_range or (0, 1),
                               w.use_w, with_alpha)
    return video_inputs(w.B, w.H, w.N, w.d, w.grid, w.seed, w.alpha_range or (0, 1),
                        w.use_w, with_alpha)


def sample_rows(B, H, N, count, seed, heads=None):
    """Seeded flat row indices ((b*H + h)*N + t), sorted, unique.  ``heads``
    restricts the draw to a subset of (b*H + h) head indices."""
    g = torch.Generator().manual_seed(seed)
    if heads is None:
        heads = list(range(B * H))
    heads = torch.tensor(heads, dtype=torch.int64)
    hsel = heads[torch.randint(0, len(heads), (count,), generator=g)]
    t = torch.randint(0, N, (count,), generator=g)
    rows = torch.unique(hsel * N + t)
    return rows

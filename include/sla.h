/*
 * sla.h -- C ABI of the B200 (sm_100a) hybrid sparse-linear attention library.
 *
 * Forward pass of hybrid sparse-linear attention for video diffusion
 * transformers, as described by
 *   [SLA2]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
 *           (gist.science summary of arXiv 2602.12675, Italian and Arabic pages)
 *   [SALAD] "SALAD: Achieve High-Sparsity Attention via Efficient Linear
 *           Attention Tuning for Video Diffusion Transformer" (2601.16515)
 *   [PISA]  "PISA - Piecewise Sparse Attention per Efficient Diffusion
 *           Transformers" (2602.01077)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are dense, row-major, d innermost:
 *      q, k, v      : bf16  [B, H, N, d]            (device memory)
 *      out          : bf16 or fp32 [B, H, N, d]     (device memory, see out_dtype)
 *      alpha        : fp32  [B, H, N]               (device memory)
 *      w_q, w_k     : fp32  [d, d], x . W, shared by all heads; NULL = identity
 *      lut          : int32 [B, H, N/Bq, topk]      (device memory)
 *  - Every pointer is a DEVICE pointer owned by the caller; q, k, v, out are
 *    aligned to 16 bytes, alpha, w_q, w_k, lut to 4 bytes.  lut may be NULL
 *    when topk == 0.  The library allocates no device memory: scratch is the caller's
 *    `workspace`, of at least sla_workspace_size() bytes, 256-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Arguments are validated on the host before anything is
 *    enqueued; on any error nothing is launched.  sla_forward and
 *    sla_pisa_forward run their K/V pre-pass on a side stream owned by the
 *    library (one per device, created with three events on first use; no device
 *    memory), forked from and joined back into `stream` with events, so work
 *    the caller enqueues on `stream` afterwards sees every result, and a
 *    capture of `stream` includes that work.
 *  - Errors are returned, never thrown.  Kernel-side checks (an out-of-range
 *    or repeated entry in a caller-given LUT, a bounded wait that ran out)
 *    set a device status word that sla_check_device_status() reads.
 *  - Numerics: products on the tensor cores with fp32 accumulation; the
 *    softmax weights P and the values V enter the P.V product as fp16 (V is
 *    converted once per call; |v| and |k| must stay below 65504, else the
 *    kernels flag SLA_ERR_DEVICE_CHECK); the router runs in fp64.
 *  - Supported shapes: d in {64, 128}; Bq in {64, 128}; Bk = 64;
 *    N % Bq == 0 and N % Bk == 0 (padding tokens are the caller's job);
 *    0 <= topk <= N/Bk; N/Bk <= 8192; B*H <= 65535.
 *    The FP8 sparse branch needs d = 128 and Bq = 128.
 *    PISA needs Bq == Bk.
 */
#ifndef SLA_B200_H
#define SLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *sla_stream_t; /* a cudaStream_t */

typedef enum {
    SLA_OK = 0,
    SLA_ERR_INVALID_ARG = 1,   /* NULL/misaligned pointer, inconsistent sizes */
    SLA_ERR_UNSUPPORTED = 2,   /* valid, but outside the shapes listed above  */
    SLA_ERR_WORKSPACE = 3,     /* workspace NULL, misaligned or too small     */
    SLA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    SLA_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out             */
    SLA_ERR_DEVICE_CHECK = 6   /* a kernel found invalid data (e.g. LUT entry)*/
} sla_status_t;

typedef enum { SLA_SPARSE_BF16 = 0, SLA_SPARSE_FP8_E4M3 = 1, SLA_SPARSE_INT8 = 2 } sla_sparse_dtype_t;
typedef enum { SLA_LUT_COMPUTE = 0, SLA_LUT_GIVEN = 1 } sla_lut_mode_t;
typedef enum { SLA_OUT_BF16 = 0, SLA_OUT_FP32 = 1 } sla_out_dtype_t;

typedef struct sla_params {
    int32_t B, H, N, d;      /* batch, heads, tokens, head dim                  */
    int32_t Bq, Bk;          /* query / key-value block sizes (tokens)          */
    int32_t topk;            /* KV blocks kept per query block                  */
    float sm_scale;          /* softmax scale tau; <= 0 means 1/sqrt(d)         */
    int32_t sparse_dtype;    /* sla_sparse_dtype_t: operand type of the sparse
                                branch's tensor-core products                   */
    int32_t lut_mode;        /* sla_lut_mode_t                                  */
    int32_t out_dtype;       /* sla_out_dtype_t: element type of `out`          */
    int32_t pisa_first_order;/* sla_pisa_forward: 1 adds the global first-order
                                correction term, 0 keeps the zero-order terms  */
    float pisa_cov_lambda;   /* sla_pisa_forward, LUT_COMPUTE: weight lambda >= 0
                                of the covariance term of the block selection
                                (0 = plain routing); must be 0 in sla_forward */
} sla_params_t;

/* Bytes of device workspace that sla_route, sla_forward, sla_pisa_forward and
 * sla_pisa_cov_norms need for these parameters (the maximum over them; the
 * covariance-aware selection's scratch is included when pisa_cov_lambda > 0).
 * It never decreases as B*H grows with the other fields fixed, so a workspace
 * for B*H heads serves a call over any subset of them.  Returns 0 if the
 * parameters are invalid. */
size_t sla_workspace_size(const sla_params_t *p);

/*
 * sla_route -- the learnable router of [SLA2] sec. 2.B ("Router
 * Apprendibile"; Arabic page sec. 2.b) at inference:
 *   1. mean-pool Q over blocks of Bq adjacent tokens and K over blocks of Bk;
 *   2. project: Qt = Qbar . w_q, Kt = Kbar . w_k (NULL = no projection);
 *   3. compressed block score s_ij = Qt_i . Kt_j (V is not used);
 *   4. hard top-k per query block i: the topk largest s_ij, ties broken
 *      toward the lower j, written to lut[b,h,i,:] in ascending j.
 * Pooling, projection and score are computed in fp64, so the LUT matches an
 * exact-arithmetic selection except where two scores lie within ~1e-12.
 * Ignores p->lut_mode, p->sm_scale, p->sparse_dtype, p->out_dtype and
 * p->pisa_first_order.  p->pisa_cov_lambda must be 0 (SLA_ERR_INVALID_ARG
 * otherwise): the covariance-aware selection is an option of sla_pisa_forward,
 * and this call does not apply it.
 */
sla_status_t sla_route(const sla_params_t *p, const void *q, const void *k,
                       const float *w_q, const float *w_k, int32_t *lut,
                       void *workspace, size_t ws_bytes, sla_stream_t stream);

/*
 * sla_route_noalloc -- the same routing as sla_route, for callers that cannot
 * allocate device memory: for example a plugin running under a host engine that
 * owns the whole device-memory budget and gives plugins no allocator, or a
 * serving loop that must never enter an allocator once it is running.  (The
 * papers have no counterpart; this is an interface convenience.)
 * It takes no workspace: its scratch is a 32 MiB array built into the library,
 * which every GPU that loads the library keeps reserved until the process
 * exits.  Calls whose scratch (8 * B*H * (N/Bq + N/Bk) * d + 8 * d*d bytes,
 * each part rounded up to 256) exceeds 32 MiB return SLA_ERR_WORKSPACE.
 * Every call made outside stream capture looks up the array's device address
 * for the current device (cudaGetSymbolAddress); a call made while `stream`
 * is capturing reuses the address of the last uncaptured call on that device,
 * so make one uncaptured call on a device before capturing one (otherwise
 * SLA_ERR_CUDA).  Parameters are read as in sla_route (same ignored fields,
 * same rule for pisa_cov_lambda).  All calls share the one array and nothing
 * in it needs clearing between calls (every region is fully written before it
 * is read), but calls that overlap on the GPU (on different streams, or on one
 * device from several threads) race on it.
 * It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
sla_status_t sla_route_noalloc(const sla_params_t *p, const void *q, const void *k,
                               const float *w_q, const float *w_k, int32_t *lut,
                               sla_stream_t stream);

/*
 * sla_forward -- SLA2 hybrid forward ([SLA2] sec. 2.A):
 *   O = alpha (.) O_s + (1 - alpha) (.) O_l
 * O_s: softmax attention of each query over the tokens of its query block's
 *      selected KV blocks only, renormalised over them (0 if topk == 0);
 * O_l: ReLU-feature linear attention ([SALAD] sec. 2, phi = ReLU) over the
 *      tokens of the blocks NOT selected:
 *      phi(q) (sum_{j not in S} h_j) / (phi(q) . sum_{j not in S} z_j),
 *      h_j = phi(K_j)^T V_j, z_j = phi(K_j)^T 1; 0 if the denominator <= 0.
 * lut: LUT_COMPUTE -> routing as in sla_route (w_q, w_k used) and the LUT is
 *      written to `lut` (which may be NULL); LUT_GIVEN -> `lut` is read and
 *      must hold topk distinct entries in [0, N/Bk) per row (any order);
 *      invalid entries are skipped and flagged SLA_ERR_DEVICE_CHECK.
 * sparse_dtype FP8_E4M3 (needs d = 128, Bq = 128): the sparse branch runs on
 *      e4m3 Q, K, P and V ([SLA2] sec. 2.C; Arabic page sec. 2.j: the forward
 *      quantises Q, K, P and V).  Q, K, V: one scale per 64-token block,
 *      s = absmax / 448 (1 for an all-zero block); each code is the e4m3
 *      rounding (to nearest even, saturating) of the exact quotient
 *      448 x / absmax, which the kernels decide exactly in fp32.
 *      Logits use the e4m3 Q.K product times s_q s_k.  P is taken against the
 *      power of two at or above the running row maximum and quantised per
 *      64-key tile as e4m3(P * 448 s_v,j / s_v,max), s_v,max the largest V
 *      scale of the query block's LUT row; O is dequantised by s_v,max / 448
 *      and divided by the row sum of the unquantised P.  The linear branch
 *      and the combine stay bf16/fp32.
 * sparse_dtype INT8 (needs d = 128, Bq = 128): as FP8_E4M3, except that Q and
 *      K take symmetric 8-bit integer codes (s = absmax / 127, code = the
 *      nearest integer to the exact quotient 127 x / absmax, ties to even), so
 *      S = Q8 K8^T is an exact integer product (tcgen05 kind::i8, s32
 *      accumulation) scaled by s_q s_k; P and V keep the e4m3 rules (an
 *      integer P.V accumulator could not take the online rescale exactly).
 */
sla_status_t sla_forward(const sla_params_t *p, const void *q, const void *k, const void *v,
                         const float *alpha, const float *w_q, const float *w_k,
                         int32_t *lut, void *out,
                         void *workspace, size_t ws_bytes, sla_stream_t stream);

/*
 * sla_pisa_forward -- PISA exact-or-approximate attention ([PISA] sec. 2,
 * "Algoritmo Core"), zero-order mode:
 *   o_t = N_t / D_t,
 *   N_t = sum_{j in S} sum_n e^{tau q.k_jn - m} v_jn + sum_{j not in S} e^{tau q.kbar_j - m} sum_n v_jn
 *   D_t = sum_{j in S} sum_n e^{tau q.k_jn - m}      + sum_{j not in S} Bk e^{tau q.kbar_j - m}
 * with kbar_j the mean key (centroid) of block j; both sums share one
 * online-softmax maximum m.  p->pisa_first_order = 1 adds the global
 * first-order correction to N_t ([PISA] sec. 2, the third numerator term):
 *   + tau (q_t Hbar) sum_{j not in S} e^{tau q.kbar_j - m},
 *   Hbar = (1/Nk) sum_j sum_{n in j} (k_n - kbar_j)^T v_n,
 * the mean over all blocks of the blocks' first-order matrices (D_t has no
 * first-order part).  S comes from the router (LUT_COMPUTE; pass
 * w_q = w_k = NULL for PISA's plain pooled score) or from `lut` (LUT_GIVEN).
 * With LUT_COMPUTE and p->pisa_cov_lambda > 0 the selection is covariance
 * aware ([PISA] sec. 2, "Routing Consapevole della Covarianza"): the top-k of
 *   s_ij + lambda M_j,   M_j = || H_j - Hbar ||_2  (largest singular value),
 *   H_j = sum_{n in j} (k_n - kbar_j)^T v_n,
 * so heterogeneous blocks go to the exact path (M_j: see sla_pisa_cov_norms).
 * Requires Bq == Bk and sparse_dtype = BF16.
 */
sla_status_t sla_pisa_forward(const sla_params_t *p, const void *q, const void *k,
                              const void *v, const float *w_q, const float *w_k,
                              int32_t *lut, void *out,
                              void *workspace, size_t ws_bytes, sla_stream_t stream);

/*
 * sla_forward_host / sla_pisa_forward_host -- sla_forward and sla_pisa_forward
 * with the inputs and the output in host memory.  The (batch, head) problems of
 * a call are independent ([SLA2] sec. 2, [PISA] sec. 2: attention, routing and
 * every statistic are per head), so the call works through chunks of
 * heads_per_chunk consecutive heads (0: about an eighth of B*H): each chunk's
 * Q, K, V (and alpha) are copied to the caller's device buffers on a library
 * stream, its forward runs on `stream` as soon as they have landed, and its
 * output is copied back on a second library stream while later chunks arrive
 * and compute.  The result is that of one sla_forward (sla_pisa_forward) call
 * on the whole problem up to summation order: the LUT is identical, and the
 * linear branch's per-head sums are split over a number of partial sums that
 * depends on the heads in a chunk.
 *   q_h, k_h, v_h: host bf16 [B,H,N,d]; alpha_h: host fp32 [B,H,N] (sla_forward_host
 *   only); out_h: host [B,H,N,d] in the type p->out_dtype selects.  Page-locked
 *   (pinned) host memory lets the copies overlap; pageable memory is correct but
 *   serialises them.
 *   q, k, v, alpha, out: the caller's device buffers of those shapes (16-byte
 *   aligned; alpha 4-byte), overwritten by the call.
 *   w_q, w_k, lut, workspace, ws_bytes: as for sla_forward / sla_pisa_forward (the
 *   workspace sized for the whole problem serves every chunk; lut, if given,
 *   is the whole problem's).
 * Asynchronous on stream: it starts after the work queued on stream before it,
 * and work queued on stream after it waits for its last copy.  The arguments
 * are checked as sla_forward (sla_pisa_forward) checks them, for the whole
 * problem, before anything is enqueued; a NULL host buffer or heads_per_chunk < 0
 * is SLA_ERR_INVALID_ARG.  A CUDA error in a later chunk leaves the earlier
 * chunks' work queued.
 */
sla_status_t sla_forward_host(const sla_params_t *p, const void *q_h, const void *k_h,
                              const void *v_h, const float *alpha_h, void *out_h, void *q,
                              void *k, void *v, float *alpha, void *out, const float *w_q,
                              const float *w_k, int32_t *lut, int32_t heads_per_chunk,
                              void *workspace, size_t ws_bytes, sla_stream_t stream);
sla_status_t sla_pisa_forward_host(const sla_params_t *p, const void *q_h, const void *k_h,
                                   const void *v_h, void *out_h, void *q, void *k, void *v,
                                   void *out, const float *w_q, const float *w_k, int32_t *lut,
                                   int32_t heads_per_chunk, void *workspace, size_t ws_bytes,
                                   sla_stream_t stream);

/*
 * sla_pisa_cov_norms -- the block covariance norms of the covariance-aware
 * selection: norms[(b*H + h)*Nk + j] = M_j = || H_j - Hbar ||_2 in fp64
 * (unscaled), j < Nk = N/Bk.  H_j and Hbar are fp32 tensor-core sums of exact
 * products (keys centred in fp64, rounded once to fp32 and split exactly into
 * three bf16 parts); the largest singular value comes from 24 Lanczos steps on
 * (H_j - Hbar)^T (H_j - Hbar) (relative error a few 1e-7).
 * k, v: device bf16 [B,H,N,d]; norms: device fp64, B*H*Nk entries, 8-byte
 * aligned, owned by the caller.  Requires Bk = 64 and p->pisa_cov_lambda > 0
 * (the workspace then holds the norms' scratch); errors as sla_pisa_forward.
 */
sla_status_t sla_pisa_cov_norms(const sla_params_t *p, const void *k, const void *v,
                                double *norms, void *workspace, size_t ws_bytes,
                                sla_stream_t stream);

/*
 * sla_cocluster -- online bidirectional Q-K co-clustering of "Training-Free
 * Sparse Attention for Fast Video Generation via Offline Layer-Wise Sparsity
 * Profiling and Online Bidirectional Co-Clustering" (SVOO), sec. 2.B.  Per head,
 * with C = n_clusters co-clusters:
 *   query centroids start as the means of C contiguous chunks of N/C queries;
 *   then iters times: each key joins the cluster whose query centroid has the
 *   largest dot product with it (ties to the lower cluster), key centroids
 *   become the means of their keys; each query joins the cluster of the largest
 *   dot product with the key centroids, query centroids become the means of
 *   their queries.  A cluster left without tokens is no candidate of the next
 *   assignment.  All in fp64 from the bf16 inputs.
 * Outputs the stable order of the tokens by their final cluster:
 *   q_perm[b,h,i] = the original index of the query at position i, k_perm the
 *   same for keys (int32 [B,H,N], device memory owned by the caller).
 * Running the block-sparse path on Q, alpha gathered by q_perm and K, V gathered
 * by k_perm (sla_permute_rows) puts tokens of one cluster into the same blocks;
 * the output rows go back with the inverse permutation.  The page recomputes
 * the clusters only every few diffusion steps (e.g. 20) and reuses them.
 * q, k: bf16 [B,H,N,d], 16-byte aligned.  Needs 1 <= n_clusters <= 1024 dividing
 * N, 1 <= iters <= 64, and a workspace of sla_cocluster_workspace_size() bytes
 * (256-byte aligned); other parameters as sla_route (p->Bq, p->Bk, p->topk must
 * be valid; they are not used).  Errors as sla_route.
 */
size_t sla_cocluster_workspace_size(const sla_params_t *p, int32_t n_clusters);
sla_status_t sla_cocluster(const sla_params_t *p, const void *q, const void *k,
                           int32_t n_clusters, int32_t iters, int32_t *q_perm, int32_t *k_perm,
                           void *workspace, size_t ws_bytes, sla_stream_t stream);

/*
 * sla_permute_rows -- reorders the rows of a [BH, N, row] tensor by a per-head
 * permutation perm (int32 [BH, N]): inverse = 0 gathers,
 *   dst[bh, i, :] = src[bh, perm[bh, i], :],
 * inverse = 1 scatters back, dst[bh, perm[bh, i], :] = src[bh, i, :].
 * row_bytes: a multiple of 4, at most 4096 (16-byte aligned pointers and a
 * multiple of 16 take 16-byte copies); src and dst must not overlap.  A perm
 * entry outside [0, N) is skipped and flagged SLA_ERR_DEVICE_CHECK.
 */
sla_status_t sla_permute_rows(const void *src, const int32_t *perm, void *dst, int64_t BH,
                              int32_t N, int32_t row_bytes, int32_t inverse, sla_stream_t stream);

/* Static text for a status code. */
const char *sla_status_string(sla_status_t s);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: SLA_OK, SLA_ERR_TIMEOUT or SLA_ERR_DEVICE_CHECK (or
 * SLA_ERR_CUDA if the synchronisation itself failed). */
sla_status_t sla_check_device_status(sla_stream_t stream);

/*
 * Kernel tracing.  While enabled, every kernel the library launches is
 * bracketed by a pair of CUDA events recorded on its own stream (no device
 * cost; about a microsecond of host time per launch), and each forward call
 * records one more pair on the caller's stream, from its entry to the start
 * of its attention kernel (SLA_PHASE_PRE_ATTN).  sla_profile_read()
 * synchronises those events and returns, per kernel kind, the summed device
 * time in milliseconds and the number of launches since the last read; it
 * then forgets them.  Host-side state only; guarded by a mutex.
 */
typedef enum {
    SLA_KERNEL_POOL = 0,        /* mean pooling of Q (and K in sla_route)      */
    SLA_KERNEL_KV_STATS = 1,    /* K/V pre-pass                                 */
    SLA_KERNEL_H_REDUCE = 2,    /* reduction of the per-chunk H partials       */
    SLA_KERNEL_FOLD_W = 3,      /* W_q W_k^T                                    */
    SLA_KERNEL_SCORE_TOPK = 4,  /* fp64 block score + top-k                     */
    SLA_KERNEL_ATTN = 5,        /* sparse / PISA attention + fused epilogue     */
    SLA_KERNEL_QUANT_Q = 6,     /* 8-bit quantisation of Q (FP8, INT8 branch)   */
    SLA_KERNEL_PROJECT = 7,     /* pooled Q times W_q W_k^T (router with W)      */
    SLA_KERNEL_COV = 8,         /* block covariance norms (PISA selection)       */
    SLA_PHASE_PRE_ATTN = 9,     /* not a kernel: from the entry of a forward call
                                   on its stream to the start of its attention
                                   kernel (router, pre-pass and their joins)     */
    SLA_KERNEL_COCLUSTER = 10,  /* the co-clustering kernels of one call          */
    SLA_KERNEL_PERMUTE = 11,    /* row permutation (co-clustered order)           */
    SLA_KERNEL_KINDS = 12
} sla_kernel_kind_t;

sla_status_t sla_profile_enable(int32_t on);
/* ms_total and launches: arrays of SLA_KERNEL_KINDS entries (either may be NULL). */
sla_status_t sla_profile_read(double *ms_total, int64_t *launches);

/* Library version, major*10000 + minor*100 + patch. */
int32_t sla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SLA_B200_H */

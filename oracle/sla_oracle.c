/*
 * sla_oracle.c -- CPU oracle for hybrid sparse-linear attention (forward).
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously-correct
 * double-precision restatement of what the method computes.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header or constant with the CUDA library.
 *
 * Sources (web summaries of the papers):
 *   [SLA2-it]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT",
 *              gist.science/it/paper/2602.12675
 *   [SLA2-ar]  the same paper, gist.science/ar/paper/2602.12675
 *   [SALAD]    "SALAD: Achieve High-Sparsity Attention via Efficient Linear
 *              Attention Tuning for Video Diffusion Transformer",
 *              gist.science/it/paper/2601.16515
 *   [PISA]     "PISA - Piecewise Sparse Attention per Efficient Diffusion
 *              Transformers", gist.science/it/paper/2602.01077
 *
 * Inputs are the same buffers the GPU path reads: bf16 Q, K, V as raw 16-bit
 * patterns in [B,H,N,d] (d innermost), fp32 alpha [B,H,N], fp32 W [d,d]
 * row-major (x . W), int32 LUT [B,H,N/Bq,topk].  Every value is converted
 * exactly to double; all arithmetic is double.
 *
 * Parity status: every function here is pinned by the CPU test-suite
 * (dense-attention and pairwise linear-attention special cases, brute-force
 * routing on tiny inputs, block-constant-key exactness of the zero-order
 * term, and its first-order error decay; the E4M3 codec against an
 * enumeration of the format and a library conversion; the FP8 sparse
 * branch against the exact forward on inputs whose every quantisation step
 * is exact, and against the size of error the format implies elsewhere).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ENOMEM (-2)

static double bf(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double relu(double x) { return x > 0.0 ? x : 0.0; }

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int check_shape(int B, int H, int N, int d, int Bq, int Bk, int topk)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || Bq <= 0 || Bk <= 0) return 0;
    if (d > 512) return 0; /* per-row scratch below is sized for d <= 512 */
    if (N % Bq || N % Bk) return 0;
    if (topk < 0 || topk > N / Bk) return 0;
    return 1;
}

/* ------------------------------------------------------------------ */
/* 8-bit floating point, E4M3 variant (the OCP 8-bit floating-point
 * specification): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities.  Normal values (1 + m/8) 2^(e-7) for e = 1..15, except
 * e = 15, m = 7, which is NaN: the largest finite magnitude is 448.
 * Subnormal values (m/8) 2^-6.  Conversion rounds to nearest, ties to even,
 * and saturates magnitudes beyond 448 to 448. */
double oracle_e4m3(double x)
{
    if (x != x) return x;
    const double a = fabs(x);
    if (a >= 448.0) return copysign(448.0, x);
    if (a == 0.0) return x;
    int e2;
    frexp(a, &e2);                 /* a in [2^(e2-1), 2^e2) */
    int lead = e2 - 1;
    if (lead < -6) lead = -6;      /* subnormals share the spacing 2^-9 */
    const double spacing = ldexp(1.0, lead - 3);
    return copysign(nearbyint(a / spacing) * spacing, x);
}

void oracle_e4m3_array(const double *in, double *out, int64_t n)
{
    for (int64_t a = 0; a < n; ++a) out[a] = oracle_e4m3(in[a]);
}

/* Symmetric 8-bit integer code: the nearest integer (ties to even), clamped to
 * [-127, 127]. */
double oracle_int8(double x)
{
    if (x != x) return 0.0;
    double r = nearbyint(x);
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return r;
}

void oracle_int8_array(const double *in, double *out, int64_t n)
{
    for (int64_t a = 0; a < n; ++a) out[a] = oracle_int8(in[a]);
}

/* A LUT row must hold topk distinct block indices in [0, Nk). */
static int lut_row_valid(const int32_t *row, int topk, int Nk)
{
    for (int a = 0; a < topk; ++a) {
        if (row[a] < 0 || row[a] >= Nk) return 0;
        for (int b = 0; b < a; ++b)
            if (row[b] == row[a]) return 0;
    }
    return 1;
}

/* ------------------------------------------------------------------ */
/* Router: [SLA2-it] sec. 2.B "Router Apprendibile", [SLA2-ar] sec. 2.b.
 *   1. mean-pool Q over blocks of Bq adjacent tokens and K over blocks of Bk
 *      ("pooling medio su blocchi di token adiacenti");
 *   2. project the pooled matrices with proj_q, proj_k (x . W; NULL = none);
 *   3. compressed score s_ij = Qt_i . Kt_j (V is not used);
 *   4. hard top-k per query block: the k largest s_ij, ties to the lower j,
 *      written in ascending block order.
 * bias ([B*H][Nk], NULL = none) is added to every query block's score of KV
 * block j before the top-k: PISA's covariance-aware selection ([PISA] sec. 2,
 * "Routing Consapevole della Covarianza") ranks blocks by s_ij + lambda M_j.
 * gap_i = s_(k) - s_(k+1) in descending order (INFINITY when k is 0 or Nk). */

typedef struct { double s; int j; } scored_t;

static int by_score_desc(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_int_asc(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

static void mean_pool(const uint16_t *x, int nblk, int blk, int d, double *out)
{
    for (int i = 0; i < nblk; ++i) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int r = 0; r < blk; ++r) acc += bf(x[((size_t)i * blk + r) * d + c]);
            out[(size_t)i * d + c] = acc / (double)blk;
        }
    }
}

static void project(const double *x, int rows, int d, const float *w, double *out)
{
    for (int i = 0; i < rows; ++i) {
        for (int e = 0; e < d; ++e) {
            if (!w) { out[(size_t)i * d + e] = x[(size_t)i * d + e]; continue; }
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += x[(size_t)i * d + c] * (double)w[(size_t)c * d + e];
            out[(size_t)i * d + e] = acc;
        }
    }
}

int oracle_route(int B, int H, int N, int d, int Bq, int Bk, int topk,
                 const uint16_t *q, const uint16_t *k, const float *w_q, const float *w_k,
                 const double *bias, int32_t *lut, double *gap, int nthreads)
{
    if (!check_shape(B, H, N, d, Bq, Bk, topk) || !q || !k || !lut) return ORC_EINVAL;
    set_threads(nthreads);
    const int Nq = N / Bq, Nk = N / Bk;
    int err = ORC_OK;
    for (int bh = 0; bh < B * H; ++bh) {
        const uint16_t *qh = q + (size_t)bh * N * d;
        const uint16_t *kh = k + (size_t)bh * N * d;
        double *qbar = malloc(sizeof(double) * (size_t)Nq * d);
        double *kbar = malloc(sizeof(double) * (size_t)Nk * d);
        double *qt = malloc(sizeof(double) * (size_t)Nq * d);
        double *kt = malloc(sizeof(double) * (size_t)Nk * d);
        if (!qbar || !kbar || !qt || !kt) {
            free(qbar); free(kbar); free(qt); free(kt);
            return ORC_ENOMEM;
        }
        mean_pool(qh, Nq, Bq, d, qbar);
        mean_pool(kh, Nk, Bk, d, kbar);
        project(qbar, Nq, d, w_q, qt);
        project(kbar, Nk, d, w_k, kt);
#pragma omp parallel for schedule(dynamic, 1)
        for (int i = 0; i < Nq; ++i) {
            scored_t *row = malloc(sizeof(scored_t) * (size_t)(Nk > 0 ? Nk : 1));
            int *sel = malloc(sizeof(int) * (size_t)(topk > 0 ? topk : 1));
            if (!row || !sel) {
#pragma omp atomic write
                err = ORC_ENOMEM;
                free(row); free(sel);
                continue;
            }
            for (int j = 0; j < Nk; ++j) {
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += qt[(size_t)i * d + e] * kt[(size_t)j * d + e];
                row[j].s = bias ? acc + bias[(size_t)bh * Nk + j] : acc;
                row[j].j = j;
            }
            qsort(row, (size_t)Nk, sizeof(scored_t), by_score_desc);
            for (int a = 0; a < topk; ++a) sel[a] = row[a].j;
            qsort(sel, (size_t)topk, sizeof(int), by_int_asc);
            int32_t *dst = lut + ((size_t)bh * Nq + i) * (size_t)topk;
            for (int a = 0; a < topk; ++a) dst[a] = sel[a];
            if (gap) {
                gap[(size_t)bh * Nq + i] =
                    (topk > 0 && topk < Nk) ? row[topk - 1].s - row[topk].s : INFINITY;
            }
            free(row); free(sel);
        }
        free(qbar); free(kbar); free(qt); free(kt);
        if (err) return err;
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Per-head block statistics of the linear branch ([SALAD] sec. 2, ReLU
 * kernel function; block form as in [SLA2-it] sec. 2.A):
 *   h_j = sum_{n in block j} phi(k_n)^T v_n   (d x d)
 *   z_j = sum_{n in block j} phi(k_n)         (d)
 * with phi = ReLU. */
static void linear_block_stats(const uint16_t *kh, const uint16_t *vh, int Nk, int Bk, int d,
                               double *hj, double *zj)
{
#pragma omp parallel for schedule(static)
    for (int j = 0; j < Nk; ++j) {
        double *h = hj + (size_t)j * d * d;
        double *z = zj + (size_t)j * d;
        memset(h, 0, sizeof(double) * (size_t)d * d);
        memset(z, 0, sizeof(double) * (size_t)d);
        for (int r = 0; r < Bk; ++r) {
            size_t n = (size_t)j * Bk + r;
            for (int c = 0; c < d; ++c) {
                double fk = relu(bf(kh[n * d + c]));
                z[c] += fk;
                if (fk == 0.0) continue;
                for (int e = 0; e < d; ++e) h[(size_t)c * d + e] += fk * bf(vh[n * d + e]);
            }
        }
    }
}

/* Sort helper: requested rows grouped by head. */
static int cmp_i64(const void *pa, const void *pb)
{
    int64_t a = *(const int64_t *)pa, b = *(const int64_t *)pb;
    return (a > b) - (a < b);
}

typedef struct { int64_t row; int64_t slot; } rowreq_t;

static int by_row(const void *pa, const void *pb)
{
    const rowreq_t *a = (const rowreq_t *)pa, *b = (const rowreq_t *)pb;
    return cmp_i64(&a->row, &b->row);
}

/* Resolve the list of requested rows.  rows == NULL means every row of
 * [B,H,N] in order.  Returns a sorted list of (row, output slot). */
static rowreq_t *gather_rows(int64_t total, int64_t nrows, const int64_t *rows, int64_t *count)
{
    int64_t n = rows ? nrows : total;
    rowreq_t *req = malloc(sizeof(rowreq_t) * (size_t)(n > 0 ? n : 1));
    if (!req) return NULL;
    for (int64_t a = 0; a < n; ++a) {
        req[a].row = rows ? rows[a] : a;
        req[a].slot = a;
    }
    if (rows) qsort(req, (size_t)n, sizeof(rowreq_t), by_row);
    *count = n;
    return req;
}

/* ------------------------------------------------------------------ */
/* SLA2 forward on a given LUT.
 *   Sparse branch ([SLA2-it] sec. 2.A, eq. O; [SLA2-ar] sec. 1, the sparse
 *   branch renormalises over the kept blocks):
 *     O_s(t) = sum_{n in S_i} e^{tau q_t.k_n - m} v_n / sum_{n in S_i} e^{tau q_t.k_n - m},
 *     O_s := 0 when S_i is empty.
 *   Linear branch over the blocks not selected (phi = ReLU, [SALAD] sec. 2):
 *     O_l(t) = phi(q_t) H_U / (phi(q_t) . Z_U),
 *     H_U = sum_{j not in S_i} h_j,  Z_U = sum_{j not in S_i} z_j,
 *     O_l := 0 when the denominator is <= 0.
 *   Combine ([SLA2-it] sec. 2.A; [SLA2-ar] sec. 2.a):
 *     O = alpha . O_s + (1 - alpha) . O_l.
 *   fp8 != 0: the sparse branch runs on quantised Q, K, P and V, as the
 *   forward pass of the low-bit sparse branch does ([SLA2-it] sec. 2.C;
 *   [SLA2-ar] sec. 2.j, QAT: the forward quantises Q, K, P and V), with E4M3
 *   and these scale rules (Bk must be 64):
 *     per 64-token block b of Q, K and V: s_b = max|x| / 448 (1 for an
 *     all-zero block) and x8 = e4m3(x / s_b), the code of the exact quotient
 *     448 x / max|x| (see quantise_blocks);
 *     logits in log2 units x_tn = (q8_t . k8_n) s_q(t) s_k(j) tau log2(e);
 *     P_tn = 2^(x_tn - M_t), l_t = sum_n P_tn, where the row reference M_t is
 *       p_plain = 0: ceil(max_n x_tn), the power of two at or above the row
 *                    maximum (every change of reference is then an exact power
 *                    of two, which commutes with the E4M3 rounding of P);
 *       p_plain = 1: max_n x_tn itself, the row maximum of the softmax;
 *     Phat_tn = e4m3(P_tn 448 s_v(j) / s_vmax), s_vmax = max over the LUT row;
 *     O_s(t) = (s_vmax / 448) sum_n Phat_tn v8_n / l_t.
 *   The linear branch and the combine are not quantised.
 *   lowbit = 2 (INT8): as above, but Q and K take 8-bit integer codes,
 *   s_b = max|x| / 127 and x8 = int8(127 x / max|x|) (nearest, ties to even,
 *   within +-127), so q8_t . k8_n is an exact integer; P and V keep the E4M3
 *   rules (an integer P.V accumulator could not take the online rescale exactly).
 *   lowbit = 1 is the FP8 mode above; 0 is the unquantised branch.
 * rows: flat indices (b*H + h)*N + t (NULL = all rows, in order).
 * out, out_s, out_l: [nrows, d] (out_s, out_l may be NULL). */

/* Per-64-token-block absmax scale and codes of one head's [N, d] tensor.  Each
 * code is the rounding of the exact quotient top * x / max|x| (top = 448 for
 * E4M3, 127 for the integer code): in double, top * x is exact for a bf16 x,
 * and the correctly rounded quotient of two exact operands rounds to the same
 * code as the exact rational, because that rational is either on a rounding
 * midpoint (and then exactly representable) or at least 2^-17 of its size
 * away from every midpoint.  The scale s = max|x| / top (double) dequantises. */
static void quantise_blocks(const uint16_t *x, int N, int d, double *x8, double *scale, int int8)
{
    const double top = int8 ? 127.0 : 448.0;
    for (int b = 0; b < N / 64; ++b) {
        double amax = 0.0;
        for (size_t e = (size_t)b * 64 * d; e < (size_t)(b + 1) * 64 * d; ++e)
            if (fabs(bf(x[e])) > amax) amax = fabs(bf(x[e]));
        scale[b] = amax > 0.0 ? amax / top : 1.0;
        for (size_t e = (size_t)b * 64 * d; e < (size_t)(b + 1) * 64 * d; ++e) {
            const double quotient = amax > 0.0 ? (top * bf(x[e])) / amax : 0.0;
            x8[e] = int8 ? oracle_int8(quotient) : oracle_e4m3(quotient);
        }
    }
}

/* The per-block codes and scales of quantise_blocks for one [N, d] bf16 tensor
 * (N a multiple of 64): codes [N*d], scales [N/64].  int8 = 0: E4M3 codes
 * (top 448); 1: 8-bit integer codes (top 127). */
int oracle_quantise(const uint16_t *x, int N, int d, int int8, double *codes, double *scales)
{
    if (!x || !codes || !scales || N <= 0 || d <= 0 || N % 64) return ORC_EINVAL;
    quantise_blocks(x, N, d, codes, scales, int8 != 0);
    return ORC_OK;
}

int oracle_sla_forward(int B, int H, int N, int d, int Bq, int Bk, int topk, double sm_scale,
                       const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const float *alpha, const int32_t *lut,
                       int64_t nrows, const int64_t *rows,
                       double *out, double *out_s, double *out_l, int lowbit, int p_plain,
                       int nthreads)
{
    if (!check_shape(B, H, N, d, Bq, Bk, topk) || !q || !k || !v || !alpha || !lut || !out)
        return ORC_EINVAL;
    if (lowbit < 0 || lowbit > 2 || p_plain < 0 || p_plain > 1) return ORC_EINVAL;
    const int fp8 = lowbit != 0;                   /* some quantised sparse branch */
    if (fp8 && Bk != 64) return ORC_EINVAL;
    set_threads(nthreads);
    const int Nq = N / Bq, Nk = N / Bk;
    const double tau = sm_scale > 0.0 ? sm_scale : 1.0 / sqrt((double)d);
    const int64_t total = (int64_t)B * H * N;
    for (int64_t a = 0; a < (int64_t)B * H * Nq; ++a)
        if (!lut_row_valid(lut + a * topk, topk, Nk)) return ORC_EINVAL;
    int64_t n = 0;
    rowreq_t *req = gather_rows(total, nrows, rows, &n);
    if (!req) return ORC_ENOMEM;
    for (int64_t a = 0; a < n; ++a)
        if (req[a].row < 0 || req[a].row >= total) { free(req); return ORC_EINVAL; }

    double *hj = malloc(sizeof(double) * (size_t)Nk * d * d);
    double *zj = malloc(sizeof(double) * (size_t)Nk * d);
    /* FP8: one head's codes and scales */
    const size_t nq8 = fp8 ? (size_t)N * d : 1, ns8 = fp8 ? (size_t)N / 64 : 1;
    double *q8 = malloc(sizeof(double) * nq8), *k8 = malloc(sizeof(double) * nq8);
    double *v8 = malloc(sizeof(double) * nq8);
    double *sq = malloc(sizeof(double) * ns8), *sk = malloc(sizeof(double) * ns8);
    double *sv = malloc(sizeof(double) * ns8);
    if (!hj || !zj || !q8 || !k8 || !v8 || !sq || !sk || !sv) {
        free(req); free(hj); free(zj);
        free(q8); free(k8); free(v8); free(sq); free(sk); free(sv);
        return ORC_ENOMEM;
    }
    const double log2e = 1.0 / log(2.0);
    int err = ORC_OK;

    int64_t a0 = 0;
    while (a0 < n) {
        const int64_t bh = req[a0].row / N;
        int64_t a1 = a0;
        while (a1 < n && req[a1].row / N == bh) ++a1;
        const uint16_t *qh = q + (size_t)bh * N * d;
        const uint16_t *kh = k + (size_t)bh * N * d;
        const uint16_t *vh = v + (size_t)bh * N * d;
        linear_block_stats(kh, vh, Nk, Bk, d, hj, zj);
        if (fp8) {
            quantise_blocks(qh, N, d, q8, sq, lowbit == 2);
            quantise_blocks(kh, N, d, k8, sk, lowbit == 2);
            quantise_blocks(vh, N, d, v8, sv, 0);
        }

        /* distinct query blocks among the requested rows of this head */
        int64_t nblk = 0;
        int64_t *blk_first = malloc(sizeof(int64_t) * (size_t)(a1 - a0 + 1));
        if (!blk_first) { err = ORC_ENOMEM; break; }
        for (int64_t a = a0; a < a1; ++a) {
            int i = (int)((req[a].row % N) / Bq);
            if (a == a0 || i != (int)((req[a - 1].row % N) / Bq)) blk_first[nblk++] = a;
        }
        blk_first[nblk] = a1;

#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t bi = 0; bi < nblk; ++bi) {
            const int i = (int)((req[blk_first[bi]].row % N) / Bq);
            const int32_t *S = lut + ((size_t)bh * Nq + i) * (size_t)topk;
            char *selected = calloc((size_t)Nk, 1);
            double *HU = calloc((size_t)d * d, sizeof(double));
            double *ZU = calloc((size_t)d, sizeof(double));
            double *logit = malloc(sizeof(double) * (size_t)(topk * Bk > 0 ? topk * Bk : 1));
            double *qd = malloc(sizeof(double) * (size_t)d);
            if (!selected || !HU || !ZU || !logit || !qd) {
#pragma omp atomic write
                err = ORC_ENOMEM;
                free(selected); free(HU); free(ZU); free(logit); free(qd);
                continue;
            }
            for (int a = 0; a < topk; ++a) selected[S[a]] = 1;
            for (int j = 0; j < Nk; ++j) {
                if (selected[j]) continue;
                for (size_t c = 0; c < (size_t)d * d; ++c) HU[c] += hj[(size_t)j * d * d + c];
                for (int c = 0; c < d; ++c) ZU[c] += zj[(size_t)j * d + c];
            }
            for (int64_t a = blk_first[bi]; a < blk_first[bi + 1]; ++a) {
                const int64_t t = req[a].row % N;
                double *o = out + req[a].slot * d;
                for (int c = 0; c < d; ++c) qd[c] = bf(qh[(size_t)t * d + c]);

                double den_s = 0.0;
                double os[512];
                double ol[512];
                for (int c = 0; c < d; ++c) { os[c] = 0.0; ol[c] = 0.0; }
                if (fp8) {
                    /* quantised sparse branch: log2-unit logits; the row reference is
                     * the power of two at or above the row maximum, or (p_plain) the
                     * row maximum itself */
                    double svmax = 0.0, mx = -INFINITY;
                    for (int s = 0; s < topk; ++s)
                        if (sv[S[s]] > svmax) svmax = sv[S[s]];
                    for (int s = 0; s < topk; ++s) {
                        for (int r = 0; r < Bk; ++r) {
                            size_t nn = (size_t)S[s] * Bk + r;
                            double acc = 0.0;
                            for (int c = 0; c < d; ++c) acc += q8[(size_t)t * d + c] * k8[nn * d + c];
                            const double x = acc * sq[t / 64] * sk[S[s]] * tau * log2e;
                            logit[s * Bk + r] = x;
                            if (x > mx) mx = x;
                        }
                    }
                    const double M = p_plain ? mx : ceil(mx);
                    for (int s = 0; s < topk; ++s) {
                        const double qf = 448.0 * sv[S[s]] / svmax;
                        for (int r = 0; r < Bk; ++r) {
                            size_t nn = (size_t)S[s] * Bk + r;
                            const double p = exp2(logit[s * Bk + r] - M);
                            den_s += p;
                            const double ph = oracle_e4m3(p * qf);
                            for (int c = 0; c < d; ++c) os[c] += ph * v8[nn * d + c];
                        }
                    }
                    for (int c = 0; c < d; ++c) os[c] = den_s > 0.0 ? os[c] * (svmax / 448.0) / den_s : 0.0;
                } else {
                    /* exact sparse branch: two passes, max then weights */
                    double m = -INFINITY;
                    for (int s = 0; s < topk; ++s) {
                        for (int r = 0; r < Bk; ++r) {
                            size_t nn = (size_t)S[s] * Bk + r;
                            double acc = 0.0;
                            for (int c = 0; c < d; ++c) acc += qd[c] * bf(kh[nn * d + c]);
                            logit[s * Bk + r] = tau * acc;
                            if (tau * acc > m) m = tau * acc;
                        }
                    }
                    for (int s = 0; s < topk; ++s) {
                        for (int r = 0; r < Bk; ++r) {
                            size_t nn = (size_t)S[s] * Bk + r;
                            double p = exp(logit[s * Bk + r] - m);
                            den_s += p;
                            for (int c = 0; c < d; ++c) os[c] += p * bf(vh[nn * d + c]);
                        }
                    }
                    for (int c = 0; c < d; ++c) os[c] = den_s > 0.0 ? os[c] / den_s : 0.0;
                }

                /* linear branch over the unselected blocks */
                double den_l = 0.0;
                for (int c = 0; c < d; ++c) den_l += relu(qd[c]) * ZU[c];
                if (den_l > 0.0) {
                    for (int c = 0; c < d; ++c) {
                        double fq = relu(qd[c]);
                        if (fq == 0.0) continue;
                        for (int e = 0; e < d; ++e) ol[e] += fq * HU[(size_t)c * d + e];
                    }
                    for (int e = 0; e < d; ++e) ol[e] /= den_l;
                }

                const double al = (double)alpha[(size_t)bh * N + t];
                for (int c = 0; c < d; ++c) o[c] = al * os[c] + (1.0 - al) * ol[c];
                if (out_s) memcpy(out_s + req[a].slot * d, os, sizeof(double) * (size_t)d);
                if (out_l) memcpy(out_l + req[a].slot * d, ol, sizeof(double) * (size_t)d);
            }
            free(selected); free(HU); free(ZU); free(logit); free(qd);
        }
        free(blk_first);
        if (err) break;
        a0 = a1;
    }
    free(hj); free(zj); free(req);
    free(q8); free(k8); free(v8); free(sq); free(sk); free(sv);
    return err;
}

/* ------------------------------------------------------------------ */
/* PISA exact-or-approximate forward on a given LUT ([PISA] sec. 2,
 * "Algoritmo Core"):
 *   o_t = N_t / D_t,
 *   N_t = sum_{j in S_i} sum_n e^{c_tn - m} v_{j,n} + sum_{j in U_i} e^{cbar_tj - m} (sum_n v_{j,n}),
 *   D_t = sum_{j in S_i} sum_n e^{c_tn - m}         + sum_{j in U_i} Bk e^{cbar_tj - m},
 * with c_tn = tau q_t . k_{j,n}, cbar_tj = tau q_t . kbar_j, kbar_j the mean
 * key of block j (the block centroid), U_i every block not in S_i, and m
 * the maximum over all exact and centroid logits.  The D_t term is the sum
 * over the block's Bk keys of the zero-order expansion e^{q kbar}; its
 * first-order part vanishes because sum_n (k_n - kbar) = 0.  The global
 * first_order != 0 adds the global first-order correction, the third N_t term:
 *   + tau (q_t Hbar) sum_{j in U_i} e^{cbar_tj - m},
 *   Hbar = (1/Nk) sum_j H_j,  H_j = sum_{n in j} (k_n - kbar_j)^T v_n,
 * the mean of the blocks' first-order matrices (the Taylor term of e^{tau q.k_n}
 * around kbar_j is tau e^{tau q.kbar_j} q.(k_n - kbar_j)); D_t has no first-order
 * part. */
int oracle_pisa_forward(int B, int H, int N, int d, int Bq, int Bk, int topk, double sm_scale,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *lut, int64_t nrows, const int64_t *rows,
                        double *out, int first_order, int nthreads)
{
    if (!check_shape(B, H, N, d, Bq, Bk, topk) || !q || !k || !v || !lut || !out)
        return ORC_EINVAL;
    set_threads(nthreads);
    const int Nq = N / Bq, Nk = N / Bk;
    const double tau = sm_scale > 0.0 ? sm_scale : 1.0 / sqrt((double)d);
    const int64_t total = (int64_t)B * H * N;
    for (int64_t a = 0; a < (int64_t)B * H * Nq; ++a)
        if (!lut_row_valid(lut + a * topk, topk, Nk)) return ORC_EINVAL;
    int64_t n = 0;
    rowreq_t *req = gather_rows(total, nrows, rows, &n);
    if (!req) return ORC_ENOMEM;
    for (int64_t a = 0; a < n; ++a)
        if (req[a].row < 0 || req[a].row >= total) { free(req); return ORC_EINVAL; }
    double *kbar = malloc(sizeof(double) * (size_t)Nk * d);
    double *vsum = malloc(sizeof(double) * (size_t)Nk * d);
    double *hbar = malloc(sizeof(double) * (size_t)d * d);
    if (!kbar || !vsum || !hbar) { free(req); free(kbar); free(vsum); free(hbar); return ORC_ENOMEM; }
    int err = ORC_OK;

    int64_t a0 = 0;
    while (a0 < n) {
        const int64_t bh = req[a0].row / N;
        int64_t a1 = a0;
        while (a1 < n && req[a1].row / N == bh) ++a1;
        const uint16_t *qh = q + (size_t)bh * N * d;
        const uint16_t *kh = k + (size_t)bh * N * d;
        const uint16_t *vh = v + (size_t)bh * N * d;
        mean_pool(kh, Nk, Bk, d, kbar);
        for (int j = 0; j < Nk; ++j)
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int r = 0; r < Bk; ++r) acc += bf(vh[((size_t)j * Bk + r) * d + c]);
                vsum[(size_t)j * d + c] = acc;
            }
        if (first_order) {
            /* Hbar = (1/Nk) sum_j H_j, H_j = sum_{n in j} (k_n - kbar_j)^T v_n ([PISA]
             * sec. 2: the mean of the blocks' first-order matrices over all blocks) */
            memset(hbar, 0, sizeof(double) * (size_t)d * d);
            for (int j = 0; j < Nk; ++j)
                for (int r = 0; r < Bk; ++r) {
                    const size_t nn = (size_t)j * Bk + r;
                    for (int c = 0; c < d; ++c) {
                        const double dk = bf(kh[nn * d + c]) - kbar[(size_t)j * d + c];
                        for (int e = 0; e < d; ++e) hbar[(size_t)c * d + e] += dk * bf(vh[nn * d + e]);
                    }
                }
            for (size_t c = 0; c < (size_t)d * d; ++c) hbar[c] /= (double)Nk;
        }

#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t a = a0; a < a1; ++a) {
            const int64_t t = req[a].row % N;
            const int i = (int)(t / Bq);
            const int32_t *S = lut + ((size_t)bh * Nq + i) * (size_t)topk;
            double *o = out + req[a].slot * d;
            char *selected = calloc((size_t)Nk, 1);
            double *ex = malloc(sizeof(double) * (size_t)(topk * Bk > 0 ? topk * Bk : 1));
            double *cb = malloc(sizeof(double) * (size_t)Nk);
            double *qd = malloc(sizeof(double) * (size_t)d);
            if (!selected || !ex || !cb || !qd) {
#pragma omp atomic write
                err = ORC_ENOMEM;
                free(selected); free(ex); free(cb); free(qd);
                continue;
            }
            for (int s = 0; s < topk; ++s) selected[S[s]] = 1;
            for (int c = 0; c < d; ++c) qd[c] = bf(qh[(size_t)t * d + c]);
            double m = -INFINITY;
            for (int s = 0; s < topk; ++s)
                for (int r = 0; r < Bk; ++r) {
                    size_t nn = (size_t)S[s] * Bk + r;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += qd[c] * bf(kh[nn * d + c]);
                    ex[s * Bk + r] = tau * acc;
                    if (ex[s * Bk + r] > m) m = ex[s * Bk + r];
                }
            for (int j = 0; j < Nk; ++j) {
                if (selected[j]) continue;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qd[c] * kbar[(size_t)j * d + c];
                cb[j] = tau * acc;
                if (cb[j] > m) m = cb[j];
            }
            double num[512];
            for (int c = 0; c < d; ++c) num[c] = 0.0;
            double den = 0.0;
            for (int s = 0; s < topk; ++s)
                for (int r = 0; r < Bk; ++r) {
                    size_t nn = (size_t)S[s] * Bk + r;
                    double w = exp(ex[s * Bk + r] - m);
                    den += w;
                    for (int c = 0; c < d; ++c) num[c] += w * bf(vh[nn * d + c]);
                }
            double wu = 0.0;      /* sum over U of e^{tau q.kbar_j - m} */
            for (int j = 0; j < Nk; ++j) {
                if (selected[j]) continue;
                double w = exp(cb[j] - m);
                wu += w;
                den += (double)Bk * w;
                for (int c = 0; c < d; ++c) num[c] += w * vsum[(size_t)j * d + c];
            }
            if (first_order && wu > 0.0) {
                /* global first-order term: tau (q_t Hbar) sum_{j in U} e^{tau q.kbar_j - m}
                 * (the derivative of e^{tau q.k} at kbar_j is tau e^{tau q.kbar_j} q) */
                for (int e = 0; e < d; ++e) {
                    double qh_e = 0.0;
                    for (int c = 0; c < d; ++c) qh_e += qd[c] * hbar[(size_t)c * d + e];
                    num[e] += tau * qh_e * wu;
                }
            }
            for (int c = 0; c < d; ++c) o[c] = num[c] / den;
            free(selected); free(ex); free(cb); free(qd);
        }
        if (err) break;
        a0 = a1;
    }
    free(kbar); free(vsum); free(hbar); free(req);
    return err;
}

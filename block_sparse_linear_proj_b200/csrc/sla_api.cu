// sla_api.cu -- host side of the C ABI declared in include/sla.h: argument
// validation, workspace carving, TMA descriptor encoding and kernel launches.
// All device code lives in the included .cuh files (one translation unit, so
// the device status word needs no relocatable device code).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/sla.h"
#include "attn.cuh"
#include "cocluster.cuh"
#include "common.cuh"
#include "cov.cuh"
#include "kv_stats.cuh"
#include "router.cuh"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ------------------------------------------------------------- validation
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sla_status_t check_params(const sla_params_t* p) {
    if (!p) return SLA_ERR_INVALID_ARG;
    if (p->B <= 0 || p->H <= 0 || p->N <= 0 || p->d <= 0 || p->Bq <= 0 || p->Bk <= 0 ||
        p->topk < 0)
        return SLA_ERR_INVALID_ARG;
    if (p->N % p->Bq != 0 || p->N % p->Bk != 0) return SLA_ERR_INVALID_ARG;
    if (p->topk > p->N / p->Bk) return SLA_ERR_INVALID_ARG;
    if (p->sparse_dtype != SLA_SPARSE_BF16 && p->sparse_dtype != SLA_SPARSE_FP8_E4M3 &&
        p->sparse_dtype != SLA_SPARSE_INT8)
        return SLA_ERR_INVALID_ARG;
    if (p->lut_mode != SLA_LUT_COMPUTE && p->lut_mode != SLA_LUT_GIVEN) return SLA_ERR_INVALID_ARG;
    if (p->pisa_first_order != 0 && p->pisa_first_order != 1) return SLA_ERR_INVALID_ARG;
    if (!(p->pisa_cov_lambda >= 0.f) || !std::isfinite(p->pisa_cov_lambda)) return SLA_ERR_INVALID_ARG;
    if (p->out_dtype != SLA_OUT_BF16 && p->out_dtype != SLA_OUT_FP32) return SLA_ERR_INVALID_ARG;
    if (!(std::isfinite(p->sm_scale))) return SLA_ERR_INVALID_ARG;
    if (p->d != 64 && p->d != 128) return SLA_ERR_UNSUPPORTED;
    if (p->Bq != 64 && p->Bq != 128) return SLA_ERR_UNSUPPORTED;
    if (p->Bk != 64) return SLA_ERR_UNSUPPORTED;
    if (p->N / p->Bk > 8192) return SLA_ERR_UNSUPPORTED;
    const long long bh = static_cast<long long>(p->B) * p->H;
    if (bh > 65535) return SLA_ERR_UNSUPPORTED;
    if (bh * p->N > 0x7fffffffLL) return SLA_ERR_UNSUPPORTED;
    return SLA_OK;
}

sla_status_t check_tensor(const void* t, size_t align) {
    if (!t) return SLA_ERR_INVALID_ARG;
    if (!aligned(t, align)) return SLA_ERR_INVALID_ARG;
    return SLA_OK;
}

// ------------------------------------------------------------- workspace
struct Ws {
    size_t qbar, kbarT, m, lut, zj, hpart, hsum, zsum, kc, vbar, v16, phik16;
    size_t q8, k8, v8t, sq, sk, sv;       // FP8 sparse branch
    size_t covhbar, covbias, covtri;   // covariance-aware PISA selection (chunk sums: hpart)
    size_t total;
    int nchunk, bpc;
};

// K/V pre-pass chunking for bh heads: ~4 waves of CTAs over the heads, >= 8
// blocks per chunk.
void kv_chunking(long long bh, long long Nk, int& bpc, int& nchunk) {
    const long long target = std::max<long long>(1, 592 / bh);
    bpc = std::max<int>(8, static_cast<int>((Nk + target - 1) / target));
    nchunk = static_cast<int>((Nk + bpc - 1) / bpc);
}

Ws layout(const sla_params_t* p) {
    Ws w{};
    const size_t BH = static_cast<size_t>(p->B) * p->H;
    const size_t d = p->d, Nq = p->N / p->Bq, Nk = p->N / p->Bk;
    kv_chunking(static_cast<long long>(BH), static_cast<long long>(Nk), w.bpc, w.nchunk);
    // The chunk partials are sized for the most that any call over at most BH
    // heads (same N, d, blocks and modes) uses, so that the workspace size never
    // falls as heads are added and a workspace for BH heads serves a call over a
    // subset of them.  Above 592 heads a head is one chunk.
    size_t parts = BH * static_cast<size_t>(w.nchunk);
    for (long long h = 1; h < std::min<long long>(static_cast<long long>(BH), 593); ++h) {
        int b_ = 0, n_ = 0;
        kv_chunking(h, static_cast<long long>(Nk), b_, n_);
        parts = std::max(parts, static_cast<size_t>(h) * n_);
    }
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.qbar = take(BH * Nq * d * 8);
    w.kbarT = take(BH * Nk * d * 8);
    w.m = take(d * d * 8);
    w.lut = take(BH * Nq * static_cast<size_t>(p->topk) * 4 + 4);
    w.zj = take(BH * Nk * d * 4);
    w.hpart = take(parts * d * d * 4);
    w.hsum = take(BH * d * d * 4);
    w.zsum = take(BH * d * 4);
    w.kc = take(BH * Nk * d * 2);
    w.vbar = take(BH * Nk * d * 2);
    w.v16 = take(BH * static_cast<size_t>(p->N) * d * 2);
    w.phik16 = take(BH * static_cast<size_t>(p->N) * d * 2);
    if (p->sparse_dtype != SLA_SPARSE_BF16) {     // 8-bit Q, K, V^T codes and their scales
        w.q8 = take(BH * static_cast<size_t>(p->N) * d);
        w.k8 = take(BH * static_cast<size_t>(p->N) * d);
        w.v8t = take(BH * static_cast<size_t>(p->N) * d);
        w.sq = take(BH * static_cast<size_t>(p->N) / 64 * 4);
        w.sk = take(BH * Nk * 4);
        w.sv = take(BH * Nk * 4);
    }
    if (p->pisa_cov_lambda > 0.f) {               // chunk sums of H_j, Hbar, lambda M_j
        w.covhbar = take(BH * d * d * 4);
        w.covbias = take(BH * Nk * 8);
        w.covtri = take(BH * Nk * sla::kTriStride * 8);
    }
    w.total = off;
    return w;
}

sla_status_t check_ws(const sla_params_t* p, void* ws, size_t ws_bytes, Ws& w) {
    w = layout(p);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < w.total) return SLA_ERR_WORKSPACE;
    return SLA_OK;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

// ------------------------------------------------------------- TMA maps
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(f);
    });
    return fn;
}

// 2-D map over [rows, d] (d innermost), box [box_bytes of columns, box_rows]
// (128 bytes, 128-byte swizzle, unless given).
bool make_map(CUtensorMap* m, const void* base, long long rows, int d, int box_rows,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int box_bytes = 128,
              CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const int es = dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : (dt == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2);
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * es};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes / es), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned long long wait_limit_ns() {
    const char* s = std::getenv("SLA_DEBUG_WAIT_LIMIT_NS");
    if (s && *s) {
        const unsigned long long v = std::strtoull(s, nullptr, 10);
        if (v > 0) return v;
    }
    return 2000000000ull;
}

// Test hook for failure detection: with SLA_DEBUG_STALL set (and not "0") the
// attention kernel's loader issues no K/V tile loads, so the consumers' bounded
// waits run out and the call reports SLA_ERR_TIMEOUT; no access is made that
// would not be made otherwise.
bool debug_stall() {
    const char* s = std::getenv("SLA_DEBUG_STALL");
    return s && *s && *s != '0';
}

bool check_after_call() {
    const char* s = std::getenv("SLA_CHECK");
    return s && *s && *s != '0';
}

sla_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

// ------------------------------------------------------------- tracing
struct Profiler {
    std::mutex mu;
    bool on = false;
    struct Rec { int kind; cudaEvent_t a, b; };
    std::vector<Rec> recs;
    std::vector<cudaEvent_t> pool;
    cudaEvent_t get() {
        if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
};
Profiler& prof() { static Profiler p; return p; }

// Brackets one launch with events when tracing is on.
struct Span {
    int kind; cudaStream_t st; cudaEvent_t a = nullptr, b = nullptr;
    Span(int k, cudaStream_t s) : kind(k), st(s) {
        Profiler& P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        if (!P.on) return;
        a = P.get(); b = P.get();
        if (a) cudaEventRecord(a, st);
    }
    ~Span() {
        if (!a || !b) return;
        cudaEventRecord(b, st);
        Profiler& P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        P.recs.push_back({kind, a, b});
    }
};

// A phase of a call on the caller's stream: opened at the call's entry, closed
// by end() (when tracing is on; otherwise both are no-ops).
struct Phase {
    int kind; cudaStream_t st; cudaEvent_t a = nullptr;
    Phase(int k, cudaStream_t s) : kind(k), st(s) {
        Profiler& P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        if (!P.on) return;
        a = P.get();
        if (a) cudaEventRecord(a, st);
    }
    void end() {
        if (!a) return;
        Profiler& P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        cudaEvent_t b = P.get();
        if (b) {
            cudaEventRecord(b, st);
            P.recs.push_back({kind, a, b});
        } else {
            P.pool.push_back(a);
        }
        a = nullptr;
    }
    ~Phase() {
        if (!a) return;
        Profiler& P = prof();
        std::lock_guard<std::mutex> g(P.mu);
        P.pool.push_back(a);   // the call failed before its attention kernel
    }
};

// ------------------------------------------------------------- launchers
int grid_blocks(long long n, int per_sm) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long cap = static_cast<long long>(sms) * per_sm;
    return static_cast<int>(std::max<long long>(1, std::min(n, cap)));
}

void launch_pool(const void* x, int rows, long long nblk_total, int nblk_per_head, int d,
                 int out_mode, double* out, cudaStream_t st) {
    // one warp per pooled block, eight warps per CTA
    const int grid = grid_blocks((nblk_total + 7) / 8, 8);
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    Span sp(SLA_KERNEL_POOL, st);
    if (d == 128)
        sla::pool_mean_kernel<128><<<grid, 256, 0, st>>>(xb, rows, nblk_total, nblk_per_head, out_mode, out);
    else
        sla::pool_mean_kernel<64><<<grid, 256, 0, st>>>(xb, rows, nblk_total, nblk_per_head, out_mode, out);
}

// shared memory of score_topk_kernel<R, D>: qhat tiles, histograms, keys
size_t score_smem(int R, int D, int Nk) {
    const size_t mt = R >= 8 ? R / 8 : 1, ldq = D + 4;
    const size_t ldk = std::max<size_t>(Nk, ldq);
    return 8 * mt * ldq * 8 + 8 * 256 * 4 + R * ldk * 8;
}

template <int R, int D, int DEPTH, int MINB>
sla_status_t launch_score_r(const double* qhat, const double* kbarT, const double* bias, int BH,
                            int Nq, int Nk, int topk, int32_t* lut, cudaStream_t st) {
    const size_t smem = score_smem(R, D, Nk);
    auto kern = sla::score_topk_kernel<R, D, DEPTH, MINB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return SLA_ERR_CUDA;
    dim3 grid((Nq + R - 1) / R, BH);
    Span sp(SLA_KERNEL_SCORE_TOPK, st);
    kern<<<grid, 256, smem, st>>>(qhat, kbarT, bias, Nq, Nk, topk, lut);
    return launch_status();
}

template <int D>
sla_status_t launch_score(const double* qhat, const double* kbarT, const double* bias, int BH,
                          int Nq, int Nk, int topk, int32_t* lut, cudaStream_t st) {
    // 16 query blocks per CTA (two 8-row tiles of the fp64 MMA per K fragment).
    // Where two CTAs fit an SM's shared memory, a two-deep fragment ring keeps
    // the registers within two CTAs; otherwise one CTA per SM with a four-deep ring.
    constexpr size_t two = 113 * 1024, one = 200 * 1024;
    if (score_smem(16, D, Nk) <= two)
        return launch_score_r<16, D, 2, 2>(qhat, kbarT, bias, BH, Nq, Nk, topk, lut, st);
    if (score_smem(16, D, Nk) <= one)
        return launch_score_r<16, D, 4, 1>(qhat, kbarT, bias, BH, Nq, Nk, topk, lut, st);
    if (score_smem(8, D, Nk) <= one) return launch_score_r<8, D, 4, 1>(qhat, kbarT, bias, BH, Nq, Nk, topk, lut, st);
    if (score_smem(4, D, Nk) <= one) return launch_score_r<4, D, 4, 1>(qhat, kbarT, bias, BH, Nq, Nk, topk, lut, st);
    if (score_smem(2, D, Nk) > 232448) return SLA_ERR_UNSUPPORTED;   // a score row beyond shared memory
    return launch_score_r<2, D, 4, 1>(qhat, kbarT, bias, BH, Nq, Nk, topk, lut, st);
}

// Router, first part: Q (and K, unless the pre-pass pools it) pooling, W folding
// and the projection qhat = qbar W_q W_k^T (in place).
sla_status_t router_pool(const sla_params_t* p, const void* q, const void* k, const float* w_q,
                         const float* w_k, void* ws, const Ws& w, bool pool_k, cudaStream_t st) {
    const int BH = p->B * p->H, Nq = p->N / p->Bq, Nk = p->N / p->Bk, d = p->d;
    double* qbar = at<double>(ws, w.qbar);
    launch_pool(q, p->Bq, static_cast<long long>(BH) * Nq, Nq, d, 0, qbar, st);
    if (pool_k) launch_pool(k, p->Bk, static_cast<long long>(BH) * Nk, Nk, d, 1, at<double>(ws, w.kbarT), st);
    if (w_q || w_k) {
        double* m = at<double>(ws, w.m);
        {
            Span sp(SLA_KERNEL_FOLD_W, st);
            sla::fold_w_kernel<<<d, 128, 0, st>>>(w_q, w_k, d, m);
        }
        const long long rows = static_cast<long long>(BH) * Nq;
        const int grid = static_cast<int>((rows + 15) / 16);
        Span sp(SLA_KERNEL_PROJECT, st);
        if (d == 128)
            sla::project_kernel<128><<<grid, 256, 0, st>>>(qbar, rows, m);
        else
            sla::project_kernel<64><<<grid, 256, 0, st>>>(qbar, rows, m);
    }
    return launch_status() == SLA_OK ? SLA_OK : SLA_ERR_CUDA;
}

// Router, second part: fp64 score + top-k (after kbar_ready, when given: the
// pooled K means of the pre-pass on the side stream).
sla_status_t router_score(const sla_params_t* p, int32_t* lut, void* ws, const Ws& w,
                          cudaStream_t st, cudaEvent_t kbar_ready = nullptr,
                          const double* bias = nullptr) {
    const int BH = p->B * p->H, Nq = p->N / p->Bq, Nk = p->N / p->Bk;
    if (kbar_ready && cudaStreamWaitEvent(st, kbar_ready, 0) != cudaSuccess) return SLA_ERR_CUDA;
    const double* qhat = at<double>(ws, w.qbar);
    const double* kbarT = at<double>(ws, w.kbarT);
    if (p->d == 128) return launch_score<128>(qhat, kbarT, bias, BH, Nq, Nk, p->topk, lut, st);
    return launch_score<64>(qhat, kbarT, bias, BH, Nq, Nk, p->topk, lut, st);
}

// Covariance norms of the PISA selection: out[bh * Nk + j] = scale * M_j.
// The K/V pre-pass has left the chunk sums of H_j in w.hpart (its exact
// three-part product, kv_stats_kernel<D, true, true>).
template <int D>
sla_status_t launch_cov_t(const sla_params_t* p, const void* k, const void* v, void* ws, const Ws& w,
                          double scale, double* out, cudaStream_t st) {
    const int BH = p->B * p->H, Nk = p->N / p->Bk;
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    float* part = at<float>(ws, w.hpart);
    float* hbar = at<float>(ws, w.covhbar);
    // (alignment slack; the four operand tiles, later H_j, take the first 2 * 64 * D * 4 bytes;
    // barrier, TMEM slot and flag after the tridiagonal matrix)
    const size_t smem_n = 1024 + 2 * sla::kCovTok * D * 4 + 9 * D * 8 +
                          (sla::kQRows * D + 10 * D + 16 + 32) * 4 + 8 + 2 * sla::kLanczos * 8 + 16;
    double* tri = at<double>(ws, w.covtri);
    auto kn = sla::cov_norm_kernel<D>;
    if (cudaFuncSetAttribute(kn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_n)) != cudaSuccess)
        return SLA_ERR_CUDA;
    {
        Span sp(SLA_KERNEL_COV, st);
        sla::cov_hbar_kernel<D><<<dim3(D * D / 256, BH), 256, 0, st>>>(part, w.nchunk, Nk, hbar);
    }
    {
        Span sp(SLA_KERNEL_COV, st);
        kn<<<dim3(Nk, BH), 256, smem_n, st>>>(kb, vb, p->N, Nk, hbar, tri, wait_limit_ns());
    }
    {
        Span sp(SLA_KERNEL_COV, st);
        const long long nblk = static_cast<long long>(BH) * Nk;
        sla::cov_eig_kernel<<<static_cast<unsigned>((nblk + 7) / 8), 256, 0, st>>>(tri, nblk, scale, out);
    }
    return launch_status();
}

sla_status_t launch_cov(const sla_params_t* p, const void* k, const void* v, void* ws, const Ws& w,
                        double scale, double* out, cudaStream_t st) {
    return p->d == 128 ? launch_cov_t<128>(p, k, v, ws, w, scale, out, st)
                       : launch_cov_t<64>(p, k, v, ws, w, scale, out, st);
}

sla_status_t run_router(const sla_params_t* p, const void* q, const void* k, const float* w_q,
                        const float* w_k, int32_t* lut, void* ws, const Ws& w, cudaStream_t st) {
    const sla_status_t s = router_pool(p, q, k, w_q, w_k, ws, w, true, st);
    return s != SLA_OK ? s : router_score(p, lut, ws, w, st);
}

template <int D>
sla_status_t launch_kv(const sla_params_t* p, const void* k, const void* v, void* ws, const Ws& w,
                       bool want_kbar, bool sla_stats, bool pisa_stats, cudaStream_t st,
                       bool fp8 = false, bool first_order = false, cudaEvent_t after_stats = nullptr,
                       bool k_int8 = false, bool cov_exact = false) {
    const int BH = p->B * p->H, Nk = p->N / p->Bk;
    sla::KvStatsArgs a{};
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.N = p->N;
    a.Nk = Nk;
    a.blocks_per_chunk = w.bpc;
    a.nchunk = w.nchunk;
    a.kbarT = want_kbar ? at<double>(ws, w.kbarT) : nullptr;
    a.zj = sla_stats ? at<float>(ws, w.zj) : nullptr;
    // cov_exact: the product sums the blocks' H_j exactly (three-part keys), for
    // the covariance norms and, with first_order, for the first-order term too
    a.hpart = (sla_stats || first_order || cov_exact) ? at<float>(ws, w.hpart) : nullptr;
    a.center = (first_order || cov_exact) ? 1 : 0;
    a.kc = pisa_stats ? at<__nv_bfloat16>(ws, w.kc) : nullptr;
    a.vbar = pisa_stats ? at<__half>(ws, w.vbar) : nullptr;
    // (the forward's fp16 V copy; a call that only wants the covariance sums makes none)
    const bool cov_only = cov_exact && !want_kbar && !sla_stats && !pisa_stats && !first_order;
    a.v16 = cov_only ? nullptr : at<__half>(ws, w.v16);
    a.phik16 = sla_stats ? at<__half>(ws, w.phik16) : nullptr;
    a.k8 = fp8 ? at<uint8_t>(ws, w.k8) : nullptr;
    a.v8t = fp8 ? at<uint8_t>(ws, w.v8t) : nullptr;
    a.sk = fp8 ? at<float>(ws, w.sk) : nullptr;
    a.sv = fp8 ? at<float>(ws, w.sv) : nullptr;
    a.k_int8 = (fp8 && k_int8) ? 1 : 0;
    a.wait_ns = wait_limit_ns();
    // alignment slack, K/V ring, column partials, maxima, column means, barrier,
    // TMEM slot, flag
    // (X3: two ring stages and two more tiles, and the fp64 column means)
    const size_t smem = 1024 + (cov_exact ? 6 : sla::kKvStages * 2) * 64 * D * 2 + 256 * 8 + 2 * 256 * 4 +
                        16 * 4 + 128 * 4 + (cov_exact ? D * 8 : 0) + 16;
    auto kern = cov_exact ? sla::kv_stats_kernel<D, true, true>
                          : a.hpart ? sla::kv_stats_kernel<D, true> : sla::kv_stats_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return SLA_ERR_CUDA;
    {
        Span sp(SLA_KERNEL_KV_STATS, st);
        kern<<<dim3(w.nchunk, BH), 256, smem, st>>>(a);
    }
    if (after_stats && cudaEventRecord(after_stats, st) != cudaSuccess) return SLA_ERR_CUDA;
    if (sla_stats || first_order) {
        // H (SLA) or the sum of the blocks' first-order matrices (PISA)
        constexpr int NHB = D * D / 256;
        Span sp(SLA_KERNEL_H_REDUCE, st);
        sla::h_reduce_kernel<D><<<dim3(NHB + 1, BH), 256, 0, st>>>(
            at<float>(ws, w.hpart), sla_stats ? at<float>(ws, w.zj) : nullptr, w.nchunk, Nk,
            at<float>(ws, w.hsum), at<float>(ws, w.zsum));
    }
    return launch_status();
}

template <int D, int MODE>
sla_status_t launch_attn(const sla_params_t* p, const void* q, const void* k, const void* v,
                         const float* alpha, const int32_t* lut, void* out, void* ws, const Ws& w,
                         cudaStream_t st) {
    using L = sla::AttnLayout<D, MODE>;
    constexpr bool PISA = L::PISA, FP8 = L::FP8;
    const int BH = p->B * p->H, Nq = p->N / p->Bq, Nk = p->N / p->Bk;
    sla::AttnMaps tm;
    std::memset(&tm, 0, sizeof tm);
    const long long rows = static_cast<long long>(BH) * p->N;
    constexpr auto F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    constexpr auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    (void)v;   // the P.V product reads the fp16 (or e4m3) copy of V made by the K/V pre-pass
    if (!make_map(&tm.out, out, rows, D, 64,
                  p->out_dtype == SLA_OUT_FP32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
        !make_map(&tm.q, q, rows, D, 128) ||
        !make_map(&tm.v, at<void>(ws, w.v16), rows, D, 64, F16))
        return SLA_ERR_CUDA;
    if (FP8) {
        if (!make_map(&tm.k, at<void>(ws, w.k8), rows, D, 64, U8) ||
            !make_map(&tm.q8, at<void>(ws, w.q8), rows, D, 128, U8) ||
            !make_map(&tm.v8t, at<void>(ws, w.v8t), static_cast<long long>(BH) * Nk * D, 64, D, U8, 64,
                      CU_TENSOR_MAP_SWIZZLE_64B))
            return SLA_ERR_CUDA;
    } else if (!make_map(&tm.k, k, rows, D, 64)) {
        return SLA_ERR_CUDA;
    }
    if (!PISA && !make_map(&tm.phi, at<void>(ws, w.phik16), rows, D, 64, F16)) return SLA_ERR_CUDA;
    if (PISA) {
        if (!make_map(&tm.kc, at<void>(ws, w.kc), static_cast<long long>(BH) * Nk, D, 64) ||
            !make_map(&tm.vc, at<void>(ws, w.vbar), static_cast<long long>(BH) * Nk, D, 64, F16))
            return SLA_ERR_CUDA;
    }
    sla::AttnArgs a{};
    a.N = p->N;
    a.Nq = Nq;
    a.Nk = Nk;
    a.Bq = p->Bq;
    // query blocks per CTA: 128 rows, except SLA with d = 128 (one block, so the
    // per-group G accumulator and Q, P fit in the 512 TMEM columns)
    a.GR = (!PISA && D == 128) ? 1 : 128 / p->Bq;
    a.topk = p->topk;
    a.tiles_per_head = (Nq + a.GR - 1) / a.GR;
    const float tau = p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt(static_cast<float>(D));
    a.scale_log2 = tau * 1.4426950408889634f;
    a.log2_bk = std::log2(static_cast<float>(p->Bk));
    a.lut = lut;
    a.alpha = alpha;
    a.hsum = PISA ? nullptr : at<float>(ws, w.hsum);
    a.zsum = PISA ? nullptr : at<float>(ws, w.zsum);
    a.zj = PISA ? nullptr : at<float>(ws, w.zj);
    a.out = out;
    a.out_f32 = p->out_dtype == SLA_OUT_FP32 ? 1 : 0;
    a.lut_sorted = p->lut_mode == SLA_LUT_COMPUTE ? 1 : 0;
    a.sq = FP8 ? at<float>(ws, w.sq) : nullptr;
    a.sk = FP8 ? at<float>(ws, w.sk) : nullptr;
    a.sv = FP8 ? at<float>(ws, w.sv) : nullptr;
    a.wait_ns = wait_limit_ns();
    a.debug_stall = debug_stall() ? 1 : 0;
    a.first_order = (PISA && p->pisa_first_order) ? 1 : 0;
    a.hbar = a.first_order ? at<float>(ws, w.hsum) : nullptr;
    a.fo_scale = tau / (static_cast<float>(Nk) * static_cast<float>(p->Bk));
    const int GR = a.GR;
    const int nwords = (Nk + 15) / 16;
    const int sched_cap = std::max(4, (std::min(Nk, GR * std::max(p->topk, 1)) + 3) & ~3);
    a.sched_cap = sched_cap;
    // misc region: barriers (384 B), zu [2][D], the three [2][128] exchange arrays,
    // the block mask, the schedule and (FP8) the per-entry scales
    const size_t smem = 1024 + L::OFF_MISC + 384 + 2 * D * 4 + 3 * 256 * 4 + ((nwords + 3) & ~3) * 4 +
                        static_cast<size_t>(sched_cap) * 4 * 3;
    if (smem > 232448) return SLA_ERR_UNSUPPORTED;   // LUT row too long for the shared-memory schedule
    auto kern = sla::attn_kernel<D, MODE>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return SLA_ERR_CUDA;
    Span sp(SLA_KERNEL_ATTN, st);
    kern<<<BH * a.tiles_per_head, sla::kAttnThreads, smem, st>>>(tm, a);
    return launch_status();
}

sla_status_t finish(sla_status_t s, cudaStream_t st) {
    if (s != SLA_OK) return s;
    if (check_after_call()) return sla_check_device_status(st);
    return SLA_OK;
}


// Argument checks of sla_forward and sla_pisa_forward, before anything is
// enqueued (also run by the host-buffer calls on the whole problem).
sla_status_t forward_args(const sla_params_t* p, const void* q, const void* k, const void* v, const float* alpha,
                          const float* w_q, const float* w_k, const int32_t* lut, const void* out,
                          void* workspace, size_t ws_bytes, Ws& w) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if (p->pisa_cov_lambda != 0.f) return SLA_ERR_INVALID_ARG;   // a PISA selection option
    if ((s = check_tensor(q, 16)) || (s = check_tensor(k, 16)) || (s = check_tensor(v, 16)) ||
        (s = check_tensor(out, 16)) || (s = check_tensor(alpha, 4)))
        return s;
    if ((w_q && !aligned(w_q, 4)) || (w_k && !aligned(w_k, 4))) return SLA_ERR_INVALID_ARG;
    if (p->lut_mode == SLA_LUT_GIVEN && !lut && p->topk > 0) return SLA_ERR_INVALID_ARG;
    if (lut && !aligned(lut, 4)) return SLA_ERR_INVALID_ARG;
    if (p->sparse_dtype != SLA_SPARSE_BF16 && (p->d != 128 || p->Bq != 128))
        return SLA_ERR_UNSUPPORTED;
    return check_ws(p, workspace, ws_bytes, w);
}

sla_status_t pisa_args(const sla_params_t* p, const void* q, const void* k, const void* v, const float* w_q,
                       const float* w_k, const int32_t* lut, const void* out, void* workspace, size_t ws_bytes,
                       Ws& w) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if ((s = check_tensor(q, 16)) || (s = check_tensor(k, 16)) || (s = check_tensor(v, 16)) ||
        (s = check_tensor(out, 16)))
        return s;
    if ((w_q && !aligned(w_q, 4)) || (w_k && !aligned(w_k, 4))) return SLA_ERR_INVALID_ARG;
    if (p->lut_mode == SLA_LUT_GIVEN && !lut && p->topk > 0) return SLA_ERR_INVALID_ARG;
    if (lut && !aligned(lut, 4)) return SLA_ERR_INVALID_ARG;
    if (p->Bq != p->Bk || p->sparse_dtype != SLA_SPARSE_BF16) return SLA_ERR_UNSUPPORTED;
    return check_ws(p, workspace, ws_bytes, w);
}

}  // namespace

extern "C" {

size_t sla_workspace_size(const sla_params_t* p) {
    if (check_params(p) != SLA_OK) return 0;
    return layout(p).total;
}

const char* sla_status_string(sla_status_t s) {
    switch (s) {
        case SLA_OK: return "ok";
        case SLA_ERR_INVALID_ARG: return "invalid argument";
        case SLA_ERR_UNSUPPORTED: return "unsupported shape or mode";
        case SLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case SLA_ERR_CUDA: return "CUDA call or kernel launch failed";
        case SLA_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
        case SLA_ERR_DEVICE_CHECK: return "a kernel found invalid data (LUT entry)";
    }
    return "unknown status";
}

int32_t sla_version(void) { return 200; }

sla_status_t sla_profile_enable(int32_t on) {
    Profiler& P = prof();
    std::lock_guard<std::mutex> g(P.mu);
    P.on = on != 0;
    return SLA_OK;
}

sla_status_t sla_profile_read(double* ms_total, int64_t* launches) {
    Profiler& P = prof();
    std::lock_guard<std::mutex> g(P.mu);
    sla_status_t rc = SLA_OK;
    for (int k = 0; k < SLA_KERNEL_KINDS; ++k) {
        if (ms_total) ms_total[k] = 0.0;
        if (launches) launches[k] = 0;
    }
    for (auto& r : P.recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            rc = SLA_ERR_CUDA;
        if (ms_total) ms_total[r.kind] += ms;
        if (launches) launches[r.kind] += 1;
        P.pool.push_back(r.a);
        P.pool.push_back(r.b);
    }
    P.recs.clear();
    return rc;
}

sla_status_t sla_check_device_status(sla_stream_t stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SLA_ERR_CUDA;
    unsigned v = 0u;
    if (cudaMemcpyFromSymbol(&v, sla::g_status, sizeof v) != cudaSuccess) return SLA_ERR_CUDA;
    if (v) {
        const unsigned zero = 0u;
        if (cudaMemcpyToSymbol(sla::g_status, &zero, sizeof zero) != cudaSuccess) return SLA_ERR_CUDA;
    }
    if (v & sla::kStatusTimeout) return SLA_ERR_TIMEOUT;
    if (v & (sla::kStatusBadData | sla::kStatusRange)) return SLA_ERR_DEVICE_CHECK;
    return SLA_OK;
}

sla_status_t sla_route(const sla_params_t* p, const void* q, const void* k, const float* w_q,
                       const float* w_k, int32_t* lut, void* workspace, size_t ws_bytes,
                       sla_stream_t stream) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if (p->pisa_cov_lambda != 0.f) return SLA_ERR_INVALID_ARG;   // a sla_pisa_forward option
    if ((s = check_tensor(q, 16)) || (s = check_tensor(k, 16))) return s;
    if (p->topk > 0 && (s = check_tensor(lut, 4))) return s;
    if ((w_q && !aligned(w_q, 4)) || (w_k && !aligned(w_k, 4))) return SLA_ERR_INVALID_ARG;
    Ws w;
    if ((s = check_ws(p, workspace, ws_bytes, w))) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return finish(run_router(p, q, k, w_q, w_k, lut, workspace, w, st), st);
}

// ------------------------------------------------------------- side stream
// The K/V pre-pass does not depend on the router's pooling of Q or on W folding, so
// a forward call runs it on a side stream of the library (one per device, created on
// first use) between a fork and two join points on the caller's stream: the router's
// score kernel waits for the pre-pass (it reads the pooled K means the pre-pass
// writes), the attention kernel also for h_reduce.  (Pooling K a second time on the
// caller's stream, so that the score could start before the pre-pass ends, was
// measured slower: the extra read of K competes with the pre-pass for HBM.)  The
// router's pooling and W folding are enqueued before the pre-pass, which fills the
// GPU, so that only the score waits for it.  The caller sees ordinary stream
// order.  The enqueue sequence of a call holds a
// per-device lock, so concurrent host threads never cross their events.  If the
// side stream cannot be created, everything runs on the caller's stream.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, kbar = nullptr, stats = nullptr;
    bool ok = false;
    std::mutex lock;
};

SideStream* side_stream() {
    static SideStream side[64];
    static std::mutex create;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    SideStream& x = side[dev];
    std::lock_guard<std::mutex> g(create);
    if (!x.ok) {
        if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        if (cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.kbar, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.stats, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        x.ok = true;
    }
    return &x;
}

sla_status_t sla_forward(const sla_params_t* p, const void* q, const void* k, const void* v,
                         const float* alpha, const float* w_q, const float* w_k, int32_t* lut,
                         void* out, void* workspace, size_t ws_bytes, sla_stream_t stream) {
    Ws w;
    sla_status_t s = forward_args(p, q, k, v, alpha, w_q, w_k, lut, out, workspace, ws_bytes, w);
    if (s != SLA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool compute = p->lut_mode == SLA_LUT_COMPUTE;
    // fp8: the 8-bit sparse branch (e4m3 P and V); int8: with integer Q and K codes
    const bool int8 = p->sparse_dtype == SLA_SPARSE_INT8;
    const bool fp8 = p->sparse_dtype == SLA_SPARSE_FP8_E4M3 || int8;
    int32_t* lut_use = (compute && !lut) ? at<int32_t>(workspace, w.lut) : lut;
    Phase pre(SLA_PHASE_PRE_ATTN, st);
    SideStream* side = side_stream();
    std::unique_lock<std::mutex> hold;
    cudaStream_t sst = st;                         // the pre-pass's stream
    if (side) {
        hold = std::unique_lock<std::mutex>(side->lock);
        if (cudaEventRecord(side->fork, st) != cudaSuccess) return SLA_ERR_CUDA;
    }
    // the router's pooling, W folding and projection go first, so that the
    // pre-pass, which fills the GPU, does not delay them (the score needs them
    // and the K means)
    if (compute && (s = router_pool(p, q, k, w_q, w_k, workspace, w, false, st))) return s;
    if (side) {
        if (cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess) return SLA_ERR_CUDA;
        sst = side->s;
    }
    s = p->d == 128 ? launch_kv<128>(p, k, v, workspace, w, compute, true, false, sst, fp8, false,
                                     side ? side->kbar : nullptr, int8)
                    : launch_kv<64>(p, k, v, workspace, w, compute, true, false, sst, false, false,
                                    side ? side->kbar : nullptr);
    if (s != SLA_OK) return s;
    if (fp8) {
        const long long nblk = static_cast<long long>(p->B) * p->H * p->N / 64;
        Span sp(SLA_KERNEL_QUANT_Q, sst);
        auto qk = int8 ? sla::quant_q_kernel<128, true> : sla::quant_q_kernel<128, false>;
        qk<<<grid_blocks(nblk, 8), 256, 0, sst>>>(static_cast<const __nv_bfloat16*>(q), nblk,
                                                  at<uint8_t>(workspace, w.q8), at<float>(workspace, w.sq));
        if (launch_status() != SLA_OK) return SLA_ERR_CUDA;
    }
    if (side && cudaEventRecord(side->stats, sst) != cudaSuccess) return SLA_ERR_CUDA;
    if (compute && (s = router_score(p, lut_use, workspace, w, st, side ? side->kbar : nullptr)))
        return s;
    if (side && cudaStreamWaitEvent(st, side->stats, 0) != cudaSuccess) return SLA_ERR_CUDA;
    pre.end();
    if (int8)
        s = launch_attn<128, sla::kModeSlaInt8>(p, q, k, v, alpha, lut_use, out, workspace, w, st);
    else if (fp8)
        s = launch_attn<128, sla::kModeSlaFp8>(p, q, k, v, alpha, lut_use, out, workspace, w, st);
    else
        s = p->d == 128 ? launch_attn<128, sla::kModeSla>(p, q, k, v, alpha, lut_use, out, workspace, w, st)
                        : launch_attn<64, sla::kModeSla>(p, q, k, v, alpha, lut_use, out, workspace, w, st);
    return finish(s, st);
}

sla_status_t sla_pisa_forward(const sla_params_t* p, const void* q, const void* k, const void* v,
                              const float* w_q, const float* w_k, int32_t* lut, void* out,
                              void* workspace, size_t ws_bytes, sla_stream_t stream) {
    Ws w;
    sla_status_t s = pisa_args(p, q, k, v, w_q, w_k, lut, out, workspace, ws_bytes, w);
    if (s != SLA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool compute = p->lut_mode == SLA_LUT_COMPUTE;
    int32_t* lut_use = (compute && !lut) ? at<int32_t>(workspace, w.lut) : lut;
    const bool fo = p->pisa_first_order != 0;
    Phase pre(SLA_PHASE_PRE_ATTN, st);
    SideStream* side = side_stream();
    std::unique_lock<std::mutex> hold;
    cudaStream_t sst = st;                         // the pre-pass's stream
    if (side) {
        hold = std::unique_lock<std::mutex>(side->lock);
        if (cudaEventRecord(side->fork, st) != cudaSuccess) return SLA_ERR_CUDA;
    }
    // the router's pooling, W folding and projection go first, so that the
    // pre-pass, which fills the GPU, does not delay them (the score needs them
    // and the K means)
    if (compute && (s = router_pool(p, q, k, w_q, w_k, workspace, w, false, st))) return s;
    if (side) {
        if (cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess) return SLA_ERR_CUDA;
        sst = side->s;
    }
    // covariance-aware selection: lambda M_j added to every score of block j; the
    // pre-pass forms the chunk sums of H_j on its way through K and V
    const bool cov = compute && p->pisa_cov_lambda > 0.f;
    s = p->d == 128 ? launch_kv<128>(p, k, v, workspace, w, compute, false, true, sst, false, fo,
                                     side ? side->kbar : nullptr, false, cov)
                    : launch_kv<64>(p, k, v, workspace, w, compute, false, true, sst, false, fo,
                                    side ? side->kbar : nullptr, false, cov);
    if (s != SLA_OK) return s;
    if (side && cudaEventRecord(side->stats, sst) != cudaSuccess) return SLA_ERR_CUDA;
    double* bias = cov ? at<double>(workspace, w.covbias) : nullptr;
    if (cov) {
        if (side && cudaStreamWaitEvent(st, side->kbar, 0) != cudaSuccess) return SLA_ERR_CUDA;
        if ((s = launch_cov(p, k, v, workspace, w, static_cast<double>(p->pisa_cov_lambda), bias, st)))
            return s;
    }
    if (compute && (s = router_score(p, lut_use, workspace, w, st, side ? side->kbar : nullptr, bias)))
        return s;
    if (side && cudaStreamWaitEvent(st, side->stats, 0) != cudaSuccess) return SLA_ERR_CUDA;
    pre.end();
    s = p->d == 128 ? launch_attn<128, sla::kModePisa>(p, q, k, v, nullptr, lut_use, out, workspace, w, st)
                    : launch_attn<64, sla::kModePisa>(p, q, k, v, nullptr, lut_use, out, workspace, w, st);
    return finish(s, st);
}

}  // extern "C"

// ------------------------------------------------- host-buffer forward calls
namespace {

// Two library streams per device (host-to-device and device-to-host copies) and
// their events, created on first use; a lock covers each call's enqueue sequence.
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t fork = nullptr, in = nullptr, done = nullptr, join = nullptr;
    bool ok = false;
    std::mutex lock;
};

HostPipe* host_pipe() {
    static HostPipe pipes[64];
    static std::mutex create;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    HostPipe& x = pipes[dev];
    std::lock_guard<std::mutex> g(create);
    if (!x.ok) {
        if (cudaStreamCreateWithFlags(&x.h2d, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&x.d2h, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.in, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.done, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        x.ok = true;
    }
    return &x;
}

// The (batch, head) problems of a call are independent and contiguous in every
// tensor, so heads [h0, h0 + n) are a call with B = 1, H = n at offset h0.  Each
// chunk's inputs are copied on the h2d stream; its forward runs on the caller's
// stream once they have landed; its output goes back on the d2h stream while
// later chunks arrive and compute.  fwd runs one chunk (device pointers).
template <typename Fwd>
sla_status_t run_host(const sla_params_t* p, const void* q_h, const void* k_h, const void* v_h,
                      const float* alpha_h, void* out_h, void* q, void* k, void* v, float* alpha, void* out,
                      int32_t* lut, int heads_per_chunk, cudaStream_t st, Fwd fwd) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if (!q_h || !k_h || !v_h || !out_h || !q || !k || !v || !out || (alpha_h && !alpha) || heads_per_chunk < 0)
        return SLA_ERR_INVALID_ARG;
    const long long BH = static_cast<long long>(p->B) * p->H;
    const size_t tok = static_cast<size_t>(p->N);
    const size_t qkv_head = tok * p->d * 2;
    const size_t out_head = tok * p->d * (p->out_dtype == SLA_OUT_FP32 ? 4 : 2);
    const size_t lut_head = static_cast<size_t>(p->N / p->Bq) * p->topk;
    const long long hc = heads_per_chunk > 0 ? heads_per_chunk : std::max<long long>(1, (BH + 7) / 8);
    HostPipe* hp = host_pipe();
    if (!hp) return SLA_ERR_CUDA;
    std::lock_guard<std::mutex> g(hp->lock);
    if (cudaEventRecord(hp->fork, st) != cudaSuccess || cudaStreamWaitEvent(hp->h2d, hp->fork, 0) != cudaSuccess)
        return SLA_ERR_CUDA;
    auto off = [](const void* b, size_t bytes) { return static_cast<const char*>(b) + bytes; };
    auto offw = [](void* b, size_t bytes) { return static_cast<char*>(b) + bytes; };
    for (long long h0 = 0; h0 < BH; h0 += hc) {
        const long long n = std::min(hc, BH - h0);
        const size_t o = static_cast<size_t>(h0) * qkv_head, nb = static_cast<size_t>(n) * qkv_head;
        if (cudaMemcpyAsync(offw(q, o), off(q_h, o), nb, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
            cudaMemcpyAsync(offw(k, o), off(k_h, o), nb, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess ||
            cudaMemcpyAsync(offw(v, o), off(v_h, o), nb, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess)
            return SLA_ERR_CUDA;
        if (alpha_h && cudaMemcpyAsync(alpha + h0 * static_cast<long long>(tok), alpha_h + h0 * static_cast<long long>(tok),
                                       static_cast<size_t>(n) * tok * 4, cudaMemcpyHostToDevice, hp->h2d) != cudaSuccess)
            return SLA_ERR_CUDA;
        if (cudaEventRecord(hp->in, hp->h2d) != cudaSuccess || cudaStreamWaitEvent(st, hp->in, 0) != cudaSuccess)
            return SLA_ERR_CUDA;
        sla_params_t pc = *p;
        pc.B = 1;
        pc.H = static_cast<int32_t>(n);
        s = fwd(&pc, offw(q, o), offw(k, o), offw(v, o), alpha ? alpha + h0 * static_cast<long long>(tok) : nullptr,
                lut ? lut + h0 * static_cast<long long>(lut_head) : nullptr,
                offw(out, static_cast<size_t>(h0) * out_head));
        if (s != SLA_OK) return s;
        if (cudaEventRecord(hp->done, st) != cudaSuccess || cudaStreamWaitEvent(hp->d2h, hp->done, 0) != cudaSuccess ||
            cudaMemcpyAsync(offw(out_h, static_cast<size_t>(h0) * out_head), off(out, static_cast<size_t>(h0) * out_head),
                            static_cast<size_t>(n) * out_head, cudaMemcpyDeviceToHost, hp->d2h) != cudaSuccess)
            return SLA_ERR_CUDA;
    }
    if (cudaEventRecord(hp->join, hp->d2h) != cudaSuccess || cudaStreamWaitEvent(st, hp->join, 0) != cudaSuccess)
        return SLA_ERR_CUDA;
    return SLA_OK;
}

}  // namespace

extern "C" {

sla_status_t sla_forward_host(const sla_params_t* p, const void* q_h, const void* k_h, const void* v_h,
                              const float* alpha_h, void* out_h, void* q, void* k, void* v, float* alpha,
                              void* out, const float* w_q, const float* w_k, int32_t* lut,
                              int32_t heads_per_chunk, void* workspace, size_t ws_bytes, sla_stream_t stream) {
    Ws w;
    sla_status_t s = forward_args(p, q, k, v, alpha, w_q, w_k, lut, out, workspace, ws_bytes, w);
    if (s != SLA_OK) return s;
    if (!alpha_h) return SLA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return run_host(p, q_h, k_h, v_h, alpha_h, out_h, q, k, v, alpha, out, lut, heads_per_chunk, st,
                    [&](const sla_params_t* pc, void* qc, void* kc, void* vc, float* ac, int32_t* lc, void* oc) {
                        return sla_forward(pc, qc, kc, vc, ac, w_q, w_k, lc, oc, workspace, ws_bytes, stream);
                    });
}

sla_status_t sla_pisa_forward_host(const sla_params_t* p, const void* q_h, const void* k_h, const void* v_h,
                                   void* out_h, void* q, void* k, void* v, void* out, const float* w_q,
                                   const float* w_k, int32_t* lut, int32_t heads_per_chunk, void* workspace,
                                   size_t ws_bytes, sla_stream_t stream) {
    Ws w;
    sla_status_t s = pisa_args(p, q, k, v, w_q, w_k, lut, out, workspace, ws_bytes, w);
    if (s != SLA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return run_host(p, q_h, k_h, v_h, nullptr, out_h, q, k, v, nullptr, out, lut, heads_per_chunk, st,
                    [&](const sla_params_t* pc, void* qc, void* kc, void* vc, float*, int32_t* lc, void* oc) {
                        return sla_pisa_forward(pc, qc, kc, vc, w_q, w_k, lc, oc, workspace, ws_bytes, stream);
                    });
}

sla_status_t sla_pisa_cov_norms(const sla_params_t* p, const void* k, const void* v, double* norms,
                                void* workspace, size_t ws_bytes, sla_stream_t stream) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if ((s = check_tensor(k, 16)) || (s = check_tensor(v, 16))) return s;
    if (!norms || !aligned(norms, 8)) return SLA_ERR_INVALID_ARG;
    if (!(p->pisa_cov_lambda > 0.f)) return SLA_ERR_INVALID_ARG;   // the workspace holds the scratch then
    Ws w;
    if ((s = check_ws(p, workspace, ws_bytes, w))) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the chunk sums of H_j from the K/V pre-pass's exact product, then the norms
    s = p->d == 128 ? launch_kv<128>(p, k, v, workspace, w, false, false, false, st, false, false, nullptr,
                                     false, true)
                    : launch_kv<64>(p, k, v, workspace, w, false, false, false, st, false, false, nullptr,
                                    false, true);
    if (s != SLA_OK) return s;
    return finish(launch_cov(p, k, v, workspace, w, 1.0, norms, st), st);
}

}  // extern "C"

// ------------------------------------------------------------ co-clustering
namespace {

struct CcWs {
    size_t qc, kc, qv, kv, label, counts, base, start, count, total;
    int nchunk;
};

CcWs cc_layout(const sla_params_t* p, int C) {
    CcWs w{};
    const size_t BH = static_cast<size_t>(p->B) * p->H, d = p->d, N = p->N;
    w.nchunk = static_cast<int>((N + sla::kCcChunk - 1) / sla::kCcChunk);
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.qc = take(BH * C * d * 8);
    w.kc = take(BH * C * d * 8);
    w.qv = take(BH * C * 4);
    w.kv = take(BH * C * 4);
    w.label = take(BH * N * 4);
    w.counts = take(BH * static_cast<size_t>(w.nchunk) * C * 4);
    w.base = take(BH * static_cast<size_t>(w.nchunk) * C * 4);
    w.start = take(BH * C * 4);
    w.count = take(BH * C * 4);
    w.total = off;
    return w;
}

sla_status_t cc_check(const sla_params_t* p, int C, int iters) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if (C < 1 || iters < 1 || iters > 64 || p->N % C != 0) return SLA_ERR_INVALID_ARG;
    if (C > 1024) return SLA_ERR_UNSUPPORTED;
    return SLA_OK;
}

// labels -> stable order by label -> centroids, for one half-step
template <int D>
sla_status_t cc_sort_means(const sla_params_t* p, int C, const __nv_bfloat16* x, void* ws, const CcWs& w,
                           int32_t* perm, double* cent, int* valid, cudaStream_t st) {
    const int BH = p->B * p->H, N = p->N;
    int* label = at<int>(ws, w.label);
    {
        Span sp(SLA_KERNEL_COCLUSTER, st);
        sla::cc_count_kernel<<<dim3(w.nchunk, BH), 256, C * 4, st>>>(label, N, C, w.nchunk, at<int>(ws, w.counts));
    }
    {
        Span sp(SLA_KERNEL_COCLUSTER, st);
        sla::cc_scan_kernel<<<BH, 1024, 0, st>>>(at<int>(ws, w.counts), C, w.nchunk, at<int>(ws, w.base),
                                                 at<int>(ws, w.start), at<int>(ws, w.count));
    }
    {
        Span sp(SLA_KERNEL_COCLUSTER, st);
        sla::cc_scatter_kernel<<<dim3(w.nchunk, BH), 32, C * 4, st>>>(label, N, C, w.nchunk, at<int>(ws, w.base),
                                                                      perm);
    }
    {
        Span sp(SLA_KERNEL_COCLUSTER, st);
        sla::cc_means_kernel<D><<<dim3(C, BH), sla::kCcMeanThreads, 0, st>>>(x, N, C, perm, at<int>(ws, w.start),
                                                           at<int>(ws, w.count), cent, valid);
    }
    return launch_status();
}

template <int D>
sla_status_t run_cocluster(const sla_params_t* p, int C, int iters, const void* q, const void* k, int32_t* q_perm,
                           int32_t* k_perm, void* ws, const CcWs& w, cudaStream_t st) {
    const int BH = p->B * p->H, N = p->N;
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    double* qc = at<double>(ws, w.qc);
    double* kc = at<double>(ws, w.kc);
    int* qv = at<int>(ws, w.qv);
    int* kv = at<int>(ws, w.kv);
    int* label = at<int>(ws, w.label);
    auto assign = sla::cc_assign_kernel<D>;
    constexpr size_t asmem = sla::cc_assign_smem<D>();
    if (cudaFuncSetAttribute(assign, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(asmem)) !=
        cudaSuccess)
        return SLA_ERR_CUDA;
    const dim3 agrid((N + sla::kCcTok - 1) / sla::kCcTok, BH);
    {
        Span sp(SLA_KERNEL_COCLUSTER, st);
        sla::cc_chunk_mean_kernel<D><<<dim3(C, BH), D, 0, st>>>(qb, N, C, qc, qv);
    }
    for (int it = 0; it < iters; ++it) {
        // keys guided by the query centroids, then queries by the updated key centroids
        {
            Span sp(SLA_KERNEL_COCLUSTER, st);
            assign<<<agrid, 128, asmem, st>>>(kb, N, C, qc, qv, label);
        }
        sla_status_t s = cc_sort_means<D>(p, C, kb, ws, w, k_perm, kc, kv, st);
        if (s != SLA_OK) return s;
        {
            Span sp(SLA_KERNEL_COCLUSTER, st);
            assign<<<agrid, 128, asmem, st>>>(qb, N, C, kc, kv, label);
        }
        s = cc_sort_means<D>(p, C, qb, ws, w, q_perm, qc, qv, st);
        if (s != SLA_OK) return s;
    }
    return launch_status();
}

}  // namespace

extern "C" size_t sla_cocluster_workspace_size(const sla_params_t* p, int32_t n_clusters) {
    if (cc_check(p, n_clusters, 1) != SLA_OK) return 0;
    return cc_layout(p, n_clusters).total;
}

extern "C" sla_status_t sla_cocluster(const sla_params_t* p, const void* q, const void* k, int32_t n_clusters,
                                      int32_t iters, int32_t* q_perm, int32_t* k_perm, void* workspace,
                                      size_t ws_bytes, sla_stream_t stream) {
    sla_status_t s = cc_check(p, n_clusters, iters);
    if (s != SLA_OK) return s;
    if ((s = check_tensor(q, 16)) || (s = check_tensor(k, 16)) || (s = check_tensor(q_perm, 4)) ||
        (s = check_tensor(k_perm, 4)))
        return s;
    const CcWs w = cc_layout(p, n_clusters);
    if (!workspace || !aligned(workspace, kAlign) || ws_bytes < w.total) return SLA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = p->d == 128 ? run_cocluster<128>(p, n_clusters, iters, q, k, q_perm, k_perm, workspace, w, st)
                    : run_cocluster<64>(p, n_clusters, iters, q, k, q_perm, k_perm, workspace, w, st);
    return finish(s, st);
}

extern "C" sla_status_t sla_permute_rows(const void* src, const int32_t* perm, void* dst, int64_t BH, int32_t N,
                                         int32_t row_bytes, int32_t inverse, sla_stream_t stream) {
    if (!src || !dst || !perm || src == dst || BH < 1 || N < 1 || BH * N > 0x7fffffffLL) return SLA_ERR_INVALID_ARG;
    if (row_bytes < 4 || row_bytes % 4 || row_bytes > 4096 || (inverse != 0 && inverse != 1))
        return SLA_ERR_INVALID_ARG;
    if (!aligned(perm, 4)) return SLA_ERR_INVALID_ARG;
    const bool vec = row_bytes % 16 == 0 && aligned(src, 16) && aligned(dst, 16);
    if (!vec && (!aligned(src, 4) || !aligned(dst, 4))) return SLA_ERR_INVALID_ARG;
    const int words = vec ? row_bytes / 16 : row_bytes / 4;
    if (words > 256) return SLA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long rows = BH * N;
    const int per_row = std::max(1, 256 / words);
    const int grid = grid_blocks((rows + per_row - 1) / per_row, 8);
    Span sp(SLA_KERNEL_PERMUTE, st);
    if (vec)
        sla::permute_rows_kernel<uint4><<<grid, 256, 0, st>>>(static_cast<const uint4*>(src), perm,
                                                             static_cast<uint4*>(dst), BH, N, words, inverse);
    else
        sla::permute_rows_kernel<uint32_t><<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src), perm,
                                                                static_cast<uint32_t*>(dst), BH, N, words, inverse);
    return finish(launch_status(), st);
}

// ------------------------------------------------------------ routing without allocation
// The scratch of sla_route_noalloc lives in this file-scope device array: the
// module's device memory, reserved on every GPU that loads the library and held
// until the process exits.  Host code only has a stand-in for the array's name,
// so its device address is looked up per device with cudaGetSymbolAddress.
namespace {

constexpr size_t kRouteScratchBytes = static_cast<size_t>(32) << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

struct RouteScratch {
    std::mutex mu;
    void* ptr[64] = {};
};

RouteScratch& route_scratch() {
    static RouteScratch r;
    return r;
}

// Device address of g_route_scratch on the current device.  Outside stream capture
// it is looked up on every call (so a context that was reset and re-created, with
// the module loaded again, never sees a stale address); under capture the address
// from the last uncaptured call on this device is used, and there must be one.
sla_status_t route_scratch_ptr(cudaStream_t st, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SLA_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return SLA_ERR_CUDA;
    RouteScratch& r = route_scratch();
    std::lock_guard<std::mutex> g(r.mu);
    if (cs == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return SLA_ERR_CUDA;
        r.ptr[dev] = p;
    } else if (!r.ptr[dev]) {
        return SLA_ERR_CUDA;        // first call on this device made under capture
    }
    *out = r.ptr[dev];
    return SLA_OK;
}

// Only the router's three scratch regions: pooled Q, pooled K (transposed), W_q W_k^T.
Ws route_layout(const sla_params_t* p) {
    Ws w{};
    const size_t BH = static_cast<size_t>(p->B) * p->H;
    const size_t d = p->d, Nq = p->N / p->Bq, Nk = p->N / p->Bk;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.qbar = take(BH * Nq * d * 8);
    w.kbarT = take(BH * Nk * d * 8);
    w.m = take(d * d * 8);
    w.total = off;
    return w;
}

}  // namespace

extern "C" sla_status_t sla_route_noalloc(const sla_params_t* p, const void* q, const void* k,
                                          const float* w_q, const float* w_k, int32_t* lut,
                                          sla_stream_t stream) {
    sla_status_t s = check_params(p);
    if (s != SLA_OK) return s;
    if (p->pisa_cov_lambda != 0.f) return SLA_ERR_INVALID_ARG;   // a sla_pisa_forward option
    if ((s = check_tensor(q, 16)) || (s = check_tensor(k, 16))) return s;
    if (p->topk > 0 && (s = check_tensor(lut, 4))) return s;
    if ((w_q && !aligned(w_q, 4)) || (w_k && !aligned(w_k, 4))) return SLA_ERR_INVALID_ARG;
    const Ws w = route_layout(p);
    if (w.total > kRouteScratchBytes) return SLA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* scratch = nullptr;
    if ((s = route_scratch_ptr(st, &scratch))) return s;
    return finish(run_router(p, q, k, w_q, w_k, lut, scratch, w, st), st);
}

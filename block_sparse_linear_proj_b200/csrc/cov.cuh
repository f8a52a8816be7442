// cov.cuh -- PISA covariance-aware routing ("Routing Consapevole della
// Covarianza", PISA page sec. 2): the norm M_j = ||H_j - Hbar||_2 of each KV
// block's first-order matrix about the mean of those matrices, which the
// router adds (times a caller-set weight) to every score of block j.
//   H_j = sum_{n in j} (k_n - kbar_j)^T v_n,   Hbar = (1/Nk) sum_j H_j,
// and ||.||_2 is the largest singular value.
//
// cov_hsum_kernel: per chunk of blocks, the sum of their H_j (fp32).  The keys
// are centred in fp64 and rounded once to fp32, so every product with a bf16
// value is exact in fp32 and only the 64-term sums round.
// cov_hbar_kernel: Hbar, the chunk sums added in order in fp64.
// cov_norm_kernel: per block, A = H_j - Hbar (the same fp32 H_j) in shared
// memory, then kLanczos Lanczos steps on A^T A (products A q and A^T y, full
// re-orthogonalisation by classical Gram-Schmidt applied twice) and the largest
// eigenvalue of the tridiagonal matrix by bisection on its Sturm sequence in
// fp64; M_j is its square root.  (Lanczos: the Ritz values of a Krylov space
// approach the extreme eigenvalues; Sturm: the number of negative pivots of
// T - x I counts the eigenvalues below x.)
// Every wait is a __syncthreads; there is no spin-wait.
#pragma once
#include "common.cuh"

namespace sla {

constexpr int kCovTok = 64;       // tokens per KV block
constexpr int kLanczos = 24;      // Lanczos steps (at most)

// Shared layout of one block: ks [64][D] fp32 centred keys, vs [64][D] fp32
// values, kmean [D] fp64.  Loads block (K, V rows given) and centres the keys.
template <int D>
__device__ __forceinline__ void cov_load_block(const __nv_bfloat16* __restrict__ kblk,
                                               const __nv_bfloat16* __restrict__ vblk, float* ks,
                                               float* vs, double* kmean) {
    const int tid = threadIdx.x;
    constexpr int CPR = D / 8;                         // 16-byte chunks per row
    for (int q = tid; q < kCovTok * CPR; q += 256) {
        const int n = q / CPR, u = q % CPR;
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(kblk + n * D + u * 8));
        const uint4 y = __ldg(reinterpret_cast<const uint4*>(vblk + n * D + u * 8));
        float4* kd = reinterpret_cast<float4*>(ks + n * D + u * 8);
        float4* vd = reinterpret_cast<float4*>(vs + n * D + u * 8);
        kd[0] = make_float4(bf16lo(x.x), bf16hi(x.x), bf16lo(x.y), bf16hi(x.y));
        kd[1] = make_float4(bf16lo(x.z), bf16hi(x.z), bf16lo(x.w), bf16hi(x.w));
        vd[0] = make_float4(bf16lo(y.x), bf16hi(y.x), bf16lo(y.y), bf16hi(y.y));
        vd[1] = make_float4(bf16lo(y.z), bf16hi(y.z), bf16lo(y.w), bf16hi(y.w));
    }
    __syncthreads();
    if (tid < D) {
        double s = 0.0;
        for (int n = 0; n < kCovTok; ++n) s += static_cast<double>(ks[n * D + tid]);
        kmean[tid] = s * (1.0 / kCovTok);
    }
    __syncthreads();
    for (int q = tid; q < kCovTok * D; q += 256)
        ks[q] = static_cast<float>(static_cast<double>(ks[q]) - kmean[q % D]);
    __syncthreads();
}

// acc[i][j] += sum_n ks[n][ty RT + i] vs[n][tx RT + j]: thread (ty, tx) =
// (tid / 16, tid % 16) owns an RT x RT tile of the D x D matrix, RT = D / 16.
template <int D>
__device__ __forceinline__ void cov_accumulate(const float* ks, const float* vs,
                                               float (&acc)[D / 16][D / 16]) {
    constexpr int RT = D / 16;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
#pragma unroll 4
    for (int n = 0; n < kCovTok; ++n) {
        float a[RT], b[RT];
#pragma unroll
        for (int i = 0; i < RT; i += 4) {
            const float4 x = *reinterpret_cast<const float4*>(ks + n * D + ty * RT + i);
            const float4 y = *reinterpret_cast<const float4*>(vs + n * D + tx * RT + i);
            a[i] = x.x; a[i + 1] = x.y; a[i + 2] = x.z; a[i + 3] = x.w;
            b[i] = y.x; b[i + 1] = y.y; b[i + 2] = y.z; b[i + 3] = y.w;
        }
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int j = 0; j < RT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

// grid (nchunk, BH), 256 threads; part [BH][nchunk][D][D] fp32 (empty chunks: zeros).
template <int D>
__global__ void __launch_bounds__(256) cov_hsum_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v, int N,
                                                       int Nk, int bpc, int nchunk,
                                                       float* __restrict__ part) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    float* ks = reinterpret_cast<float*>(smem_raw);
    float* vs = ks + kCovTok * D;
    double* kmean = reinterpret_cast<double*>(vs + kCovTok * D);
    constexpr int RT = D / 16;
    const long long bh = blockIdx.y;
    const int chunk = blockIdx.x;
    const int jb0 = chunk * bpc;
    const int nb = min(bpc, Nk - jb0);
    float acc[RT][RT];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RT; ++j) acc[i][j] = 0.f;
    for (int b = 0; b < nb; ++b) {
        const long long row0 = (bh * N + static_cast<long long>(jb0 + b) * kCovTok) * D;
        cov_load_block<D>(k + row0, v + row0, ks, vs, kmean);
        cov_accumulate<D>(ks, vs, acc);
        __syncthreads();                               // before the next block's load
    }
    float* dst = part + (bh * nchunk + chunk) * static_cast<long long>(D) * D;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RT; j += 4)
            *reinterpret_cast<float4*>(dst + (ty * RT + i) * D + tx * RT + j) =
                make_float4(acc[i][j], acc[i][j + 1], acc[i][j + 2], acc[i][j + 3]);
}

// grid (D*D/256, BH), 256 threads: hbar[bh] = (sum over chunks of part) / Nk.
template <int D>
__global__ void __launch_bounds__(256) cov_hbar_kernel(const float* __restrict__ part, int nchunk,
                                                       int Nk, float* __restrict__ hbar) {
    const long long bh = blockIdx.y;
    const int idx = blockIdx.x * 256 + threadIdx.x;
    const float* src = part + bh * nchunk * static_cast<long long>(D) * D + idx;
    double s = 0.0;
    for (int c = 0; c < nchunk; ++c) s += static_cast<double>(src[static_cast<long long>(c) * D * D]);
    hbar[bh * D * D + idx] = static_cast<float>(s / static_cast<double>(Nk));
}

// Sum of one value per thread over the CTA (fixed order); every thread gets it.
// red: [8] floats of shared memory; two __syncthreads.
__device__ __forceinline__ float cov_block_sum(float x, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w];
    __syncthreads();
    return s;
}

// grid (Nk, BH), 256 threads.  out[bh * Nk + j] = scale * M_j (fp64).
template <int D>
__global__ void __launch_bounds__(256, 2) cov_norm_kernel(const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          int N, int Nk,
                                                          const float* __restrict__ hbar,
                                                          double scale, double* __restrict__ out) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr int RT = D / 16, LDA = D + 1;
    constexpr int R0 = (2 * kCovTok * D > D * LDA ? 2 * kCovTok * D : D * LDA);   // floats
    float* ks = reinterpret_cast<float*>(smem_raw);          // block tiles, then A
    float* vs = ks + kCovTok * D;
    float* am = ks;                                          // A [D][D + 1]
    double* kmean = reinterpret_cast<double*>(ks + R0);      // [D]
    float* qv = reinterpret_cast<float*>(kmean + D);         // Lanczos vectors [kLanczos + 1][D]
    float* yv = qv + (kLanczos + 1) * D;                     // [D]
    float* red = yv + D;                                     // [(kLanczos + 1) * 8]
    float* coef = red + (kLanczos + 1) * 8;                  // [kLanczos + 1]
    double* alpha = reinterpret_cast<double*>(
        (reinterpret_cast<uintptr_t>(coef + kLanczos + 1) + 7) & ~static_cast<uintptr_t>(7));  // [kLanczos]
    double* beta = alpha + kLanczos;                                  // [kLanczos]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long bh = blockIdx.y;
    const int j = blockIdx.x;
    const long long row0 = (bh * N + static_cast<long long>(j) * kCovTok) * D;

    // 1. H_j, then A = H_j - Hbar over the tiles (shared memory reused)
    cov_load_block<D>(k + row0, v + row0, ks, vs, kmean);
    float acc[RT][RT];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int jj = 0; jj < RT; ++jj) acc[i][jj] = 0.f;
    cov_accumulate<D>(ks, vs, acc);
    __syncthreads();
    {
        const int ty = tid / 16, tx = tid % 16;
        const float* hb = hbar + bh * D * D;
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int jj = 0; jj < RT; ++jj) {
                const int r = ty * RT + i, c = tx * RT + jj;
                am[r * LDA + c] = acc[i][jj] - hb[r * D + c];
            }
    }
    // 2. Lanczos on B = A^T A from q_0 proportional to (1 + t / D)
    const bool own = tid < D;                                 // thread t holds element t
    const float x0 = own ? 1.f + static_cast<float>(tid) / D : 0.f;
    const float n0 = cov_block_sum(x0 * x0, red);            // (also orders the writes of A)
    if (own) qv[tid] = x0 / sqrtf(n0);
    __syncthreads();
    int m = 0;
    float b_prev = 0.f, a_max = 0.f;      // (every thread holds the same sums)
    for (int it = 0; it < kLanczos; ++it) {
        const float* q = qv + it * D;
        if (own) {                                            // y = A q
            float s = 0.f;
            for (int c = 0; c < D; ++c) s = fmaf(am[tid * LDA + c], q[c], s);
            yv[tid] = s;
        }
        __syncthreads();
        float w = 0.f;
        if (own) {                                            // w = A^T y - beta q_prev
            float s = 0.f;
            for (int r = 0; r < D; ++r) s = fmaf(am[r * LDA + tid], yv[r], s);
            w = s - (it > 0 ? b_prev * qv[(it - 1) * D + tid] : 0.f);
        }
        const float al = cov_block_sum(own ? w * q[tid] : 0.f, red);
        if (own) w -= al * q[tid];
        // full re-orthogonalisation against q_0 .. q_it, twice
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            for (int i = 0; i <= it; ++i) {
                float p = own ? w * qv[i * D + tid] : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
                if (lane == 0) red[i * 8 + warp] = p;
            }
            __syncthreads();
            if (tid <= it) {
                float s = 0.f;
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8) s += red[tid * 8 + w8];
                coef[tid] = s;
            }
            __syncthreads();
            if (own)
                for (int i = 0; i <= it; ++i) w -= coef[i] * qv[i * D + tid];
        }
        const float bsq = cov_block_sum(own ? w * w : 0.f, red);
        const float be = sqrtf(bsq);
        if (tid == 0) {
            alpha[it] = static_cast<double>(al);
            beta[it] = static_cast<double>(be);
        }
        m = it + 1;
        a_max = fmaxf(a_max, fabsf(al));
        // an invariant subspace (or A = 0): the tridiagonal matrix is complete
        // (al, be and a_max are CTA-wide sums, so every thread takes the same exit)
        if (!(be > 1e-7f * a_max + 1e-30f)) break;
        if (own) qv[(it + 1) * D + tid] = w / be;
        b_prev = be;
        __syncthreads();
    }
    __syncthreads();
    // 3. the largest eigenvalue of T (m x m) by bisection; M_j = sqrt of it
    if (tid == 0) {
        double hi = 0.0;
        for (int i = 0; i < m; ++i) {
            const double g = fabs(alpha[i]) + (i > 0 ? fabs(beta[i - 1]) : 0.0) +
                             (i + 1 < m ? fabs(beta[i]) : 0.0);
            hi = fmax(hi, g);
        }
        double lo = 0.0;
        for (int s = 0; s < 200 && hi - lo > 1e-15 * hi; ++s) {
            const double x = 0.5 * (lo + hi);
            int below = 0;                                  // eigenvalues of T below x
            double d = alpha[0] - x;
            if (d < 0.0) ++below;
            for (int i = 1; i < m; ++i) {
                const double dd = d != 0.0 ? d : 1e-300;
                d = alpha[i] - x - beta[i - 1] * beta[i - 1] / dd;
                if (d < 0.0) ++below;
            }
            if (below == m) hi = x; else lo = x;
        }
        out[bh * Nk + j] = scale * sqrt(fmax(hi, 0.0));
    }
}

}  // namespace sla

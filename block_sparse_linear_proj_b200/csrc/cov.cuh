// cov.cuh -- PISA covariance-aware routing ("Routing Consapevole della
// Covarianza", PISA page sec. 2): the norm M_j = ||H_j - Hbar||_2 of each KV
// block's first-order matrix about the mean of those matrices, which the
// router adds (times a caller-set weight) to every score of block j.
//   H_j = sum_{n in j} (k_n - kbar_j)^T v_n,   Hbar = (1/Nk) sum_j H_j,
// and ||.||_2 is the largest singular value.
//
// The chunk sums of the H_j come from the K/V pre-pass (kv_stats_kernel, its
// exact mode): keys centred in fp64 by the block's column means, rounded once to
// fp32 and split exactly into three bf16 parts, so every product with a bf16
// value is exact in fp32; the tensor core accumulates them in fp32.
// cov_hbar_kernel: Hbar, the chunk sums added in order in fp64.
// cov_norm_kernel: per block, H_j again on the tensor core (the same centring,
// split and products), A = H_j - Hbar as the threads' register tiles, then
// kLanczos Lanczos steps on A^T A (products A q and A^T y from the tiles; full
// re-orthogonalisation by classical Gram-Schmidt); writes the tridiagonal matrix
// T of the steps.  (Lanczos: the Ritz values of a Krylov space approach the
// extreme eigenvalues.)
// cov_eig_kernel: per block, the largest eigenvalue of T by multisection on its
// Sturm sequence in fp64 (the sign changes of the leading minors of T - x I
// count the eigenvalues below x), one warp per block; M_j is its square root.
// Every wait is a __syncthreads, a __syncwarp or the bounded wait on the product.
#pragma once
#include "common.cuh"
#include "kv_stats.cuh"

namespace sla {

constexpr int kCovTok = 64;       // tokens per KV block
constexpr int kLanczos = 24;      // Lanczos steps (at most)
constexpr int kQRows = 28;        // Lanczos vector rows kept: kLanczos + 1, padded to 4 with zeros
constexpr int kTriStride = 2 * kLanczos + 1;   // fp64 words per block of the tridiagonal output

// Tile layout of a D x D matrix over 256 threads: thread (ty, tx) = (tid / 16,
// tid % 16) owns rows cov_idx(ty, i) and columns cov_idx(tx, jj), i, jj < RT =
// D / 16, where cov_idx(t, i) = 64 (i / 4) + 4 t + i % 4 -- runs of four, 64
// apart, so that a half-warp's 16-byte reads of a row cover 256 contiguous bytes.
__device__ __forceinline__ int cov_idx(int t, int i) { return (i >> 2) * 64 + t * 4 + (i & 3); }

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

// The sums over the warp's 32 lanes of R partial values per lane (R a power of
// two, 1 < R <= 32), reduce-scattered: each step swaps half of the remaining
// values with the lane 16, 8, ... apart and keeps the sums of the other half, so
// after log2 R steps lane l holds the sum, over the lanes that agree with l in
// bits log2(32 / R) and up, of row l / (32 / R); the lanes below finish it with
// plain shuffles.  Every lane returns the full sum of its row.
template <int R>
__device__ __forceinline__ float cov_warp_rows(float (&p)[R], int lane) {
#pragma unroll
    for (int n = R, o = 16; n > 1; n >>= 1, o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? p[i] : p[i + n / 2];
            const float keep = up ? p[i + n / 2] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float s = p[0];
#pragma unroll
    for (int o = 16 / R; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// The sums over each half-warp's 16 lanes of RT partial values per lane (RT = 4
// or 8): a reduce-scatter within the half (offsets 8, 4, ...) leaves value i's
// sum on lane i * 16 / RT of the half, from where every lane of the half
// gathers all RT sums into out.
template <int RT>
__device__ __forceinline__ void cov_half_rows(float (&p)[RT], int lane, float (&out)[RT]) {
#pragma unroll
    for (int n = RT, o = 8; n > 1; n >>= 1, o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? p[i] : p[i + n / 2];
            const float keep = up ? p[i + n / 2] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float s = p[0];
#pragma unroll
    for (int o = 8 / RT; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
    for (int i = 0; i < RT; ++i) out[i] = __shfl_sync(0xffffffffu, s, (lane & 16) | (i * (16 / RT)));
}

// grid (Nk, BH), 256 threads.  tri[(bh * Nk + j) * kTriStride ..]: the Lanczos
// tridiagonal matrix T of block j -- alpha_0 .. alpha_{m-1}, beta_0 .. beta_{m-2}
// (beta_{m-1} and the unused entries are zero) and m, all fp64.
// H_j runs on tcgen05: the block's K and V rows land (cp.async) in the operand
// layout of the K/V pre-pass (64-column halves, 128-byte swizzle), the keys are
// centred by fp64 column means, rounded once to fp32 and split exactly into three
// bf16 parts (split3_bf16), and one thread issues the twelve M = 128, K = 16
// products of the parts with V into a D-column fp32 accumulator in tensor memory.
// The accumulator passes through shared memory (rows of 16-byte chunks XOR-
// swizzled by the row) into each thread's register tile.  The product waits on
// one mbarrier, bounded (wait_ns): on expiry the status word is set and the block
// continues on a zero matrix.
template <int D>
__global__ void __launch_bounds__(256, 2) cov_norm_kernel(const __nv_bfloat16* __restrict__ k,
                                                          const __nv_bfloat16* __restrict__ v,
                                                          int N, int Nk,
                                                          const float* __restrict__ hbar,
                                                          double* __restrict__ tri,
                                                          unsigned long long wait_ns) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr int RT = D / 16;
    constexpr int TILE = kCovTok * D * 2;                    // one bf16 operand tile
    // the swizzled tiles need a 1024-byte aligned base (the launch adds 1024 bytes)
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* tK = base;                                // K, then the parts' hi
    unsigned char* tV = base + TILE;                         // V (the B operand)
    unsigned char* tM = base + 2 * TILE;                     // mid parts
    unsigned char* tL = base + 3 * TILE;                     // lo parts
    float* hs = reinterpret_cast<float*>(base);              // then H_j [D][D], after the product
    double* kmean = reinterpret_cast<double*>(base + 4 * TILE);   // [D]
    double* kpart = kmean + D;                               // [8][D]
    float* qv = reinterpret_cast<float*>(kpart + 8 * D);     // Lanczos vectors [kQRows][D]
    float* wv = qv + kQRows * D;                             // [D] w before re-orthogonalisation
    float* wraw = wv + D;                                    // [D] w after it, not yet normalised
    float* part = wraw + D;                                  // [8][D] per-warp sums of A^T y
    float* red = part + 8 * D;                               // [16]
    float* coef = red + 16;                                  // [32]
    double* alpha = reinterpret_cast<double*>(
        (reinterpret_cast<uintptr_t>(coef + 32) + 7) & ~static_cast<uintptr_t>(7));  // [kLanczos]
    double* beta = alpha + kLanczos;                                  // [kLanczos]
    uint64_t* mma_bar = reinterpret_cast<uint64_t*>(beta + kLanczos);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ty = tid / 16, tx = tid % 16, half = (lane >> 4) & 1;
    const long long bh = blockIdx.y;
    const int j = blockIdx.x;
    const long long row0 = (bh * N + static_cast<long long>(j) * kCovTok) * D;

    // 1. H_j on the tensor core, then A = H_j - Hbar as this thread's RT x RT tile
    if (warp == 0) {
        tmem_alloc(tmem_slot, D);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    {
        constexpr int CPR = D / 8;                           // 16-byte chunks per row
        for (int q = tid; q < kCovTok * CPR; q += 256) {
            const int n = q / CPR, u = q % CPR;
            const uint32_t off = kv_off<D, true>(n, u * 8);
            cp_async16(tK + off, k + row0 + n * D + u * 8);
            cp_async16(tV + off, v + row0 + n * D + u * 8);
        }
        cp_async_commit();
        cp_async_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    {                                                         // fp64 column means of the keys
        constexpr int HALVES = 256 / D, RPH = kCovTok / HALVES;
        const int col = tid % D, hf = tid / D;
        double sm = 0.0;
        for (int n = hf * RPH; n < (hf + 1) * RPH; ++n)
            sm += static_cast<double>(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tK + kv_off<D, true>(n, col))));
        kpart[tid] = sm;
        __syncthreads();
        if (tid < D) {
            double t = kpart[tid];
#pragma unroll
            for (int h = 1; h < HALVES; ++h) t += kpart[h * D + tid];
            kmean[tid] = t * (1.0 / kCovTok);
        }
        __syncthreads();
    }
    {                                                         // the keys' three bf16 parts
        constexpr int CPR = D / 8;
        for (int q = tid; q < kCovTok * CPR; q += 256) {
            const int n = q / CPR, u = q % CPR;
            const uint32_t off = kv_off<D, true>(n, u * 8);
            const uint4 x = *reinterpret_cast<const uint4*>(tK + off);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            uint32_t wh[4], wm[4], wl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float h0, m0, l0, h1, m1, l1;
                split3_bf16(static_cast<float>(static_cast<double>(bf16lo(w[e])) - kmean[u * 8 + 2 * e]), h0, m0, l0);
                split3_bf16(static_cast<float>(static_cast<double>(bf16hi(w[e])) - kmean[u * 8 + 2 * e + 1]), h1, m1, l1);
                wh[e] = pack_bf16(h0, h1);
                wm[e] = pack_bf16(m0, m1);
                wl[e] = pack_bf16(l0, l1);
            }
            *reinterpret_cast<uint4*>(tK + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            *reinterpret_cast<uint4*>(tM + off) = make_uint4(wm[0], wm[1], wm[2], wm[3]);
            *reinterpret_cast<uint4*>(tL + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
        fence_proxy_async_smem();
    }
    __syncthreads();
    if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID_H = idesc_bf16(128, D, 1, 1);
        const uint32_t lbo = D == 128 ? kCovTok * 128 : 0;   // the second 64-feature half (D = 64: rows repeat)
        const uint32_t vt_s = smem_u32(tV);
#pragma unroll
        for (int p3 = 0; p3 < 3; ++p3) {
            const uint32_t a_s = smem_u32(p3 == 0 ? tK : p3 == 1 ? tM : tL);
#pragma unroll
            for (int kk = 0; kk < kCovTok / 16; ++kk) {
                const uint64_t ad = sdesc(a_s + kk * 2048, lbo, 1024, kSwizzle128B);
                const uint64_t bd = sdesc(vt_s + kk * 2048, kCovTok * 128, 1024, kSwizzle128B);
                umma_f16_ss(tmem, ad, bd, ID_H, (p3 > 0 || kk > 0) ? 1u : 0u);
            }
        }
        umma_commit(mma_bar);
        if (!mbar_wait(mma_bar, 0, abort_flag, wait_ns)) {
            report(kStatusTimeout);
            *abort_flag = 1;
        }
    }
    __syncthreads();
    tc_fence_after();
    const bool dead = *abort_flag != 0;
    constexpr int C4 = D / 4;                                // 16-byte chunks per row of H_j
    if (!dead && 32 * (warp & 3) < D) {
        // warp w: rows 32 (w % 4) + lane (its tensor-memory lanes), columns of half w / 4
        const int r = 32 * (warp & 3) + lane;
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
#pragma unroll 1
        for (int cc = (warp >> 2) * (D / 2); cc < (warp >> 2) * (D / 2) + D / 2; cc += 32) {
            uint32_t vv[32];
            tmem_ld32(tl + cc, vv);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
                const int c4 = ((cc + x) >> 2) ^ (r & (C4 - 1));
                *reinterpret_cast<float4*>(hs + r * D + c4 * 4) =
                    make_float4(__uint_as_float(vv[x]), __uint_as_float(vv[x + 1]), __uint_as_float(vv[x + 2]),
                                __uint_as_float(vv[x + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, D);
    float a[RT][RT];
    {
        const float* hb = hbar + bh * D * D;
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = cov_idx(ty, i);
#pragma unroll
            for (int jj = 0; jj < RT; jj += 4) {
                const int c = cov_idx(tx, jj);
                const float4 h = __ldg(reinterpret_cast<const float4*>(hb + r * D + c));
                const float4 x = dead ? make_float4(h.x, h.y, h.z, h.w)
                                      : *reinterpret_cast<const float4*>(hs + r * D + (((c >> 2) ^ (r & (C4 - 1))) << 2));
                a[i][jj] = x.x - h.x;
                a[i][jj + 1] = x.y - h.y;
                a[i][jj + 2] = x.z - h.z;
                a[i][jj + 3] = x.w - h.w;
            }
        }
    }
    // 2. Lanczos on B = A^T A from q_0 proportional to (1 + t / D).  Thread t < D owns
    //    element t of the vectors (q_it and q_{it-1} in registers).  A q: each thread
    //    multiplies its tile by its columns of q, the half-warp sums the rows
    //    (cov_half_rows), so every lane holds y = A q on its RT rows; A^T y: each
    //    thread multiplies its tile by those, the two halves of the warp add up,
    //    and the eight warps' sums meet in shared memory.  alpha = q . A^T A q is
    //    |A q|^2.  w leaves each step unnormalised in wraw; the next product scales
    //    it by 1 / beta on the way in.
    const bool own = tid < D;
    float qc = own ? 1.f + static_cast<float>(tid) / D : 0.f;
    for (int i = D + tid; i < kQRows * D; i += 256) qv[i] = 0.f;
    const float n0 = cov_block_sum(qc * qc, red);            // (also orders the writes of qv)
    const float inv0 = 1.f / sqrtf(n0);
    qc *= inv0;
    if (own) {
        qv[tid] = qc;
        wraw[tid] = qc;
    }
    __syncthreads();
    int m = 0;
    float qp = 0.f, inv_b = 1.f, b_prev = 0.f, a_max = 0.f;   // (every thread holds the same sums)
    for (int it = 0; it < kLanczos; ++it) {
        {
            float x[RT], p[RT], y[RT];
#pragma unroll
            for (int jj = 0; jj < RT; jj += 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(wraw + cov_idx(tx, jj));
                x[jj] = t4.x * inv_b;
                x[jj + 1] = t4.y * inv_b;
                x[jj + 2] = t4.z * inv_b;
                x[jj + 3] = t4.w * inv_b;
            }
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                float s = a[i][0] * x[0];
#pragma unroll
                for (int jj = 1; jj < RT; ++jj) s = fmaf(a[i][jj], x[jj], s);
                p[i] = s;
            }
            cov_half_rows<RT>(p, lane, y);
            float y2 = 0.f;                                   // |y|^2 over the warp's rows
            if (tx == 0) {
#pragma unroll
                for (int i = 0; i < RT; ++i) y2 = fmaf(y[i], y[i], y2);
            }
            y2 += __shfl_xor_sync(0xffffffffu, y2, 16);
            if (lane == 0) red[warp] = y2;
            float c[RT], r[RT / 2];
#pragma unroll
            for (int jj = 0; jj < RT; ++jj) {
                float s = a[0][jj] * y[0];
#pragma unroll
                for (int i = 1; i < RT; ++i) s = fmaf(a[i][jj], y[i], s);
                c[jj] = s;
            }
            // the halves add up; half h keeps columns cov_idx(tx, h RT/2 + kk), contiguous
#pragma unroll
            for (int kk = 0; kk < RT / 2; ++kk) {
                const float send = half ? c[kk] : c[kk + RT / 2];
                const float keep = half ? c[kk + RT / 2] : c[kk];
                r[kk] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
            float* dst = part + warp * D + cov_idx(tx, half * (RT / 2));
            if constexpr (RT / 2 == 4) {
                *reinterpret_cast<float4*>(dst) = make_float4(r[0], r[1], r[2], r[3]);
            } else {
                *reinterpret_cast<float2*>(dst) = make_float2(r[0], r[1]);
            }
        }
        __syncthreads();
        float al = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) al += red[u];
        float w = 0.f;                                        // w = A^T y - alpha q - beta q_prev
        if (own) {
            float s = part[tid];
#pragma unroll
            for (int u = 1; u < 8; ++u) s += part[u * D + tid];
            w = s - al * qc - b_prev * qp;
            wv[tid] = w;
        }
        __syncthreads();
        // full re-orthogonalisation against q_0 .. q_it (one classical Gram-Schmidt
        // pass: in an fp32 emulation on Gaussian and video-latent blocks a second
        // pass changed no norm by more than 1e-9 relative): warp u forms the
        // coefficients q_i . w of i = u, u + 8, u + 16, u + 24 together (lanes over
        // the elements, one butterfly; zero for i > it), then every element
        // subtracts the multiples of the q_i, rows past it being zero
        {
            constexpr int E = D / 32;
            float wl[E], pc[4];
#pragma unroll
            for (int e = 0; e < E; ++e) wl[e] = wv[lane + 32 * e];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int i = warp + 8 * kk;
                float s = 0.f;
                if (i <= it) {
#pragma unroll
                    for (int e = 0; e < E; ++e) s = fmaf(qv[i * D + lane + 32 * e], wl[e], s);
                }
                pc[kk] = s;
            }
            const float cs = cov_warp_rows<4>(pc, lane);
            if ((lane & 7) == 0) coef[warp + lane] = cs;          // i = warp + 8 (lane / 8)
        }
        __syncthreads();
        if (own) {
            float w0 = w, w1 = 0.f;
            for (int i = 0; i <= it; i += 4) {
                w0 = fmaf(-coef[i], qv[i * D + tid], w0);
                w1 = fmaf(-coef[i + 1], qv[(i + 1) * D + tid], w1);
                w0 = fmaf(-coef[i + 2], qv[(i + 2) * D + tid], w0);
                w1 = fmaf(-coef[i + 3], qv[(i + 3) * D + tid], w1);
            }
            w = w0 + w1;
            wraw[tid] = w;
        }
        {                                                     // beta = |w|
            float w2 = own ? w * w : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) w2 += __shfl_xor_sync(0xffffffffu, w2, o);
            if (lane == 0) red[8 + warp] = w2;
        }
        __syncthreads();
        float bsq = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) bsq += red[8 + u];
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
        inv_b = 1.f / be;
        const float qn = w * inv_b;                           // q_{it+1}, as the next product sees it
        if (own) qv[(it + 1) * D + tid] = qn;
        qp = qc;
        qc = qn;
        b_prev = be;
    }
    __syncthreads();
    // 3. T out, for cov_eig_kernel
    double* t = tri + (bh * Nk + j) * kTriStride;
    if (tid < kLanczos) {
        t[tid] = tid < m ? alpha[tid] : 0.0;
        t[kLanczos + tid] = tid + 1 < m ? beta[tid] : 0.0;
    }
    if (tid == 0) t[2 * kLanczos] = static_cast<double>(m);
}

// The largest eigenvalue of each block's T by multisection, one warp per block:
// grid ceil(nblk / 8), 256 threads; out[blk] = scale * M_j.  The lanes scale T by
// 2^-e, the power of two that brings its largest Gershgorin bound g into [1/2, 1)
// (exact, no division), and pad it to kLanczos rows with decoupled diagonal
// entries 2 (above every point tried, so they change no count).  Each round every
// lane counts the eigenvalues of T below its own point x of the interval, as the
// sign changes along the leading principal minors of T - x I (Sturm sequence;
// three-term recurrence, no division; a zero minor may take either sign, since
// its neighbours then have opposite signs and one change is counted across it
// either way), and the interval shrinks to the two points around the largest
// eigenvalue, 33 times per round; seven rounds narrow it by 33^7 = 4.3e10.  M_j
// is the square root of 2^e times the upper end.
__global__ void __launch_bounds__(256) cov_eig_kernel(const double* __restrict__ tri, long long nblk,
                                                      double scale, double* __restrict__ out) {
    __shared__ double sa[8][kLanczos], sb[8][kLanczos];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long blk = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (blk >= nblk) return;                               // (whole warps; no barrier below)
    const double* t = tri + blk * kTriStride;
    const int m = static_cast<int>(t[2 * kLanczos]);
    const double al = lane < kLanczos ? t[lane] : 0.0;
    const double be = lane < kLanczos ? t[kLanczos + lane] : 0.0;          // beta_lane (zero from m - 1 on)
    const double bp = __shfl_up_sync(0xffffffffu, be, 1);                 // beta_{lane-1}
    double g = lane < m ? fabs(al) + (lane > 0 ? fabs(bp) : 0.0) + fabs(be) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g = fmax(g, __shfl_xor_sync(0xffffffffu, g, o));
    int e = 0;
    const double gs = g > 0.0 ? frexp(g, &e) : 0.0;                      // g = gs 2^e, gs in [1/2, 1)
    if (lane < kLanczos) {
        const double b = ldexp(be, -e);
        sa[warp][lane] = lane < m ? ldexp(al, -e) : 2.0;
        sb[warp][lane] = b * b;
    }
    __syncwarp();
    const double* A = sa[warp];
    const double* B2 = sb[warp];
    double lo = 0.0, hi = gs;
    for (int round = 0; round < 7; ++round) {
        const double step = (hi - lo) * (1.0 / 33.0);
        const double x = lo + step * (lane + 1);
        double pm = 1.0, pc = A[0] - x;
        int below = __double2hiint(pc) < 0;
#pragma unroll
        for (int i = 1; i < kLanczos; ++i) {
            const double pn = fma(A[i] - x, pc, -B2[i - 1] * pm);
            below += (__double2hiint(pn) ^ __double2hiint(pc)) < 0;
            pm = pc;
            pc = pn;
        }
        // points below the largest eigenvalue count fewer than m eigenvalues below them
        const int kb = __popc(__ballot_sync(0xffffffffu, below < m));
        const double nlo = kb > 0 ? lo + step * kb : lo;
        const double nhi = kb < 32 ? lo + step * (kb + 1) : hi;
        lo = nlo;
        hi = nhi;
    }
    if (lane == 0) out[blk] = scale * sqrt(fmax(ldexp(hi, e), 0.0));
}

}  // namespace sla

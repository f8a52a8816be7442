// router.cuh -- the SLA2 learnable router at inference ("Router Apprendibile",
// SLA2 page sec. 2.B; Arabic page sec. 2.b): mean pooling of Q and K over
// blocks of adjacent tokens, the proj_q / proj_k projections, the compressed
// block score and a hard top-k per query block, emitted as an ascending LUT.
//
// Precision: pooling, projection and score run in fp64.  Sums of bf16 values
// in fp64 are exact for any realistic exponent spread, so the selected set
// equals an exact-arithmetic selection except where two block scores lie
// within ~1e-12 of each other.
#pragma once
#include "common.cuh"

namespace sla {

// ------------------------------------------------------------------ pooling
// One warp per pooled block: blocks blk = warp id, + total warps, ... of `rows`
// consecutive rows of x [nblk_total * rows, d] (bf16, d innermost).  Lane l
// reads 16-byte vector l % (d/8) of rows l / (d/8), + 32/(d/8), ... (unrolled,
// independent loads), sums in fp64, and the lanes holding the same columns
// are combined by shuffles; no block-level synchronisation.
// out_mode 0: out[blk][c]  (row-major [BH*nblk, d])
// out_mode 1: out[bh][c][j] with blk = bh*nblk_per_head + j (transposed per head)
// The value written is the block mean, sum / rows (rows is a power of two, so
// the division is exact; fp64 sums of bf16 values are exact for any realistic
// exponent spread, so the result does not depend on the order of the sum).
template <int D>
__global__ void __launch_bounds__(256, 4) pool_mean_kernel(const __nv_bfloat16* __restrict__ x,
                                                        int rows, long long nblk_total,
                                                        int nblk_per_head, int out_mode,
                                                        double* __restrict__ out) {
    constexpr int VPR = D / 8;            // 16-byte vectors per row
    constexpr int RPL = 32 / VPR;         // rows covered by one warp-wide load
    const int lane = threadIdx.x & 31;
    const int vec = lane % VPR, rsub = lane / VPR;
    const long long nw = static_cast<long long>(gridDim.x) * 8;
    const double inv = 1.0 / static_cast<double>(rows);
    for (long long blk = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); blk < nblk_total;
         blk += nw) {
        const uint4* src = reinterpret_cast<const uint4*>(x + blk * rows * D);
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 16
        for (int r = rsub; r < rows; r += RPL) {
            const uint4 u = __ldg(src + static_cast<long long>(r) * VPR + vec);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += static_cast<double>(bf16lo(w[e]));
                acc[2 * e + 1] += static_cast<double>(bf16hi(w[e]));
            }
        }
#pragma unroll
        for (int o = VPR; o < 32; o <<= 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
        }
        if (rsub == 0) {
            if (out_mode == 0) {
                double2* dst = reinterpret_cast<double2*>(out + blk * D + vec * 8);
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[e] = make_double2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
            } else {
                const long long bh = blk / nblk_per_head;
                const long long j = blk % nblk_per_head;
#pragma unroll
                for (int e = 0; e < 8; ++e) out[(bh * D + vec * 8 + e) * nblk_per_head + j] = acc[e] * inv;
            }
        }
    }
}

// --------------------------------------------------------------- W folding
// The router score is (Qbar W_q) . (Kbar W_k) = Qbar (W_q W_k^T) Kbar^T.
// M = W_q W_k^T in fp64 (W_q alone if W_k is NULL, W_k^T alone if W_q is NULL).
__global__ void fold_w_kernel(const float* __restrict__ wq, const float* __restrict__ wk, int d,
                              double* __restrict__ m) {
    const int c = blockIdx.x;
    for (int e = threadIdx.x; e < d; e += blockDim.x) {
        double s;
        if (wq && wk) {
            // each thread streams its own row of W_k and the broadcast row c of
            // W_q (16-byte loads when both bases allow it; rows are d*4 bytes
            // apart, a multiple of 16); the sum runs over t in order
            s = 0.0;
            if (((reinterpret_cast<uintptr_t>(wq) | reinterpret_cast<uintptr_t>(wk)) & 15u) == 0) {
                const float4* a4 = reinterpret_cast<const float4*>(wq + c * d);
                const float4* b4 = reinterpret_cast<const float4*>(wk + e * d);
#pragma unroll 8
                for (int t4 = 0; t4 < d / 4; ++t4) {
                    const float4 x = __ldg(a4 + t4), y = __ldg(b4 + t4);
                    s += static_cast<double>(x.x) * static_cast<double>(y.x);
                    s += static_cast<double>(x.y) * static_cast<double>(y.y);
                    s += static_cast<double>(x.z) * static_cast<double>(y.z);
                    s += static_cast<double>(x.w) * static_cast<double>(y.w);
                }
            } else {
                for (int t = 0; t < d; ++t)
                    s += static_cast<double>(wq[c * d + t]) * static_cast<double>(wk[e * d + t]);
            }
        } else if (wq) {
            s = static_cast<double>(wq[c * d + e]);
        } else {
            s = static_cast<double>(wk[e * d + c]);
        }
        m[c * d + e] = s;
    }
}

// ------------------------------------------------------------ score + top-k
// Order-preserving map from fp64 to uint64 (larger double -> larger key);
// -0.0 is folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ unsigned long long order_key(double v) {
    v = v + 0.0;
    const long long b = __double_as_longlong(v);
    return b < 0 ? ~static_cast<unsigned long long>(b)
                 : (static_cast<unsigned long long>(b) | 0x8000000000000000ull);
}

// One CTA: head bh = blockIdx.y, query blocks i0 = blockIdx.x * R ... i0 + R - 1.
// Shared memory: qhat^T [D][R] fp64, hist [8][256] u32, keys [R][max(Nk, D)] u64
// (the key area doubles as the [R][D] staging buffer of step 1).
// PF: step 2 reads the kbar columns eight feature rows ahead of use (pays off on
// long rows, where each warp walks several column chunks).
template <int R, int D, bool PF>
__global__ void __launch_bounds__(256) score_topk_kernel(const double* __restrict__ qbar,
                                                         const double* __restrict__ kbarT,
                                                         const double* __restrict__ m, int Nq,
                                                         int Nk, int topk,
                                                         int32_t* __restrict__ lut) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    double* qhT = reinterpret_cast<double*>(smem_raw);                        // [D][R]
    unsigned* hist = reinterpret_cast<unsigned*>(qhT + D * R);                  // [8][256]
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(hist + 8 * 256);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long bh = blockIdx.y;
    const int i0 = blockIdx.x * R;
    const int nrows = min(R, Nq - i0);
    const double* qb = qbar + (bh * Nq + i0) * D;
    const double* kt = kbarT + bh * D * static_cast<long long>(Nk);

    // 1. qhat = qbar . M (or qbar) for the R rows, stored transposed.
    {
        double* qtmp = reinterpret_cast<double*>(keys);   // [R][D] scratch
        for (int a = tid; a < R * D; a += 256) {
            const int r = a / D;
            qtmp[a] = r < nrows ? qb[a] : 0.0;
        }
        __syncthreads();
        constexpr int RG = 256 / D;       // row groups
        constexpr int RPT = R / RG > 0 ? R / RG : 1;
        const int e = tid % D;
        const int g = tid / D;
        if (g < RG && g * RPT < R) {
            double acc[RPT];
#pragma unroll
            for (int r = 0; r < RPT; ++r) acc[r] = 0.0;
            if (m) {
                for (int c = 0; c < D; ++c) {
                    const double mv = __ldg(m + c * D + e);
#pragma unroll
                    for (int r = 0; r < RPT; ++r) acc[r] += qtmp[(g * RPT + r) * D + c] * mv;
                }
            } else {
#pragma unroll
                for (int r = 0; r < RPT; ++r) acc[r] = qtmp[(g * RPT + r) * D + e];
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) qhT[e * R + g * RPT + r] = acc[r];
        }
        __syncthreads();
    }

    // 2. scores s[r][j] = qhat_r . kbar_j, fp64; warp w covers 64 columns at a time.
    for (int j0 = warp * 64; j0 < Nk; j0 += 8 * 64) {
        const int ja = j0 + lane, jb = j0 + 32 + lane;
        const bool va = ja < Nk, vb = jb < Nk;
        double acc0[R], acc1[R];
#pragma unroll
        for (int r = 0; r < R; ++r) { acc0[r] = 0.0; acc1[r] = 0.0; }
        if (PF) {
            double ka[8], kb[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                ka[x] = va ? __ldg(kt + static_cast<long long>(x) * Nk + ja) : 0.0;
                kb[x] = vb ? __ldg(kt + static_cast<long long>(x) * Nk + jb) : 0.0;
            }
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 8) {
                double na[8], nb[8];
                const bool more = c0 + 8 < D;
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    na[x] = (more && va) ? __ldg(kt + static_cast<long long>(c0 + 8 + x) * Nk + ja) : 0.0;
                    nb[x] = (more && vb) ? __ldg(kt + static_cast<long long>(c0 + 8 + x) * Nk + jb) : 0.0;
                }
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const double2* qrow = reinterpret_cast<const double2*>(qhT + (c0 + x) * R);
#pragma unroll
                    for (int r2 = 0; r2 < R / 2; ++r2) {
                        const double2 qq = qrow[r2];
                        acc0[2 * r2] = fma(qq.x, ka[x], acc0[2 * r2]);
                        acc1[2 * r2] = fma(qq.x, kb[x], acc1[2 * r2]);
                        acc0[2 * r2 + 1] = fma(qq.y, ka[x], acc0[2 * r2 + 1]);
                        acc1[2 * r2 + 1] = fma(qq.y, kb[x], acc1[2 * r2 + 1]);
                    }
                }
#pragma unroll
                for (int x = 0; x < 8; ++x) { ka[x] = na[x]; kb[x] = nb[x]; }
            }
        } else {
#pragma unroll 4
            for (int c = 0; c < D; ++c) {
                const double ka = va ? __ldg(kt + static_cast<long long>(c) * Nk + ja) : 0.0;
                const double kb = vb ? __ldg(kt + static_cast<long long>(c) * Nk + jb) : 0.0;
                const double2* qrow = reinterpret_cast<const double2*>(qhT + c * R);
#pragma unroll
                for (int r2 = 0; r2 < R / 2; ++r2) {
                    const double2 qq = qrow[r2];
                    acc0[2 * r2] = fma(qq.x, ka, acc0[2 * r2]);
                    acc1[2 * r2] = fma(qq.x, kb, acc1[2 * r2]);
                    acc0[2 * r2 + 1] = fma(qq.y, ka, acc0[2 * r2 + 1]);
                    acc1[2 * r2 + 1] = fma(qq.y, kb, acc1[2 * r2 + 1]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (va) keys[static_cast<size_t>(r) * Nk + ja] = order_key(acc0[r]);
            if (vb) keys[static_cast<size_t>(r) * Nk + jb] = order_key(acc1[r]);
        }
    }
    __syncthreads();
    if (topk <= 0) return;

    // 3. per row: radix-select the topk-th largest key, then emit ascending.
    unsigned* h = hist + warp * 256;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int r = warp; r < nrows; r += 8) {
        const unsigned long long* kr = keys + static_cast<size_t>(r) * Nk;
        int32_t* dst = lut + ((bh * Nq) + i0 + r) * static_cast<long long>(topk);
        unsigned long long prefix = 0ull, pmask = 0ull;
        int rem = topk;
        if (topk < Nk) {
            for (int shift = 56; shift >= 0; shift -= 8) {
                for (int b = lane; b < 256; b += 32) h[b] = 0u;
                __syncwarp();
                for (int j = lane; j < Nk; j += 32) {
                    const unsigned long long key = kr[j];
                    if ((key & pmask) == prefix) atomicAdd(&h[(key >> shift) & 255ull], 1u);
                }
                __syncwarp();
                int cnt[8], s = 0;
#pragma unroll
                for (int b = 0; b < 8; ++b) { cnt[b] = static_cast<int>(h[255 - 8 * lane - b]); s += cnt[b]; }
                int incl = s;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const int excl = incl - s;
                const bool mine = excl < rem && rem <= incl;
                const unsigned bal = __ballot_sync(0xffffffffu, mine);
                int digit = 0, newrem = 0;
                if (mine) {
                    int a = excl;
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        if (a + cnt[b] >= rem) { digit = 255 - 8 * lane - b; newrem = rem - a; break; }
                        a += cnt[b];
                    }
                }
                const int src = bal ? __ffs(bal) - 1 : 0;
                digit = __shfl_sync(0xffffffffu, digit, src);
                newrem = __shfl_sync(0xffffffffu, newrem, src);
                prefix |= static_cast<unsigned long long>(digit) << shift;
                pmask |= 255ull << shift;
                rem = newrem;
                __syncwarp();
            }
        } else {
            prefix = 0ull;      // every key is >= 0: take all of them
            rem = 0;
        }
        int out = 0, eqseen = 0;
        for (int j0 = 0; j0 < Nk; j0 += 32) {
            const int j = j0 + lane;
            const unsigned long long key = j < Nk ? kr[j] : 0ull;
            const bool gt = j < Nk && (topk >= Nk || key > prefix);
            const bool eq = j < Nk && topk < Nk && key == prefix;
            const unsigned beq = __ballot_sync(0xffffffffu, eq);
            const int eqrank = eqseen + __popc(beq & lt_mask);
            const bool sel = gt || (eq && eqrank < rem);
            const unsigned bsel = __ballot_sync(0xffffffffu, sel);
            if (sel) dst[out + __popc(bsel & lt_mask)] = j;
            out += __popc(bsel);
            eqseen += __popc(beq);
        }
    }
}

}  // namespace sla

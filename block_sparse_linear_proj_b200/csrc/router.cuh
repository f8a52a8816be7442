// router.cuh -- the SLA2 learnable router at inference ("Router Apprendibile",
// SLA2 page sec. 2.B; Arabic page sec. 2.b): mean pooling of Q and K over
// blocks of adjacent tokens, the proj_q / proj_k projections, the compressed
// block score and a hard top-k per query block, emitted as an ascending LUT.
//
// Precision: pooling, projection and score run in fp64 (the products on the
// fp64 tensor-core MMA).  Sums of bf16 values in fp64 are exact for any
// realistic exponent spread, so the selected set equals an exact-arithmetic
// selection except where two block scores lie within ~1e-12 of each other; the
// top-k itself is an exact selection on the fp64 scores (ties to the lower j).
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

// fp64 tensor-core product D(8x8) += A(8x4) B(4x8), A row-major, B column-major:
// lane l holds A[l/4][l%4], B[l%4][l/4] and D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_884(double (&d)[2], double a, double b) {
    asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
        : "+d"(d[0]), "+d"(d[1])
        : "d"(a), "d"(b));
}

__device__ __forceinline__ unsigned long long warp_min_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// qhat = qbar . M in place, 16 pooled rows per CTA (rows [16 b, 16 b + 16) of
// the [nrows][D] fp64 array x), on the fp64 MMA: warp w computes output columns
// [w D/8, (w+1) D/8) of both 8-row tiles from M fragments three k-steps ahead.
// Each CTA reads its rows into shared memory before writing them back.
template <int D>
__global__ void __launch_bounds__(256) project_kernel(double* __restrict__ x, long long nrows,
                                                      const double* __restrict__ m) {
    constexpr int LDQ = D + 4, NT = D / 64;
    __shared__ double xs[16 * LDQ];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const long long r0 = static_cast<long long>(blockIdx.x) * 16;
    const int rows = static_cast<int>(min(16LL, nrows - r0));
    for (int a = tid; a < 16 * D; a += 256) {
        const int r = a / D, c = a % D;
        xs[r * LDQ + c] = r < rows ? x[(r0 + r) * D + c] : 0.0;
    }
    __syncthreads();
    double acc[2][NT][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = 0.0;
    const int n0 = warp * (D / 8);
    double bm[4][NT];
    auto load_m = [&](double (&b)[NT], int c0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) b[nt] = __ldg(m + (c0 + t) * D + n0 + nt * 8 + g);
    };
#pragma unroll
    for (int u = 0; u < 4; ++u) load_m(bm[u], u * 4);
#pragma unroll 1
    for (int ks = 0; ks < D / 4; ks += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            double a[2];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) a[mt] = xs[(mt * 8 + g) * LDQ + (ks + u) * 4 + t];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) dmma_884(acc[mt][nt], a[mt], bm[u][nt]);
            if (ks + u + 4 < D / 4) load_m(bm[u], (ks + u + 4) * 4);
        }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const int r = mt * 8 + g;
        if (r >= rows) continue;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            double* dst = x + (r0 + r) * D + n0 + nt * 8 + 2 * t;
            dst[0] = acc[mt][nt][0];
            dst[1] = acc[mt][nt][1];
        }
    }
}

// One CTA: head bh = blockIdx.y, query blocks i0 = blockIdx.x * R ... i0 + R - 1.
// qhat = qbar M (project_kernel) or qbar itself; bias (null: none) [BH][Nk] is
// added to every score of block j (PISA's covariance-aware selection).  The product runs on the fp64
// MMA (m8n8k4, eight-row tiles; R < 8 pads the tile).  Shared memory: qhat
// [8 MT][D + 4] fp64 (rows padded so that the A-fragment loads spread over the
// banks), hist [8][256] u32, keys [R][max(Nk, D + 4)] u64.
// DEPTH: k-steps of K fragments in flight per warp; MINB: CTAs per SM the
// register budget is sized for.
template <int R, int D, int DEPTH, int MINB>
__global__ void __launch_bounds__(256, MINB) score_topk_kernel(const double* __restrict__ qhat_all,
                                                         const double* __restrict__ kbarT,
                                                         const double* __restrict__ bias, int Nq,
                                                         int Nk, int topk,
                                                         int32_t* __restrict__ lut) {
    constexpr int MT = R >= 8 ? R / 8 : 1;      // eight-row MMA tiles
    constexpr int LDQ = D + 4;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    double* qh = reinterpret_cast<double*>(smem_raw);                              // [8 MT][LDQ]
    unsigned* hist = reinterpret_cast<unsigned*>(qh + 8 * MT * LDQ);               // [8][256]
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(hist + 8 * 256);
    const int ldk = max(Nk, LDQ);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const long long bh = blockIdx.y;
    const int i0 = blockIdx.x * R;
    const int nrows = min(R, Nq - i0);
    const double* qhat = qhat_all + (bh * Nq + i0) * D;
    const double* kt = kbarT + bh * D * static_cast<long long>(Nk);
    const double* brow = bias ? bias + bh * Nk : nullptr;   // per-block score term, or none

    // 1. the R rows of qhat (padding rows are zero)
    for (int a = tid; a < 8 * MT * D; a += 256) {
        const int r = a / D, c = a % D;
        qh[r * LDQ + c] = r < nrows ? qhat[static_cast<long long>(r) * D + c] : 0.0;
    }
    __syncthreads();

    // 2. scores s[r][j] = qhat_r . kbar_j on the fp64 MMA.  Warp w covers 64
    //    columns (eight 8-column tiles) at a time; a ring of DEPTH k-steps of B
    //    fragments, each slot refilled DEPTH k-steps ahead right after its use.
    for (int j0 = warp * 64; j0 < Nk; j0 += 8 * 64) {
        double acc[MT][8][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = 0.0;
        bool live[8];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) live[nt] = j0 + nt * 8 + g < Nk;
        const double* kc = kt + j0 + g;
        auto load = [&](double (&b)[8], int c0) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                b[nt] = live[nt] ? __ldg(kc + static_cast<long long>(c0 + t) * Nk + nt * 8) : 0.0;
        };
        static_assert((D / 4) % DEPTH == 0, "ring depth must divide the k-steps");
        double bq[DEPTH][8];
#pragma unroll
        for (int u = 0; u < DEPTH; ++u) load(bq[u], u * 4);
#pragma unroll 1
        for (int ks = 0; ks < D / 4; ks += DEPTH) {
#pragma unroll
            for (int u = 0; u < DEPTH; ++u) {
                double a[MT];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) a[mt] = qh[(mt * 8 + g) * LDQ + (ks + u) * 4 + t];
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) dmma_884(acc[mt][nt], a[mt], bq[u][nt]);
                if (ks + u + DEPTH < D / 4) load(bq[u], (ks + u + DEPTH) * 4);
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r = mt * 8 + g;
            if (r >= R) continue;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int j = j0 + nt * 8 + 2 * t;
                if (j < Nk)
                    keys[static_cast<size_t>(r) * ldk + j] = order_key(brow ? acc[mt][nt][0] + brow[j] : acc[mt][nt][0]);
                if (j + 1 < Nk)
                    keys[static_cast<size_t>(r) * ldk + j + 1] =
                        order_key(brow ? acc[mt][nt][1] + brow[j + 1] : acc[mt][nt][1]);
            }
        }
    }
    __syncthreads();
    if (topk <= 0) return;

    // 3. per row (one warp): find the topk-th largest key and emit the selected
    //    block indices ascending.  The candidates are the keys of an interval
    //    [klo, khi] (every key above it is taken, rem more are needed from it).
    //    A pass bins them by (key - klo) >> s, s chosen so that 256 bins cover the
    //    interval, and keeps the bin holding the rem-th largest: the interval
    //    shrinks at least 128-fold per pass (at most 10 passes).  It stops when
    //    that bin's keys are exactly the ones still needed (take every key >= its
    //    lower bound), or when the interval is one key value (take the rem of
    //    those keys with the lowest j).
    unsigned* h = hist + warp * 256;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int r = warp; r < nrows; r += 8) {
        const unsigned long long* kr = keys + static_cast<size_t>(r) * ldk;
        int32_t* dst = lut + ((bh * Nq) + i0 + r) * static_cast<long long>(topk);
        unsigned long long T = 0ull;      // threshold key
        int rem = topk;                   // keys equal to T still to take (lowest j first)
        bool ge = false;                  // take every key >= T
        if (topk < Nk) {
            unsigned long long klo = ~0ull, khi = 0ull;
            for (int j = lane; j < Nk; j += 32) {
                const unsigned long long key = kr[j];
                klo = min(klo, key);
                khi = max(khi, key);
            }
            klo = warp_min_u64(klo);
            khi = warp_max_u64(khi);
            for (int pass = 0; pass < 12 && klo != khi; ++pass) {
                const unsigned long long span = khi - klo;
                const int sh = max(64 - __clzll(static_cast<long long>(span)) - 8, 0);
                for (int b = lane; b < 256; b += 32) h[b] = 0u;
                __syncwarp();
                for (int j = lane; j < Nk; j += 32) {
                    const unsigned long long key = kr[j];
                    if (key >= klo && key <= khi) atomicAdd(&h[static_cast<int>((key - klo) >> sh)], 1u);
                }
                __syncwarp();
                // bins from the top: lane l owns bins 255 - 8l ... 248 - 8l
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
                int digit = 0, newrem = 0, dcnt = 0;
                if (mine) {
                    int a = excl;
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        if (a + cnt[b] >= rem) { digit = 255 - 8 * lane - b; newrem = rem - a; dcnt = cnt[b]; break; }
                        a += cnt[b];
                    }
                }
                const int src = bal ? __ffs(bal) - 1 : 0;
                digit = __shfl_sync(0xffffffffu, digit, src);
                rem = __shfl_sync(0xffffffffu, newrem, src);
                dcnt = __shfl_sync(0xffffffffu, dcnt, src);
                const unsigned long long nlo = klo + (static_cast<unsigned long long>(digit) << sh);
                const unsigned long long width = (1ull << sh) - 1ull;
                __syncwarp();
                klo = nlo;
                if (rem == dcnt) { ge = true; break; }
                if (khi - nlo > width) khi = nlo + width;   // (no wrap past 2^64)
            }
            T = klo;
        } else {
            ge = true;                    // every key is taken
            rem = 0;
        }
        int out = 0, eqseen = 0;
        for (int j0 = 0; j0 < Nk; j0 += 32) {
            const int j = j0 + lane;
            const unsigned long long key = j < Nk ? kr[j] : 0ull;
            const bool gt = j < Nk && key > T;
            const bool eq = j < Nk && key == T;
            const unsigned beq = __ballot_sync(0xffffffffu, eq);
            const int eqrank = eqseen + __popc(beq & lt_mask);
            const bool sel = gt || (eq && (ge || eqrank < rem));
            const unsigned bsel = __ballot_sync(0xffffffffu, sel);
            if (sel) dst[out + __popc(bsel & lt_mask)] = j;
            out += __popc(bsel);
            eqseen += __popc(beq);
        }
    }
}

}  // namespace sla

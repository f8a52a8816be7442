// kv_stats.cuh -- one streaming pass over K and V (HBM-bound) that produces
// every per-KV-block statistic the forward needs:
//   * router:  Kbar_j = mean of the block's keys (fp64, stored [bh][c][j]);
//   * linear branch ([SALAD] ReLU kernel, block form): z_j = sum phi(k_n)
//     (fp32 [bh][j][c]) and a per-chunk partial of H = phi(K)^T V (fp32 d x d),
//     reduced over chunks by h_reduce_kernel in a fixed order;
//   * PISA precompute ("Pre-calcolo" of the PISA page): the block centroid
//     kbar_j (bf16) and the value mean vbar_j = (sum_n v_n)/Bk (fp16), both
//     [bh][j][c], the operands of the zero-order pseudo-tiles;
//   * an fp16 copy of V, the B operand of the attention kernel's P.V product,
//     and (SLA) phi(K) = max(K, 0) in fp16, the A operand of its phi(K)^T V
//     product (the conversion from bf16 is exact inside the fp16 range; values
//     outside it are flagged).
// phi(K)^T V uses warp-level bf16 tensor-core MMA (m16n8k16) with fp32
// accumulation; K and V tiles of 64 tokens stream through a 3-stage cp.async
// ring with an XOR swizzle so ldmatrix reads are conflict-free.
#pragma once
#include "common.cuh"

namespace sla {

constexpr int kKvTok = 64;     // tokens per KV block (Bk)
constexpr int kKvStages = 3;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
    h = __hmax2(h, __floats2bfloat162_rn(0.f, 0.f));
    return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of element (row n, col c) in a [64][D] bf16 tile whose 16-byte
// chunks are XOR-swizzled by (n & 7).
template <int D>
__device__ __forceinline__ uint32_t kv_off(int n, int c) {
    return static_cast<uint32_t>(n * D * 2 + ((((c >> 3) ^ (n & 7))) << 4) + (c & 7) * 2);
}

struct KvStatsArgs {
    const __nv_bfloat16* k;     // [BH][N][D]
    const __nv_bfloat16* v;     // [BH][N][D] (may be null when only kbarT is wanted)
    int N, Nk, blocks_per_chunk, nchunk;
    double* kbarT;              // [BH][D][Nk]           (null: skip)
    float* zj;                  // [BH][Nk][D]           (null: skip)
    float* hpart;               // [BH][nchunk][D][D]    (null: skip the MMA)
    __nv_bfloat16* kc;          // [BH][Nk][D] centroids (null: skip)
    __half* vbar;               // [BH][Nk][D] value means (null: skip)
    __half* v16;                // [BH][N][D] fp16 copy of V (null: skip)
    __half* phik16;             // [BH][N][D] fp16 phi(K) (null: skip)
    // FP8 sparse branch (null: skip): e4m3 K [BH][N][D] and V transposed per
    // 64-token block [BH][Nk][D][64], one absmax scale per block (absmax / 448)
    uint8_t* k8;
    uint8_t* v8t;
    float* sk;                  // [BH][Nk]
    float* sv;                  // [BH][Nk]
    // PISA first-order term: the product uses K centred by its block mean,
    // (k_n - kbar_j), instead of phi(K), so hpart sums the blocks' H_j
    int center;
    // with k8: symmetric 8-bit integer K codes (absmax / 127) instead of e4m3
    int k_int8;
};

// grid (nchunk, BH), 256 threads.
template <int D>
__global__ void __launch_bounds__(256, 2) kv_stats_kernel(KvStatsArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr int TILE = kKvTok * D * 2;               // bytes of one K or V tile
    unsigned char* ring = smem_raw;                    // [stages][K tile | V tile]
    double* kpart = reinterpret_cast<double*>(smem_raw + kKvStages * 2 * TILE);   // [256]
    float* zpart = reinterpret_cast<float*>(kpart + 256);                          // [256]
    float* vpart = zpart + 256;                                                    // [256]
    float* amax = vpart + 256;                                                     // [2][8]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long bh = blockIdx.y;
    const int chunk = blockIdx.x;
    const int jb0 = chunk * a.blocks_per_chunk;
    const int nblk = min(a.blocks_per_chunk, a.Nk - jb0);
    if (nblk <= 0) return;
    const bool want_v = a.v != nullptr;
    const __nv_bfloat16* kh = a.k + bh * static_cast<long long>(a.N) * D;
    const __nv_bfloat16* vh = want_v ? a.v + bh * static_cast<long long>(a.N) * D : nullptr;

    auto load_block = [&](int blk, int stage) {
        unsigned char* kd = ring + stage * 2 * TILE;
        unsigned char* vd = kd + TILE;
        const long long row0 = static_cast<long long>(jb0 + blk) * kKvTok;
        constexpr int CPR = D / 8;                      // 16-byte chunks per row
        for (int q = tid; q < kKvTok * CPR; q += 256) {
            const int n = q / CPR, u = q % CPR;
            const uint32_t off = kv_off<D>(n, u * 8);
            cp_async16(kd + off, kh + (row0 + n) * D + u * 8);
            if (want_v) cp_async16(vd + off, vh + (row0 + n) * D + u * 8);
        }
    };

    // MMA tiling of the D x D partial: 8 warps, warp tile (D/4) x (D/2).
    constexpr int WM = D / 4, WN = D / 2;
    constexpr int MT = WM / 16, NT = WN / 8;
    const int m0 = (warp & 3) * WM, n0 = (warp >> 2) * WN;
    float acc[MT][NT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    const bool do_mma = a.hpart != nullptr;

#pragma unroll
    for (int s = 0; s < kKvStages - 1; ++s) {
        if (s < nblk) load_block(s, s);
        cp_async_commit();
    }

    constexpr int HALVES = 256 / D;                 // row groups for the column sums
    constexpr int RPH = kKvTok / HALVES;
    const int col = tid % D, half = tid / D;

    for (int blk = 0; blk < nblk; ++blk) {
        const int stage = blk % kKvStages;
        cp_async_wait<kKvStages - 2>();
        __syncthreads();
        {   // prefetch the block kKvStages-1 ahead into the stage freed last iteration
            const int nb = blk + kKvStages - 1;
            if (nb < nblk) load_block(nb, nb % kKvStages);
            cp_async_commit();
        }
        const unsigned char* kt = ring + stage * 2 * TILE;
        const unsigned char* vt = kt + TILE;
        const uint32_t kt_s = smem_u32(kt), vt_s = smem_u32(vt);

        // column statistics of this block
        {
            double ks = 0.0;
            float zs = 0.f, vs = 0.f, kmax = 0.f;
            for (int n = half * RPH; n < (half + 1) * RPH; ++n) {
                const float kv = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(kt + kv_off<D>(n, col)));
                ks += static_cast<double>(kv);
                zs += fmaxf(kv, 0.f);
                kmax = fmaxf(kmax, fabsf(kv));
                if (want_v)
                    vs += __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D>(n, col)));
            }
            kpart[tid] = ks;
            zpart[tid] = zs;
            vpart[tid] = vs;
            if (a.v16 && !(kmax < 65504.f)) report(kStatusRange);
            if (a.k8) {
                // per-block absmax of K and V (warp max, then 8 partials in smem)
                float vmax = 0.f;
                for (int n = half * RPH; n < (half + 1) * RPH; ++n)
                    vmax = fmaxf(vmax, fabsf(__bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D>(n, col)))));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
                    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
                }
                if (lane == 0) { amax[warp] = kmax; amax[8 + warp] = vmax; }
            }
        }
        // fp16 copy of the V tile (coalesced 16-byte stores)
        if (a.v16) {
            constexpr int CPR = D / 8;
            const long long row0 = static_cast<long long>(jb0 + blk) * kKvTok;
            __half* vo = a.v16 + bh * static_cast<long long>(a.N) * D;
            bool bad = false;
            for (int q = tid; q < kKvTok * CPR; q += 256) {
                const int n = q / CPR, u = q % CPR;
                const uint4 x = *reinterpret_cast<const uint4*>(vt + kv_off<D>(n, u * 8));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float lo = bf16lo(w[e]), hi = bf16hi(w[e]);
                    bad |= !(fabsf(lo) < 65504.f) || !(fabsf(hi) < 65504.f);
                    h[e] = pack_half2(lo, hi);
                }
                *reinterpret_cast<uint4*>(vo + (row0 + n) * D + u * 8) = make_uint4(h[0], h[1], h[2], h[3]);
            }
            if (bad) report(kStatusRange);
        }
        // e4m3 K (row-major) and V (transposed per block) with one scale per block
        if (a.k8) {
            __syncthreads();
            float km = 0.f, vm = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) { km = fmaxf(km, amax[w]); vm = fmaxf(vm, amax[8 + w]); }
            // codes are picked by the correctly rounded quotient x / s (not x * (1/s),
            // which lands on the other side of a rounding midpoint now and then)
            const float s_k = km > 0.f ? km / (a.k_int8 ? 127.f : 448.f) : 1.f;
            const float s_v = vm > 0.f ? vm / 448.f : 1.f;
            const int j = jb0 + blk;
            if (tid == 0) {
                a.sk[bh * a.Nk + j] = s_k;
                a.sv[bh * a.Nk + j] = s_v;
            }
            constexpr int CPR = D / 8;
            const long long row0 = static_cast<long long>(j) * kKvTok;
            uint8_t* ko = a.k8 + bh * static_cast<long long>(a.N) * D;
            for (int q = tid; q < kKvTok * CPR; q += 256) {
                const int n = q / CPR, u = q % CPR;
                const uint4 x = *reinterpret_cast<const uint4*>(kt + kv_off<D>(n, u * 8));
                uint32_t w0, w1;
                if (a.k_int8) {
                    w0 = pack_s8x4(bf16lo(x.x) / s_k, bf16hi(x.x) / s_k, bf16lo(x.y) / s_k, bf16hi(x.y) / s_k);
                    w1 = pack_s8x4(bf16lo(x.z) / s_k, bf16hi(x.z) / s_k, bf16lo(x.w) / s_k, bf16hi(x.w) / s_k);
                } else {
                    w0 = pack_e4m3x4(bf16lo(x.x) / s_k, bf16hi(x.x) / s_k, bf16lo(x.y) / s_k, bf16hi(x.y) / s_k);
                    w1 = pack_e4m3x4(bf16lo(x.z) / s_k, bf16hi(x.z) / s_k, bf16lo(x.w) / s_k, bf16hi(x.w) / s_k);
                }
                *reinterpret_cast<uint2*>(ko + (row0 + n) * D + u * 8) = make_uint2(w0, w1);
            }
            // V^T: row c of the block holds the 64 tokens of feature c
            uint8_t* vo = a.v8t + (bh * a.Nk + j) * static_cast<long long>(D) * kKvTok;
            for (int q = tid; q < D * (kKvTok / 8); q += 256) {
                const int c = q % D, n0 = (q / D) * 8;
                float f[8];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    f[t] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D>(n0 + t, c))) / s_v;
                *reinterpret_cast<uint2*>(vo + c * kKvTok + n0) =
                    make_uint2(pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]));
            }
        }
        // fp16 phi(K) = max(K, 0)
        if (a.phik16) {
            constexpr int CPR = D / 8;
            const long long row0 = static_cast<long long>(jb0 + blk) * kKvTok;
            __half* ko = a.phik16 + bh * static_cast<long long>(a.N) * D;
            for (int q = tid; q < kKvTok * CPR; q += 256) {
                const int n = q / CPR, u = q % CPR;
                const uint4 x = *reinterpret_cast<const uint4*>(kt + kv_off<D>(n, u * 8));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    h[e] = pack_half2(fmaxf(bf16lo(w[e]), 0.f), fmaxf(bf16hi(w[e]), 0.f));
                *reinterpret_cast<uint4*>(ko + (row0 + n) * D + u * 8) = make_uint4(h[0], h[1], h[2], h[3]);
            }
        }

        // centred keys: this block's column means (from the column statistics
        // above), for the two feature rows of each A fragment
        float kb0[MT], kb1[MT];
        if (a.center) {
            __syncthreads();
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int c0 = m0 + i * 16 + (lane >> 2);
                double s0 = 0.0, s1 = 0.0;
#pragma unroll
                for (int hh = 0; hh < HALVES; ++hh) {
                    s0 += kpart[hh * D + c0];
                    s1 += kpart[hh * D + c0 + 8];
                }
                kb0[i] = static_cast<float>(s0 * (1.0 / kKvTok));
                kb1[i] = static_cast<float>(s1 * (1.0 / kKvTok));
            }
        }
        if (do_mma) {
#pragma unroll
            for (int k0 = 0; k0 < kKvTok; k0 += 16) {
                uint32_t afr[MT][4];
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    // A = phi(K)^T: matrices (n k0..+7 | k0+8..+15) x (c m..m+7 | m+8..m+15)
                    const int n = k0 + (lane & 7) + ((lane >> 4) << 3);
                    const int c = m0 + i * 16 + (((lane >> 3) & 1) << 3);
                    ldsm_x4_trans(kt_s + kv_off<D>(n, c), afr[i][0], afr[i][1], afr[i][2],
                                  afr[i][3]);
                    if (a.center) {
                        // fragments 0, 2 hold feature row m + g, fragments 1, 3 row m + 8 + g
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float kb = (e & 1) ? kb1[i] : kb0[i];
                            afr[i][e] = pack_bf16(bf16lo(afr[i][e]) - kb, bf16hi(afr[i][e]) - kb);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) afr[i][e] = relu_bf16x2(afr[i][e]);
                    }
                }
#pragma unroll
                for (int j = 0; j < NT; j += 2) {
                    const int n = k0 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int e = n0 + j * 8 + ((lane >> 4) << 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vt_s + kv_off<D>(n, e), b0, b1, b2, b3);
#pragma unroll
                    for (int i = 0; i < MT; ++i) {
                        mma_bf16_16816(acc[i][j], afr[i], b0, b1);
                        mma_bf16_16816(acc[i][j + 1], afr[i], b2, b3);
                    }
                }
            }
        }
        __syncthreads();
        if (tid < D) {
            double ks = 0.0;
            float zs = 0.f, vs = 0.f;
#pragma unroll
            for (int h = 0; h < HALVES; ++h) {
                ks += kpart[h * D + tid];
                zs += zpart[h * D + tid];
                vs += vpart[h * D + tid];
            }
            const int j = jb0 + blk;
            const double kmean = ks * (1.0 / kKvTok);
            if (a.kbarT) a.kbarT[(bh * D + tid) * a.Nk + j] = kmean;
            if (a.zj) a.zj[(bh * a.Nk + j) * D + tid] = zs;
            if (a.kc) a.kc[(bh * a.Nk + j) * D + tid] = __float2bfloat16_rn(static_cast<float>(kmean));
            if (a.vbar) a.vbar[(bh * a.Nk + j) * D + tid] = __float2half_rn(vs * (1.f / kKvTok));
        }
    }
    cp_async_wait<0>();

    if (do_mma) {
        float* hp = a.hpart + (bh * a.nchunk + chunk) * static_cast<long long>(D) * D;
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const int r = m0 + i * 16 + g, c = n0 + j * 8 + 2 * t;
                *reinterpret_cast<float2*>(hp + r * D + c) = make_float2(acc[i][j][0], acc[i][j][1]);
                *reinterpret_cast<float2*>(hp + (r + 8) * D + c) =
                    make_float2(acc[i][j][2], acc[i][j][3]);
            }
    }
}

// H[bh] = sum over chunks of hpart (fixed order), stored transposed
// (hsum[bh][e][c] = H[c][e]); Z[bh] = sum_j z_j.
// grid (D*D/256 + 1, BH), 256 threads; the last x-block reduces Z: its eight
// warps take interleaved blocks j, each thread four columns with independent
// loads, and the eight partial sums are added in a fixed order.
template <int D>
__global__ void __launch_bounds__(256) h_reduce_kernel(const float* __restrict__ hpart,
                                                       const float* __restrict__ zj, int nchunk,
                                                       int Nk, float* __restrict__ hsum,
                                                       float* __restrict__ zsum) {
    const long long bh = blockIdx.y;
    constexpr int NHB = D * D / 256;
    if (blockIdx.x < NHB) {
        const int idx = blockIdx.x * 256 + threadIdx.x;
        const float* src = hpart + bh * nchunk * static_cast<long long>(D) * D + idx;
        float s = 0.f;
#pragma unroll 8
        for (int c = 0; c < nchunk; ++c) s += __ldg(src + static_cast<long long>(c) * D * D);
        const int c = idx / D, e = idx % D;
        hsum[bh * D * D + e * D + c] = s;
    } else if (zj) {
        __shared__ float zp[8][D];
        constexpr int CPT = D / 32;                      // columns per thread
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const float* src = zj + bh * static_cast<long long>(Nk) * D;
        float acc[CPT];
#pragma unroll
        for (int x = 0; x < CPT; ++x) acc[x] = 0.f;
#pragma unroll 4
        for (int j = warp; j < Nk; j += 8) {
#pragma unroll
            for (int x = 0; x < CPT; ++x) acc[x] += __ldg(src + static_cast<long long>(j) * D + lane + 32 * x);
        }
#pragma unroll
        for (int x = 0; x < CPT; ++x) zp[warp][lane + 32 * x] = acc[x];
        __syncthreads();
        if (threadIdx.x < D) {
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) t += zp[w][threadIdx.x];
            zsum[bh * D + threadIdx.x] = t;
        }
    }
}

// e4m3 Q (I8: symmetric 8-bit integer Q) with one absmax scale per 64-token
// block (absmax / 448, or absmax / 127).
// Grid-stride over the BH*N/64 blocks; 256 threads, 64 x D tile in registers.
template <int D, bool I8>
__global__ void __launch_bounds__(256) quant_q_kernel(const __nv_bfloat16* __restrict__ q,
                                                      long long nblk, uint8_t* __restrict__ q8,
                                                      float* __restrict__ sq) {
    constexpr int VEC = 64 * D / 8 / 256;          // uint4 per thread
    __shared__ float part[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long long blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(q + blk * 64 * D);
        uint4 x[VEC];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            x[i] = __ldg(src + i * 256 + tid);
            const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[e])), fabsf(bf16hi(w[e]))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) part[warp] = m;
        __syncthreads();
        float am = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) am = fmaxf(am, part[w]);
        // codes from the rounded quotient x / s
        const float s = am > 0.f ? am / (I8 ? 127.f : 448.f) : 1.f;
        if (tid == 0) sq[blk] = s;
        uint2* dst = reinterpret_cast<uint2*>(q8 + blk * 64 * D);
        auto pack = [](float a0, float a1, float a2, float a3) {
            return I8 ? pack_s8x4(a0, a1, a2, a3) : pack_e4m3x4(a0, a1, a2, a3);
        };
#pragma unroll
        for (int i = 0; i < VEC; ++i)
            dst[i * 256 + tid] = make_uint2(
                pack(bf16lo(x[i].x) / s, bf16hi(x[i].x) / s, bf16lo(x[i].y) / s, bf16hi(x[i].y) / s),
                pack(bf16lo(x[i].z) / s, bf16hi(x[i].z) / s, bf16lo(x[i].w) / s, bf16hi(x[i].w) / s));
        __syncthreads();
    }
}

}  // namespace sla

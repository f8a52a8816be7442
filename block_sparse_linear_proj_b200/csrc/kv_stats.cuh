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
// K and V tiles of 64 tokens stream through a 3-stage cp.async ring.  When the
// call runs the product below, each tile is stored as 64-column halves of 64
// rows x 128 bytes with the 128-byte swizzle (the tcgen05 operand layout);
// otherwise as swizzled rows of 2d bytes, which the statistics and copy passes
// read faster.  phi(K)^T V (or, for the PISA first-order
// term, (K - kbar_j)^T V) runs on tcgen05: after the statistics and copies
// have read the raw K tile, it is replaced in place by phi(K) (or the centred
// keys) in bf16, and one thread issues the block's four M = 128, K = 16
// products (bf16 operands, both MN-major) into an fp32 accumulator in tensor
// memory that sums the CTA's blocks.
// X3 (the covariance norms' H_j, exactly): the keys are centred in fp64 by the
// block's column means and rounded once to fp32, as the covariance kernels do,
// and that fp32 value is split exactly into three bf16 parts (hi, then the
// rounded remainder, then the rest: 8 + 8 + 8 bits of the 24); each part's
// product with V is exact in fp32 and the three (twelve K = 16 MMAs) add into
// the accumulator.  Two ring stages leave room for the two extra parts' tiles.
#pragma once
#include "common.cuh"

namespace sla {

constexpr int kKvTok = 64;     // tokens per KV block (Bk)
constexpr int kKvStages = 3;

__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&x);
    h = __hmax2(h, __floats2bfloat162_rn(0.f, 0.f));
    return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of element (row n, col c) in a [64][D] bf16 tile.  TC (the tile
// is a tensor-core operand): D/64 halves of 64 rows x 128 bytes, whose 16-byte
// chunks are XOR-swizzled by (n & 7) within each 128-byte row (the 128-byte
// swizzle of the operand descriptors; halves are 8 KB apart).  Otherwise rows
// of 2D bytes whose 16-byte chunks are XOR-swizzled by (n & 7).
template <int D, bool TC>
__device__ __forceinline__ uint32_t kv_off(int n, int c) {
    if (TC)
        return static_cast<uint32_t>((c >> 6) * (kKvTok * 128) + n * 128 +
                                     ((((c >> 3) & 7) ^ (n & 7)) << 4) + (c & 7) * 2);
    return static_cast<uint32_t>(n * D * 2 + (((c >> 3) ^ (n & 7)) << 4) + (c & 7) * 2);
}

// the three bf16 parts of x: hi + mid + lo == x exactly (x fp32; each
// remainder is exact in fp32 and the last has at most 8 significant bits)
__device__ __forceinline__ void split3_bf16(float x, float& hi, float& mid, float& lo) {
    hi = __bfloat162float(__float2bfloat16_rn(x));
    const float r1 = x - hi;
    mid = __bfloat162float(__float2bfloat16_rn(r1));
    lo = __bfloat162float(__float2bfloat16_rn(r1 - mid));
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
    // (k_n - kbar_j), instead of phi(K), so hpart sums the blocks' H_j (in the
    // X3 kernel exactly, from fp64-centred keys split into three bf16 parts)
    int center;
    // with k8: symmetric 8-bit integer K codes (absmax / 127) instead of e4m3
    int k_int8;
    unsigned long long wait_ns;  // limit of the bounded waits on the tensor-core product
};

// grid (nchunk, BH), 256 threads.  TC: the call wants the tensor-core product
// (hpart non-null); without it the tiles keep a plain swizzled row layout.
// X3 (with TC and center): the exact three-part product, two ring stages.
template <int D, bool TC, bool X3 = false>
__global__ void __launch_bounds__(256, 2) kv_stats_kernel(KvStatsArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr int TILE = kKvTok * D * 2;               // bytes of one K or V tile
    constexpr int kKvStages = X3 ? 2 : ::sla::kKvStages;
    // the swizzled tiles need a 1024-byte aligned base (the launch adds 1024 bytes)
    unsigned char* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    unsigned char* xpart = ring + kKvStages * 2 * TILE;                            // X3: [2] tiles
    double* kpart = reinterpret_cast<double*>(xpart + (X3 ? 2 * TILE : 0));         // [256]
    float* zpart = reinterpret_cast<float*>(kpart + 256);                          // [256]
    float* vpart = zpart + 256;                                                    // [256]
    float* amax = vpart + 256;                                                     // [2][8]
    float* kmf = amax + 16;                                                        // [D] column means
    double* kmd = reinterpret_cast<double*>(kmf + 128);                            // X3: [D] fp64 means
    uint64_t* mma_bar = reinterpret_cast<uint64_t*>(kmd + (X3 ? D : 0));           // product done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

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
            const uint32_t off = kv_off<D, TC>(n, u * 8);
            cp_async16(kd + off, kh + (row0 + n) * D + u * 8);
            if (want_v) cp_async16(vd + off, vh + (row0 + n) * D + u * 8);
        }
    };

    // The D x D product accumulates in tensor memory: lane m = feature of the
    // left operand, column n = feature of V.  (D = 64: an M = 128 product whose
    // rows 64-127 repeat rows 0-63.)
    const bool do_mma = TC && a.hpart != nullptr;
    constexpr uint32_t TCOLS = D;                       // 64 or 128 columns
    constexpr uint32_t ID_H = idesc_bf16(128, D, 1, 1);
    uint32_t tmem = 0;
    if (do_mma) {
        if (warp == 0) {
            tmem_alloc(tmem_slot, TCOLS);
            tmem_relinquish();
        }
        if (tid == 0) {
            mbar_init(mma_bar, 1);
            *abort_flag = 0;
            fence_barrier_init();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        tmem = *tmem_slot;
    }

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
        unsigned char* kt = ring + stage * 2 * TILE;
        const unsigned char* vt = kt + TILE;
        // without the product, the stage of the previous block is free now:
        // prefetch kKvStages-1 blocks ahead right away
        if (!do_mma) {
            const int nb = blk + kKvStages - 1;
            if (nb < nblk) load_block(nb, nb % kKvStages);
            cp_async_commit();
        }

        // column statistics of this block
        {
            double ks = 0.0;
            float zs = 0.f, vs = 0.f, kmax = 0.f;
            for (int n = half * RPH; n < (half + 1) * RPH; ++n) {
                const float kv = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(kt + kv_off<D, TC>(n, col)));
                ks += static_cast<double>(kv);
                zs += fmaxf(kv, 0.f);
                kmax = fmaxf(kmax, fabsf(kv));
                if (want_v)
                    vs += __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D, TC>(n, col)));
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
                        *reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D, TC>(n, col)))));
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
                const uint4 x = *reinterpret_cast<const uint4*>(vt + kv_off<D, TC>(n, u * 8));
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
            // dequantisation scales; each code rounds the exact quotient top x / absmax
            const float s_k = km > 0.f ? km / (a.k_int8 ? 127.f : 448.f) : 1.f;
            const float s_v = vm > 0.f ? vm / 448.f : 1.f;
            const CodeQuot ck(km, a.k_int8 ? 127.f : 448.f), cv(vm, 448.f);
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
                const uint4 x = *reinterpret_cast<const uint4*>(kt + kv_off<D, TC>(n, u * 8));
                uint32_t w0, w1;
                if (a.k_int8) {
                    w0 = pack_s8x4(ck(bf16lo(x.x)), ck(bf16hi(x.x)), ck(bf16lo(x.y)), ck(bf16hi(x.y)));
                    w1 = pack_s8x4(ck(bf16lo(x.z)), ck(bf16hi(x.z)), ck(bf16lo(x.w)), ck(bf16hi(x.w)));
                } else {
                    w0 = pack_e4m3x4(ck(bf16lo(x.x)), ck(bf16hi(x.x)), ck(bf16lo(x.y)), ck(bf16hi(x.y)));
                    w1 = pack_e4m3x4(ck(bf16lo(x.z)), ck(bf16hi(x.z)), ck(bf16lo(x.w)), ck(bf16hi(x.w)));
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
                    f[t] = cv(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(vt + kv_off<D, TC>(n0 + t, c))));
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
                const uint4 x = *reinterpret_cast<const uint4*>(kt + kv_off<D, TC>(n, u * 8));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                uint32_t h[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    h[e] = pack_half2(fmaxf(bf16lo(w[e]), 0.f), fmaxf(bf16hi(w[e]), 0.f));
                *reinterpret_cast<uint4*>(ko + (row0 + n) * D + u * 8) = make_uint4(h[0], h[1], h[2], h[3]);
            }
        }

        // every raw read of this K tile is done, the column partials are in
        // shared memory, and (thread 0) the previous block's product has
        // completed, so its ring stage may be refilled
        if (do_mma && blk > 0 && tid == 0 && !*abort_flag &&
            !mbar_wait(mma_bar, (blk - 1) & 1, abort_flag, a.wait_ns)) {
            report(kStatusTimeout);
            *abort_flag = 1;
        }
        __syncthreads();
        const bool dead = do_mma && *abort_flag;
        if (do_mma) {   // the previous block's product is done: refill its stage
            const int nb = blk + kKvStages - 1;
            if (nb < nblk && !dead) load_block(nb, nb % kKvStages);
            cp_async_commit();
        }
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
            kmf[tid] = static_cast<float>(kmean);
            if (X3) kmd[tid] = kmean;
        }
        if (do_mma && a.center) __syncthreads();        // the column means, for the centring
        if (do_mma && !dead) {
            // the product's left operand in place: phi(K) = max(K, 0), or the keys
            // centred by this block's column means (bf16)
            constexpr int CPR = D / 8;
            for (int q = tid; q < kKvTok * CPR; q += 256) {
                const int n = q / CPR, u = q % CPR;
                uint4* px = reinterpret_cast<uint4*>(kt + kv_off<D, TC>(n, u * 8));
                uint4 x = *px;
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
                if (X3) {
                    // fp64-centred keys, rounded once to fp32, as three bf16 parts
                    uint32_t wm[4], wl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float h0, m0, l0, h1, m1, l1;
                        split3_bf16(static_cast<float>(static_cast<double>(bf16lo(w[e])) - kmd[u * 8 + 2 * e]), h0, m0, l0);
                        split3_bf16(static_cast<float>(static_cast<double>(bf16hi(w[e])) - kmd[u * 8 + 2 * e + 1]), h1, m1, l1);
                        w[e] = pack_bf16(h0, h1);
                        wm[e] = pack_bf16(m0, m1);
                        wl[e] = pack_bf16(l0, l1);
                    }
                    const uint32_t off = kv_off<D, TC>(n, u * 8);
                    *reinterpret_cast<uint4*>(xpart + off) = make_uint4(wm[0], wm[1], wm[2], wm[3]);
                    *reinterpret_cast<uint4*>(xpart + TILE + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
                } else if (a.center) {
                    const float4 m0 = *reinterpret_cast<const float4*>(kmf + u * 8);
                    const float4 m1 = *reinterpret_cast<const float4*>(kmf + u * 8 + 4);
                    w[0] = pack_bf16(bf16lo(w[0]) - m0.x, bf16hi(w[0]) - m0.y);
                    w[1] = pack_bf16(bf16lo(w[1]) - m0.z, bf16hi(w[1]) - m0.w);
                    w[2] = pack_bf16(bf16lo(w[2]) - m1.x, bf16hi(w[2]) - m1.y);
                    w[3] = pack_bf16(bf16lo(w[3]) - m1.z, bf16hi(w[3]) - m1.w);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[e] = relu_bf16x2(w[e]);
                }
                *px = make_uint4(w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();
        }
        __syncthreads();
        if (do_mma && !dead && tid == 0) {
            tc_fence_after();
            const uint32_t kt_s = smem_u32(kt), vt_s = smem_u32(vt), xp_s = smem_u32(xpart);
            const uint32_t lbo = D == 128 ? kKvTok * 128 : 0;     // the second 64-feature half
#pragma unroll
            for (int part = 0; part < (X3 ? 3 : 1); ++part) {
                const uint32_t a_s = part == 0 ? kt_s : xp_s + (part - 1) * TILE;
#pragma unroll
                for (int kk = 0; kk < kKvTok / 16; ++kk) {
                    const uint64_t ad = sdesc(a_s + kk * 2048, lbo, 1024, kSwizzle128B);
                    const uint64_t bd = sdesc(vt_s + kk * 2048, kKvTok * 128, 1024, kSwizzle128B);
                    umma_f16_ss(tmem, ad, bd, ID_H, (blk > 0 || part > 0 || kk > 0) ? 1u : 0u);
                }
            }
            umma_commit(mma_bar);
        }
    }
    cp_async_wait<0>();

    if (do_mma) {
        // the last product, then the accumulator to this chunk's partial
        if (tid == 0 && !*abort_flag && !mbar_wait(mma_bar, (nblk - 1) & 1, abort_flag, a.wait_ns)) {
            report(kStatusTimeout);
            *abort_flag = 1;
        }
        __syncthreads();
        tc_fence_after();
        if (!*abort_flag && warp < D / 32) {
            float* hp = a.hpart + (bh * a.nchunk + chunk) * static_cast<long long>(D) * D;
            const int r = warp * 32 + lane;                  // feature row of H
            const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
            for (int cc = 0; cc < D; cc += 32) {
                uint32_t v[32];
                tmem_ld32(tl + cc, v);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4*>(hp + r * D + cc + x) =
                        make_float4(__uint_as_float(v[x]), __uint_as_float(v[x + 1]),
                                    __uint_as_float(v[x + 2]), __uint_as_float(v[x + 3]));
            }
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, TCOLS);
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
// block (absmax / 448, or absmax / 127); codes round top x / absmax.
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
        // dequantisation scale; each code rounds the exact quotient top x / absmax
        const float s = am > 0.f ? am / (I8 ? 127.f : 448.f) : 1.f;
        const CodeQuot cq(am, I8 ? 127.f : 448.f);
        if (tid == 0) sq[blk] = s;
        uint2* dst = reinterpret_cast<uint2*>(q8 + blk * 64 * D);
        auto pack = [](float a0, float a1, float a2, float a3) {
            return I8 ? pack_s8x4(a0, a1, a2, a3) : pack_e4m3x4(a0, a1, a2, a3);
        };
#pragma unroll
        for (int i = 0; i < VEC; ++i)
            dst[i * 256 + tid] = make_uint2(
                pack(cq(bf16lo(x[i].x)), cq(bf16hi(x[i].x)), cq(bf16lo(x[i].y)), cq(bf16hi(x[i].y))),
                pack(cq(bf16lo(x[i].z)), cq(bf16hi(x[i].z)), cq(bf16lo(x[i].w)), cq(bf16hi(x[i].w))));
        __syncthreads();
    }
}

}  // namespace sla

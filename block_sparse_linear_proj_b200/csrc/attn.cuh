// attn.cuh -- block-sparse attention on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA owns up to 128 query rows = GR query blocks ("groups") of one head
// (GR = 128/Bq, except the SLA mode with d = 128, where GR = 1 so that the
// per-group G accumulators fit in tensor memory).  It walks the union of its
// groups' selected KV blocks (each entry tagged with the groups that selected
// it; the walk starts at a per-tile rotation of the ascending order) and, in
// PISA mode, then the head's centroid pseudo-tiles.  The query tile stays in
// shared memory; tensor memory holds S_0 | S_1 | O_0 | O_1 | G.  Entry e goes
// to softmax warpgroup h = e % 2, which owns S buffer h, accumulator O_h and
// its own running maximum and row sum:
//   S  = Q K_e^T                        tcgen05.mma M=128 N=64, A and B from shared memory
//   P  = 2^(S*tau*log2e - m_h)          warpgroup h, one row per thread, online max with
//                                       lazy rescale of O_h; packed fp16 exp2 (e4m3 in
//                                       FP8 mode), written over the first columns of S_h
//   O_h += P V_e                        tcgen05.mma M=128 N=d, A (P) from tensor memory
//   G_g -= phi(K_e)^T V_e  (SLA only)   tcgen05.mma M=128 N=d, per group; G_g starts as H
// S(e) is issued only after P.V(e-2) has completed (P(e-2) sits in S buffer h),
// so each softmax step waits on one barrier and O_h needs no extra wait before
// a rescale.  The epilogue merges the two partial softmaxes per row.
// Linear branch (SALAD ReLU kernel; SLA2 combine): after the loop,
//   O_l = phi(Q) (H - G_g) / (phi(q) . (Z - sum_{j in S_g} z_j))
// with (H - G_g) split into bf16 hi + lo and multiplied on the tensor core
// (phi(Q) formed over the query tile in shared memory), then
// out = alpha O_s + (1 - alpha) O_l.
// PISA (zero-order "exact-or-approximate"): a centroid pseudo-tile holds 64
// block centroids kbar_j and value means vbar_j; its logits get + log2(Bk)
// (the block multiplicity) and the groups' own selected blocks are masked, so
// e^{q.kbar_j - m} (sum_n v_n) enters N_t and Bk e^{q.kbar_j - m} enters D_t in
// the same online softmax; out = N_t / D_t.  With the global first-order term,
// tau (q . Hbar) sum_U e^{q.kbar_j - m} is added to N_t in the epilogue (q . Hbar
// on the tensor core, the centroid sum tracked next to the row sum).
//
// K tiles and V (+ phi(K)) tiles stream through two separate rings: a K slot is
// released as soon as S of its block completes, so K loads run ahead of the
// P.V / G products.
// Warp roles (384 threads): w0 TMA producer for both rings (thread 0 also starts
// the query-tile load at set-up), w1 issues S = Q K^T (and owns TMEM), w3 issues
// P.V, the G updates and the epilogue products (two issuers, so one's barrier
// waits overlap the other's MMAs: an MMA issue blocks until the tensor pipe
// takes it), w2 the per-group sums of z_j and the linear-branch denominators
// (SLA), w4-11 the two softmax warpgroups and the epilogue.  Every wait is
// bounded; a wait that runs out sets the device status word and the CTA
// unwinds after draining its own TMA loads and MMAs.
#pragma once
#include "common.cuh"

namespace sla {

constexpr float kRescaleLog2 = 8.0f;    // lazy O rescale threshold (log2 units)

enum : int { kModeSla = 0, kModePisa = 1, kModeSlaFp8 = 2, kModeSlaInt8 = 3 };

// Tensor maps of one launch (see the host for shapes, boxes and swizzles).
struct AttnMaps {
    CUtensorMap q;      // bf16 Q [BH*N, d], box 64 x 128 rows
    CUtensorMap k;      // K tiles: bf16 K (box 64 x 64) or, FP8, e4m3 K (box 128 B x 64)
    CUtensorMap v;      // fp16 V copy, box 64 x 64
    CUtensorMap phi;    // fp16 phi(K), box 64 x 64
    CUtensorMap kc;     // PISA centroids (bf16 [BH*Nk, d])
    CUtensorMap vc;     // PISA value means (fp16 [BH*Nk, d])
    CUtensorMap out;    // output, box 128 B x 64 rows
    CUtensorMap q8;     // FP8: e4m3 Q, box 128 B x 128 rows
    CUtensorMap v8t;    // FP8: e4m3 V^T per block [BH*Nk*d, 64], box 64 B x d, 64-byte swizzle
};

struct AttnArgs {
    int N, Nq, Nk, Bq, GR, topk, tiles_per_head;
    float scale_log2;              // tau * log2(e)
    float log2_bk;                 // log2(Bk), PISA pseudo-tile bias
    const int32_t* lut;            // [BH][Nq][topk]
    const float* alpha;            // [BH][N]        (SLA)
    const float* hsum;             // [BH][D][D]     (SLA), transposed: H^T[e][c]
    const float* zsum;             // [BH][D]        (SLA)
    const float* zj;               // [BH][Nk][D]    (SLA)
    void* out;                     // [BH][N][D] bf16 or fp32
    int out_f32;
    int lut_sorted;                // LUT rows strictly ascending and in range (router output)
    int sched_cap;                 // capacity of the shared-memory schedule
    const float* sq;               // FP8: [BH][N/64] Q block scales
    const float* sk;               // FP8: [BH][Nk]  K block scales
    const float* sv;               // FP8: [BH][Nk]  V block scales
    unsigned long long wait_ns;
    int debug_stall;               // test hook: load no K/V tiles, so the consumers' waits run out
    // PISA global first-order term: + fo_scale * (sum of the centroid P) * (q . Hsum)
    // with Hsum = sum_j H_j stored transposed [BH][D][D], fo_scale = tau / (Nk * Bk)
    int first_order;
    const float* hbar;
    float fo_scale;
};

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^x for two fp16 values at once (one MUFU operation).
__device__ __forceinline__ uint32_t exp2_h2(uint32_t x) {
    uint32_t y;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t hadd2_u(uint32_t a, uint32_t b) {
    __half2 r = __hadd2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// P = 2^(x - m) for the 32 logits sv[OFF .. OFF+31] as 16 packed fp16 pairs;
// returns their sum.  EXACT: sv holds raw scores (x = s*c), else x itself.
// Rows with nothing to add (!live) get P = 0.  PACKED forms the arguments two at
// a time with the packed fp32 FMA and handles !live rows through m = +inf (every
// P exactly +0); the two forms give identical results, and each is faster in one
// mode of the kernel (PACKED in the PISA mode).
template <int OFF, bool EXACT, bool PACKED>
__device__ __forceinline__ float softmax_half(const uint32_t (&sv)[64], float c, float m, bool live,
                                              uint32_t (&pw)[16]) {
    const float mp = (PACKED && !live) ? INFINITY : m;
    const uint64_t c2 = f2pack(EXACT ? c : 1.f, EXACT ? c : 1.f), nm2 = f2pack(-mp, -mp);
    float ls = 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int j = OFF + ch * 8 + 2 * x;
            float x0, x1;
            if (PACKED) {
                f2unpack(ffma2(f2pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2, nm2), x0, x1);
                pw[4 * ch + x] = exp2_h2(pack_half2(x0, x1));
            } else {
                if (EXACT) {
                    x0 = fmaf(__uint_as_float(sv[j]), c, -m);
                    x1 = fmaf(__uint_as_float(sv[j + 1]), c, -m);
                } else {
                    x0 = __uint_as_float(sv[j]) - m;
                    x1 = __uint_as_float(sv[j + 1]) - m;
                }
                pw[4 * ch + x] = live ? exp2_h2(pack_half2(x0, x1)) : 0u;
            }
        }
        const uint32_t s4 = hadd2_u(hadd2_u(pw[4 * ch], pw[4 * ch + 1]), hadd2_u(pw[4 * ch + 2], pw[4 * ch + 3]));
        ls += half_lo(s4) + half_hi(s4);
    }
    return ls;
}

// FP8 P for the 32 logits sv[OFF .. OFF+31] (raw scores, x = s*ce): fp32 exp2,
// quantised as e4m3(P * qf) four per 32-bit word; returns the fp32 sum of P.
template <int OFF>
__device__ __forceinline__ float softmax_half_e4m3(const uint32_t (&sv)[64], float ce, float m, bool live,
                                                   float qf, uint32_t (&p8)[8]) {
    float ls = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        float p[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            p[x] = live ? fast_exp2(fmaf(__uint_as_float(sv[OFF + 4 * w + x]), ce, -m)) : 0.f;
            ls += p[x];
        }
        p8[w] = pack_e4m3x4(p[0] * qf, p[1] * qf, p[2] * qf, p[3] * qf);
    }
    return ls;
}

// Stage 32 consecutive output values of row r (columns cc .. cc+31) in shared
// memory for the tensor store: boxes of 128-byte rows (64 bf16 or 32 fp32
// columns), 128 rows each, 128-byte swizzle.
__device__ __forceinline__ void stage_row32(unsigned char* stage, int f32, int r, int cc,
                                            const float (&v)[32]) {
    if (f32) {
        unsigned char* box = stage + (cc >> 5) * 16384;
#pragma unroll
        for (int x = 0; x < 8; ++x)
            *reinterpret_cast<float4*>(box + sw128(r, x)) =
                make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
    } else {
        unsigned char* box = stage + (cc >> 6) * 16384;
        const int c0 = (cc & 63) >> 3;
#pragma unroll
        for (int x = 0; x < 4; ++x)
            *reinterpret_cast<uint4*>(box + sw128(r, c0 + x)) =
                make_uint4(pack_bf16(v[8 * x], v[8 * x + 1]), pack_bf16(v[8 * x + 2], v[8 * x + 3]),
                           pack_bf16(v[8 * x + 4], v[8 * x + 5]), pack_bf16(v[8 * x + 6], v[8 * x + 7]));
    }
}

template <int D, int MODE>
struct AttnLayout {
    // INT8 shares every FP8 rule except the Q and K codes and the S product
    static constexpr bool PISA = MODE == kModePisa, I8 = MODE == kModeSlaInt8;
    static constexpr bool FP8 = MODE == kModeSlaFp8 || I8;
    static constexpr int KS = PISA ? (D == 128 ? 5 : 6) : (FP8 ? 6 : 4);   // K ring slots
    static constexpr int VS = PISA ? (D == 128 ? 5 : 6) : (D == 128 ? 3 : 4);  // V ring slots
    static constexpr int T16 = 64 * D * 2;            // one 64-token tile of 16-bit values
    static constexpr int KT = 64 * D * (FP8 ? 1 : 2);    // one K tile
    // V slot: [P.V operand | fp16 phi(K) | fp16 V (FP8: the G operand)]
    static constexpr int V_PV = 0;
    static constexpr int V_PHI = FP8 ? 64 * D : T16;
    static constexpr int V_V16 = FP8 ? 64 * D + T16 : 0;
    static constexpr int VT = PISA ? T16 : (FP8 ? 64 * D + 2 * T16 : 2 * T16);
    static constexpr int KBOX = 64 * 128;             // one 64-row x 128-byte box
    static constexpr int QBOX = 128 * 128;            // one 128-row x 128-byte box
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KS * KT;
    // the query tile stays in shared memory for the whole CTA: e4m3 Q (FP8), bf16 Q
    static constexpr int OFF_Q8 = OFF_V + VS * VT;
    static constexpr int OFF_Q = OFF_Q8 + (FP8 ? 128 * D : 0);
    static constexpr int QB = 128 * D * (FP8 ? 3 : 2);   // bytes of the query-tile load
    static constexpr int OFF_MISC = OFF_Q + 128 * D * 2;
    static constexpr int GRMAX = D == 128 ? 1 : 2;    // query blocks per CTA (SLA mode)
    static constexpr int BBUF = D * D * 2;            // one (H - G) hi or lo buffer
    static constexpr int BBOX = D * 128;              // one 64-column box of it
    // epilogue buffers reuse the rings: (H - G) hi/lo (PISA: Hsum hi/lo for the
    // first-order term), then the output staging
    static constexpr int OUT_OFF = OFF_K + 2 * (PISA ? 1 : GRMAX) * BBUF;
    static_assert(OUT_OFF + D * 4 * 128 <= OFF_Q8, "epilogue buffers fit in the K/V rings");
};

constexpr int kAttnThreads = 384;

template <int D, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ AttnMaps tm, const AttnArgs a) {
    using L = AttnLayout<D, MODE>;
    constexpr bool PISA = L::PISA, FP8 = L::FP8, I8 = L::I8;
    constexpr bool SLA = !PISA;
    constexpr int NBOX = D / 64;
    constexpr int KS = L::KS, VS = L::VS;
    // tensor memory columns: S_0 | S_1 | O_0 | O_1 | G_0 (| G_1 when d = 64).
    // SLA: P(e) is written over the first columns of its S buffer (packed fp16
    // pairs, or e4m3 quads in FP8 mode).  PISA (no G): P(e) has buffers of its own,
    // P_0 | P_1 after O_1, so S(e+2) may overwrite S buffer h as soon as the
    // softmax has read S(e), while P.V(e) still reads P(e).
    constexpr uint32_t NCOLS = 512;
    constexpr uint32_t COL_O = 128;                   // + h * D
    constexpr uint32_t COL_G0 = 128 + 2 * D;          // + g * D
    constexpr uint32_t COL_P = 128 + 2 * D;           // PISA: + h * 32
    static_assert(PISA || COL_G0 + L::GRMAX * D <= NCOLS, "tensor memory budget");
    static_assert(!PISA || COL_P + 64 <= NCOLS, "tensor memory budget");

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);

    // misc region
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_MISC);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;                  // [KS]
    uint64_t* k_empty = k_full + KS;              // [KS]
    uint64_t* v_full = k_empty + KS;              // [VS]
    uint64_t* v_empty = v_full + VS;              // [VS]
    uint64_t* s_full = v_empty + VS;              // [2] S(e) in buffer e & 1
    uint64_t* p_full = s_full + 2;                // [2] P(e) written (4 warps)
    uint64_t* pv_done = p_full + 2;               // [2] P.V(e) complete: buffer free, O_{e&1} current
    uint64_t* s_free = pv_done + 2;               // [2] PISA: S(e) read by the softmax (4 warps)
    uint64_t* final_bar = s_free + 2;
    uint64_t* epi_ready = final_bar + 1;
    uint64_t* lin_done = epi_ready + 1;
    uint64_t* drain_bar = lin_done + 1;
    uint64_t* drain2_bar = drain_bar + 1;
    uint64_t* g_init = drain2_bar + 1;            // G accumulators preloaded with H
    uint64_t* xl_bar = g_init + 1;                // [4] exchanges between the two warpgroups
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xl_bar + 4);
    int* n_exact_s = reinterpret_cast<int*>(tmem_slot + 1);
    volatile int* abort_flag = n_exact_s + 1;
    int* g_any = n_exact_s + 2;                   // [2] group selected >= 1 block
    float* svmax_s = reinterpret_cast<float*>(g_any + 2);
    float* zu = reinterpret_cast<float*>(smem + L::OFF_MISC + 384);       // [2][D]
    float* xm = zu + 2 * D;                                              // [2][128] row maxima
    float* xl = xm + 256;                                                // [2][128] row sums
    float* xd = xl + 256;                                                // [128] linear-branch denominators
    uint32_t* mark = reinterpret_cast<uint32_t*>(xd + 256);              // [ceil(Nk/16)]
    const int nwords = (a.Nk + 15) >> 4;
    int32_t* sched = reinterpret_cast<int32_t*>(mark + ((nwords + 3) & ~3));
    float* ent_sk = reinterpret_cast<float*>(sched + a.sched_cap);       // FP8: per-entry K scale
    float* ent_sv = ent_sk + a.sched_cap;                                // FP8: per-entry V scale

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / a.tiles_per_head;
    const int tile = blockIdx.x % a.tiles_per_head;
    const int GR = a.GR;
    const int qb0 = tile * GR;
    const int row0 = qb0 * a.Bq;                  // first token of the tile
    const int n_groups = min(GR, a.Nq - qb0);

    // ------------------------------------------------------------ set-up
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 4);
            mbar_init(&pv_done[b], 1);
            mbar_init(&s_free[b], 4);
        }
        mbar_init(final_bar, 1);
        mbar_init(epi_ready, 9);
        mbar_init(lin_done, 1);
        mbar_init(drain_bar, 1);
        mbar_init(drain2_bar, 1);
        mbar_init(g_init, 8);
        for (int x = 0; x < 4; ++x) mbar_init(&xl_bar[x], 2);
        *abort_flag = 0;
        fence_barrier_init();
        // the query tile does not depend on the schedule: start its load now, so
        // that it overlaps the set-up below (no role waits on q_full before the
        // CTA-wide barrier that follows the set-up)
        prefetch_tmap(&tm.q);
        if (FP8) prefetch_tmap(&tm.q8);
        const int qrow = bh * a.N + row0;
        mbar_arrive_expect_tx(q_full, L::QB);
        if (FP8) tma_load_2d(smem + L::OFF_Q8, &tm.q8, q_full, 0, qrow);
        for (int b = 0; b < NBOX; ++b)
            tma_load_2d(smem + L::OFF_Q + b * L::QBOX, &tm.q, q_full, b * 64, qrow);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, NCOLS);
        tmem_relinquish();
    }
    // Schedule.  Router-made LUT rows are ascending, distinct and in range: with one
    // group per CTA the row is the schedule.  Otherwise the groups' rows are merged
    // (and checked) through a per-block bit mask.
    const bool fast = a.lut_sorted && GR == 1;
    if (fast) {
        if (warp == 0) {
            const int cnt = a.topk;
            const int rot = cnt > 0 ? static_cast<int>((static_cast<unsigned>(tile) * 2654435761u >> 7) % cnt) : 0;
            const int32_t* row = a.lut + (static_cast<long long>(bh) * a.Nq + qb0) * a.topk;
            for (int x = lane; x < cnt; x += 32) {
                int at = x - rot;
                if (at < 0) at += cnt;
                sched[at] = row[x] | (1 << 16);
            }
            if (lane == 0) {
                *n_exact_s = cnt;
                g_any[0] = cnt > 0;
                g_any[1] = 0;
            }
        }
    } else {
    for (int w = tid; w < nwords; w += kAttnThreads) mark[w] = 0u;
    __syncthreads();
    for (int x = tid; x < n_groups * a.topk; x += kAttnThreads) {
        const int g = x / a.topk;
        const int j = a.lut[(static_cast<long long>(bh) * a.Nq + qb0 + g) * a.topk + x % a.topk];
        if (j < 0 || j >= a.Nk) { report(kStatusBadData); continue; }
        const uint32_t bit = (1u << g) << (2 * (j & 15));
        const uint32_t old = atomicOr(&mark[j >> 4], bit);
        if (old & bit) report(kStatusBadData);
    }
    __syncthreads();
    if (warp == 0) {
        // count, then write the selected blocks in ascending order rotated by a
        // per-tile offset: the CTAs of one head (which run concurrently) then
        // start their walks at different KV blocks instead of all requesting
        // the same tiles from L2 at the same moment
        int cnt = 0;
        uint32_t any = 0u;
        const uint32_t lt = (1u << lane) - 1u;
        for (int j0 = 0; j0 < a.Nk; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t bits = j < a.Nk ? (mark[j >> 4] >> (2 * (j & 15))) & 3u : 0u;
            cnt += __popc(__ballot_sync(0xffffffffu, bits != 0u));
            any |= bits;
        }
        const int rot = cnt > 0 ? static_cast<int>((static_cast<unsigned>(tile) * 2654435761u >> 7) % cnt) : 0;
        int pos = 0;
        for (int j0 = 0; j0 < a.Nk; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t bits = j < a.Nk ? (mark[j >> 4] >> (2 * (j & 15))) & 3u : 0u;
            const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
            if (bits) {
                int at = pos + __popc(bal & lt) - rot;
                if (at < 0) at += cnt;
                sched[at] = j | static_cast<int>(bits << 16);
            }
            pos += __popc(bal);
        }
        any = __reduce_or_sync(0xffffffffu, any);
        if (lane == 0) {
            *n_exact_s = cnt;
            g_any[0] = any & 1u;
            g_any[1] = (any >> 1) & 1u;
        }
    }
    }
    if (FP8 && warp == 0) {
        // per-entry K and V scales; the V scales' maximum fixes the P quantisation
        __syncwarp();
        const int cnt = *n_exact_s;
        float vm = 0.f;
        for (int e = lane; e < cnt; e += 32) {
            const int j = sched[e] & 0xFFFF;
            ent_sk[e] = a.sk[static_cast<long long>(bh) * a.Nk + j];
            ent_sv[e] = a.sv[static_cast<long long>(bh) * a.Nk + j];
            vm = fmaxf(vm, ent_sv[e]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
        if (lane == 0) *svmax_s = vm > 0.f ? vm : 1.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_exact = *n_exact_s;
    const int n_cent = PISA ? (a.Nk + 63) / 64 : 0;
    const int n_total = n_exact + n_cent;
    const unsigned long long lim = a.wait_ns;
    const unsigned long long drain_lim = 4000000000ull;

    auto sK = [&](int s) { return sbase + L::OFF_K + s * L::KT; };
    auto sV = [&](int s) { return sbase + L::OFF_V + s * L::VT; };
    auto sPhi = [&](int s) { return sbase + L::OFF_V + s * L::VT + L::V_PHI; };
    auto sV16 = [&](int s) { return sbase + L::OFF_V + s * L::VT + L::V_V16; };
    // K-major 128-byte-swizzled descriptor of the query tile (bf16) at K-step kk (16 columns)
    auto qdesc = [&](int kk) {
        return sdesc(sbase + L::OFF_Q + (kk >> 2) * L::QBOX + (kk & 3) * 32, 16, 1024, kSwizzle128B);
    };

    auto fail = [&]() {
        *abort_flag = 1;
        report(kStatusTimeout);
    };

    if (warp == 0) {
        // ======================================================== TMA producer
        // Two rings, one thread: issue whichever pending load is needed first and
        // has a free slot.  K(e) is consumed by S(e), which runs about two blocks
        // ahead of P.V(e), so K(kn) goes first while kn <= vn + 2.
        if (lane == 0) {
            prefetch_tmap(&tm.k);
            prefetch_tmap(&tm.v);
            if (SLA) prefetch_tmap(&tm.phi);
            if (PISA) { prefetch_tmap(&tm.kc); prefetch_tmap(&tm.vc); }
            if (FP8) prefetch_tmap(&tm.v8t);
            int kn = 0, vn = 0;
            const int n_load = a.debug_stall ? 0 : n_total;
            unsigned long long t0 = globaltimer_ns();
            uint32_t idle = 0;
            while (kn < n_load || vn < n_load) {
                bool did = false;
                const bool want_k = kn < n_load && (vn >= n_load || kn <= vn + 2);
                if (want_k) {
                    const int s = kn % KS, r = kn / KS;
                    if (mbar_ready(&k_empty[s], (r & 1) ^ 1)) {
                        mbar_arrive_expect_tx(&k_full[s], L::KT);
                        unsigned char* kd = smem + L::OFF_K + s * L::KT;
                        if (kn < n_exact) {
                            const int row = bh * a.N + (sched[kn] & 0xFFFF) * 64;
                            if (FP8) tma_load_2d(kd, &tm.k, &k_full[s], 0, row);
                            else for (int b = 0; b < NBOX; ++b) tma_load_2d(kd + b * L::KBOX, &tm.k, &k_full[s], b * 64, row);
                        } else {
                            const int row = bh * a.Nk + (kn - n_exact) * 64;
                            for (int b = 0; b < NBOX; ++b) tma_load_2d(kd + b * L::KBOX, &tm.kc, &k_full[s], b * 64, row);
                        }
                        ++kn;
                        did = true;
                    }
                }
                if (!did && vn < n_load) {
                    const int s = vn % VS, r = vn / VS;
                    if (mbar_ready(&v_empty[s], (r & 1) ^ 1)) {
                        mbar_arrive_expect_tx(&v_full[s], L::VT);
                        unsigned char* vd = smem + L::OFF_V + s * L::VT;
                        if (vn < n_exact) {
                            const int j = sched[vn] & 0xFFFF;
                            const int row = bh * a.N + j * 64;
                            if (FP8) tma_load_2d(vd + L::V_PV, &tm.v8t, &v_full[s], 0, (bh * a.Nk + j) * D);
                            for (int b = 0; b < NBOX; ++b) {
                                if (SLA) tma_load_2d(vd + L::V_PHI + b * L::KBOX, &tm.phi, &v_full[s], b * 64, row);
                                tma_load_2d(vd + (FP8 ? L::V_V16 : L::V_PV) + b * L::KBOX, &tm.v, &v_full[s], b * 64, row);
                            }
                        } else {
                            const int row = bh * a.Nk + (vn - n_exact) * 64;
                            for (int b = 0; b < NBOX; ++b) tma_load_2d(vd + b * L::KBOX, &tm.vc, &v_full[s], b * 64, row);
                        }
                        ++vn;
                        did = true;
                    }
                }
                if (did) {
                    idle = 0;
                    t0 = globaltimer_ns();
                } else if (++idle >= 64) {
                    idle = 0;
                    if (*abort_flag || globaltimer_ns() - t0 > lim) { fail(); break; }
                }
            }
            // drain: every load this thread issued has landed before the CTA exits
            mbar_wait(q_full, 0, abort_flag, drain_lim);
            for (int e = max(0, kn - KS); e < kn; ++e)
                mbar_wait(&k_full[e % KS], (e / KS) & 1, abort_flag, drain_lim);
            for (int e = max(0, vn - VS); e < vn; ++e)
                mbar_wait(&v_full[e % VS], (e / VS) & 1, abort_flag, drain_lim);
        }
    } else if (warp == 1) {
        // ======================================================== S = Q K^T issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = I8 ? idesc_s8(128, 64) : FP8 ? idesc_e4m3(128, 64) : idesc_bf16(128, 64, 0, 0);
            bool ok = mbar_wait(q_full, 0, abort_flag, lim);
            for (int e = 0; ok && e < n_total; ++e) {
                // S(e) needs its K tile and its buffer back: SLA, P(e-2), written over
                // S(e-2), has been consumed once P.V(e-2) completed; PISA, the softmax
                // has read S(e-2)
                const int s = e % KS, b = e & 1;
                if (!mbar_wait(&k_full[s], (e / KS) & 1, abort_flag, lim) ||
                    (e >= 2 && !mbar_wait(PISA ? &s_free[b] : &pv_done[b], ((e >> 1) - 1) & 1, abort_flag, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (FP8) {
                    // e4m3 (or s8, exact s32 sums): 32 elements (32 bytes) per instruction
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        const uint64_t ad = sdesc(sbase + L::OFF_Q8 + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = sdesc(sK(s) + kk * 32, 16, 1024, kSwizzle128B);
                        if (I8)
                            umma_i8_ss(tmem + b * 64, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                        else
                            umma_f8_ss(tmem + b * 64, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bd = sdesc(sK(s) + (kk >> 2) * L::KBOX + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                        umma_f16_ss(tmem + b * 64, qdesc(kk), bd, ID_S, kk > 0 ? 1u : 0u);
                    }
                }
                umma_commit(&s_full[b]);
                umma_commit(&k_empty[s]);
            }
            if (!ok) fail();
            // drain: this thread's MMAs complete before TMEM is released
            umma_commit(drain_bar);
            mbar_wait(drain_bar, 0, abort_flag, drain_lim);
        }
    } else if (warp == 3) {
        // ======================================================== P.V / G / linear issuer
        if (lane == 0) {
            constexpr uint32_t ID_PV = FP8 ? idesc_e4m3(128, D) : idesc_f16(128, D, 0, 1);
            // G_g starts as H (preloaded by the softmax warps) and accumulates
            // -phi(K_j)^T V_j, so it ends as H - sum_{j in S_g} h_j
            constexpr uint32_t ID_G = idesc_f16(128, D, 1, 1, 1);
            bool ok = true;
            bool g_ready = !SLA;
            for (int e = 0; ok && e < n_total; ++e) {
                const int s = e % VS, b = e & 1, u = e >> 1;
                if (!mbar_wait(&v_full[s], (e / VS) & 1, abort_flag, lim) ||
                    !mbar_wait(&p_full[b], u & 1, abort_flag, lim)) { ok = false; break; }
                tc_fence_after();
                // O_b += P(e) V_e, P read from the first columns of S buffer b (PISA:
                // from P buffer b)
                const uint32_t o_col = tmem + COL_O + b * D;
                const uint32_t p_col = tmem + (PISA ? COL_P + b * 32 : b * 64);
                if (FP8) {
                    // B = V^T (e4m3, K-major: 64 tokens = 64 bytes per row, 64-byte swizzle)
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const uint64_t bd = sdesc(sV(s) + kk * 32, 16, 512, kSwizzle64B);
                        umma_f8_ts(o_col, tmem + b * 64 + kk * 8, bd, ID_PV, (u > 0 || kk > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = sdesc(sV(s) + kk * 2048, L::KBOX, 1024, kSwizzle128B);
                        umma_f16_ts(o_col, p_col + kk * 8, bd, ID_PV, (u > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&pv_done[b]);
                if (SLA) {
                    if (!g_ready) {
                        if (!mbar_wait(g_init, 0, abort_flag, lim)) { ok = false; break; }
                        tc_fence_after();
                        g_ready = true;
                    }
                    const int bits = (sched[e] >> 16) & 3;
                    for (int g = 0; g < 2; ++g) {
                        if (!((bits >> g) & 1)) continue;
                        const uint32_t lbo = D == 128 ? L::KBOX : 0;   // D = 64: M rows 64-127 repeat
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = sdesc(sPhi(s) + kk * 2048, lbo, 1024, kSwizzle128B);
                            const uint64_t bd = sdesc(sV16(s) + kk * 2048, L::KBOX, 1024, kSwizzle128B);
                            umma_f16_ss(tmem + COL_G0 + g * D, ad, bd, ID_G, 1u);
                        }
                    }
                }
                umma_commit(&v_empty[s]);
            }
            if (!ok) fail();
            umma_commit(final_bar);
            if ((SLA || a.first_order) && ok) {
                // SLA linear branch: D_lin_g = phi(Q) (H - G_g), hi + lo, into G_g's
                // columns (phi(Q) was written over the query tile in shared memory).
                // PISA first-order term: Q Hsum, hi + lo, into the same columns.
                if (mbar_wait(epi_ready, 0, abort_flag, lim)) {
                    tc_fence_after();
                    constexpr uint32_t ID_L = idesc_bf16(128, D, 0, 1);
                    for (int g = 0; g < (SLA ? n_groups : 1); ++g) {
                        for (int part = 0; part < 2; ++part) {
                            const uint32_t bb = sbase + L::OFF_K + (2 * g + part) * L::BBUF;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t bd = sdesc(bb + kk * 2048, L::BBOX, 1024, kSwizzle128B);
                                umma_f16_ss(tmem + COL_G0 + g * D, qdesc(kk), bd, ID_L,
                                            (part > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    }
                    umma_commit(lin_done);
                } else {
                    fail();
                }
            }
            umma_commit(drain2_bar);
            mbar_wait(drain2_bar, 0, abort_flag, drain_lim);
        }
    } else if (warp == 2) {
        // ======================================================== z sums (SLA)
        // Zu_g = Z - sum_{j in S_g} z_j, the linear-branch denominator vector.
        if (SLA) {
            const int t = lane;                          // 0..31, columns t + 32 c
            const float* zjh = a.zj + static_cast<long long>(bh) * a.Nk * D;
            const float* zs = a.zsum + static_cast<long long>(bh) * D;
            for (int g = 0; g < 2; ++g) {
                float acc[D / 32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) acc[c] = 0.f;
                if (g < n_groups) {
                    const int32_t* row = a.lut + (static_cast<long long>(bh) * a.Nq + qb0 + g) * a.topk;
#pragma unroll 4
                    for (int x = 0; x < a.topk; ++x) {
                        const int j = row[x];
                        if (j < 0 || j >= a.Nk) continue;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) acc[c] += __ldg(zjh + static_cast<long long>(j) * D + t + 32 * c);
                    }
                }
                // every block selected: the unselected set is empty and its sum is
                // exactly zero (so is the linear branch), not the rounding residue
                // of Z minus all z_j
                const bool none_left = a.topk >= a.Nk;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) zu[g * D + t + 32 * c] = none_left ? 0.f : zs[t + 32 * c] - acc[c];
            }
            __syncwarp();
            // the linear-branch denominators phi(q_r) . Zu_g(r) of the tile's 128 rows,
            // from the query tile in shared memory (read only, while the main loop runs)
            if (__all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, lim) ? 1 : 0)) {
                for (int rr = lane; rr < 128; rr += 32) {
                    const float* z = zu + min(rr / a.Bq, 1) * D;
                    float den = 0.f;
#pragma unroll 4
                    for (int x = 0; x < D / 8; ++x) {
                        const int c8 = 8 * x;
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            smem + L::OFF_Q + (c8 >> 6) * L::QBOX + sw128(rr, (c8 & 63) >> 3));
                        const uint32_t w4[4] = {relu_bf16x2_u(v.x), relu_bf16x2_u(v.y), relu_bf16x2_u(v.z),
                                                relu_bf16x2_u(v.w)};
#pragma unroll
                        for (int y = 0; y < 4; ++y)
                            den += bf16lo(w4[y]) * z[c8 + 2 * y] + bf16hi(w4[y]) * z[c8 + 2 * y + 1];
                    }
                    xd[rr] = den;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_ready);
        } else if (a.first_order && lane == 0) {
            mbar_arrive(epi_ready);
        }
    } else {
        // ======================================================== softmax + epilogue
        // Warpgroup h takes the entries e with e % 2 == h: S buffer h, O_h and its
        // own running maximum and row sum, so the two warpgroups work on two
        // entries at once; their partial results are merged in the epilogue.
        const int q4 = warp & 3;                         // TMEM lane quarter
        const int h = (warp - 4) >> 2;                   // warpgroup
        const int r = q4 * 32 + lane;                    // row within the tile
        const int g = r / a.Bq;
        const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        // warp-uniform bounded wait: if any lane gives up, the whole warp does
        auto wwait = [&](uint64_t* bar, uint32_t par) {
            return __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag, lim) ? 1 : 0) != 0;
        };
        const float c = a.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;          // this warpgroup's running max (log2 units) and sum
        float lc_run = 0.f;                            // PISA: the centroid pseudo-tiles' part of l_run
        bool ok = true;
        if (SLA) {
            // G_g := H (row r = c of the d x d matrix, this warpgroup's half of the
            // columns); H is stored transposed per head, H^T[e][c], so lane r's loads
            // are coalesced
            if (r < D) {
                const float* hcol = a.hsum + static_cast<long long>(bh) * D * D + r;
#pragma unroll 1
                for (int cc = h * (D / 2); cc < (h + 1) * (D / 2); cc += 32) {
                    uint32_t hv[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) hv[x] = __float_as_uint(__ldg(hcol + static_cast<long long>(cc + x) * D));
                    for (int gg = 0; gg < n_groups; ++gg) tmem_st32(tl + COL_G0 + gg * D + cc, hv);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(g_init);
        }
        // FP8: this row's Q block scale and the tile's P quantisation reference
        const float sq = FP8 ? a.sq[(static_cast<long long>(bh) * a.N + row0 + r) / 64] : 1.f;
        const float svmax = FP8 ? *svmax_s : 1.f;
        const uint32_t o_h = COL_O + h * D;
        // this row's combine weight, read now so its latency is off the epilogue
        const float al = (SLA && g < n_groups && row0 + r < a.N)
                             ? a.alpha[static_cast<long long>(bh) * a.N + row0 + r] : 0.f;
        uint32_t sv[64];
        for (int e = h; e < n_total; e += 2) {
            const int u = e >> 1;
            if (!wwait(&s_full[h], u & 1)) { ok = false; break; }
            tc_fence_after();
            // PISA: P(e) goes to P buffer h once P.V(e-2) has read P(e-2) (and O_h
            // may be rescaled only then); SLA: S(e) was issued after P.V(e-2)
            // completed, so both hold already
            bool pv_ok = !PISA || e < 2;
            auto wait_pv = [&]() {
                if (!pv_ok) {
                    if (!wwait(&pv_done[h], (u - 1) & 1)) return false;
                    tc_fence_after();
                    pv_ok = true;
                }
                return true;
            };
            const uint32_t p_dst = tl + (PISA ? COL_P + h * 32 : h * 64);
            if (e < n_exact && !__any_sync(0xffffffffu, (sched[e] >> (16 + g)) & 1)) {
                // no row of this warp selected the block (the other group did): its P
                // is zero, with nothing to load, exponentiate or rescale
                if (PISA) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free[h]);
                }
                if (!wait_pv()) { ok = false; break; }
                uint32_t z[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) z[x] = 0u;
                tmem_st16(p_dst, z);
                if (!FP8) tmem_st16(p_dst + 16, z);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[h]);
                continue;
            }
            tmem_ld32(tl + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(tl + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_ld_wait();
            if (PISA) {
                // S buffer h is free for S(e+2)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[h]);
            }
            if (I8) {
                // s32 scores, |S| <= 128 * 127^2 < 2^22: exact in fp32
#pragma unroll
                for (int j = 0; j < 64; ++j) sv[j] = __float_as_uint(small_int_to_float(sv[j]));
            }

            // row maximum over the 64 logits (x = s * c, + log2 Bk for centroids;
            // masked ones are -inf)
            bool act = true;
            float mx = -INFINITY;
            // logit scale of this block (FP8: times the Q and K block scales)
            const float ce = FP8 ? c * sq * ent_sk[e] : c;
            if (e < n_exact) {
                act = (sched[e] >> (16 + g)) & 1;
                if (act) mx = max64_bits(sv) * ce;
            } else {
                const int c0 = (e - n_exact) * 64;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int cw = c0 + 16 * w;
                    const uint32_t mw = (cw >> 4) < nwords ? mark[cw >> 4] : 0u;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int j = 16 * w + jj;
                        const bool masked = (c0 + j) >= a.Nk || ((mw >> (2 * jj + g)) & 1u);
                        const float x = masked ? -INFINITY : fmaf(__uint_as_float(sv[j]), c, a.log2_bk);
                        sv[j] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
                }
            }
            // lazy rescale (P <= 2^8).  FP8: the reference is the power of two at or
            // above the running maximum, so P <= 1 and every rescale is an exact
            // power of two (it commutes with the e4m3 rounding of earlier P)
            const bool need = mx > m_run + (FP8 ? 0.f : kRescaleLog2);
            const float m_new = need ? (FP8 ? ceilf(mx) : mx) : m_run;
            const bool rescale_o = need && m_run != -INFINITY;
            if (__any_sync(0xffffffffu, rescale_o)) {
                // O_h holds P.V of this warpgroup's entries up to e-2, all complete
                if (!wait_pv()) { ok = false; break; }
                const float f = rescale_o ? (FP8 ? exp2_int(m_run - m_new) : fast_exp2(m_run - m_new)) : 1.f;
#pragma unroll 1
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tl + o_h + cc, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * f);
                    tmem_st32(tl + o_h + cc, ov);
                }
                tmem_st_wait();
                l_run *= f;
                lc_run *= f;
            }
            m_run = m_new;
            // P = 2^(x - m) over the 64 keys, written over the first columns of S
            // buffer h: packed fp16 pairs, or (FP8) e4m3 quads of
            // P * 448 * s_v,j / s_v,max with the row sum from fp32 P
            const bool live = act && m_run != -INFINITY;
            float ls;
            if (FP8) {
                uint32_t p8[16];
                const float qf = 448.f * ent_sv[e] / svmax;
                ls = softmax_half_e4m3<0>(sv, ce, m_run, live, qf, *reinterpret_cast<uint32_t(*)[8]>(&p8[0]));
                ls += softmax_half_e4m3<32>(sv, ce, m_run, live, qf, *reinterpret_cast<uint32_t(*)[8]>(&p8[8]));
                tmem_st16(tl + h * 64, p8);
            } else {
                uint32_t pwa[16], pwb[16];
                const bool exact = e < n_exact;
                ls = exact ? softmax_half<0, true, PISA>(sv, c, m_run, live, pwa)
                           : softmax_half<0, false, PISA>(sv, c, m_run, live, pwa);
                ls += exact ? softmax_half<32, true, PISA>(sv, c, m_run, live, pwb)
                            : softmax_half<32, false, PISA>(sv, c, m_run, live, pwb);
                if (!wait_pv()) { ok = false; break; }
                tmem_st16(p_dst, pwa);
                tmem_st16(p_dst + 16, pwb);
            }
            tmem_st_wait();
            l_run += ls;
            if (PISA && e >= n_exact) lc_run += ls;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[h]);
        }
        if (!ok) fail();

        // ------------------------------------------------ epilogue
        // merge the two warpgroups' partial softmaxes (exchanged once through shared memory)
        xm[h * 128 + r] = m_run;
        xl[h * 128 + r] = l_run;
        if (PISA) xd[h * 128 + r] = lc_run;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xl_bar[q4]);
        const bool xok = wwait(&xl_bar[q4], 0);
        if (ok && !xok) fail();
        float f0 = 0.f, f1 = 0.f, l_tot = 0.f;
        if (xok) {
            const float m0 = xm[r], m1 = xm[128 + r];
            const float mm = fmaxf(m0, m1);
            if (m0 != -INFINITY) f0 = FP8 ? exp2_int(m0 - mm) : fast_exp2(m0 - mm);
            if (m1 != -INFINITY) f1 = FP8 ? exp2_int(m1 - mm) : fast_exp2(m1 - mm);
            l_tot = f0 * xl[r] + f1 * xl[128 + r];
        }
        // PISA: the centroid part of the row sum (= Bk * sum over U of e^{tau q.kbar_j - m})
        const float lc_tot = (PISA && xok) ? f0 * xd[r] + f1 * xd[128 + r] : 0.f;
        const bool fin = ok && xok && wwait(final_bar, 0);
        if (ok && xok && !fin) fail();
        tc_fence_after();
        // FP8: O accumulated P * 448 * s_v,j / s_v,max times V / s_v,j
        const float inv_l = l_tot > 0.f ? (FP8 ? svmax / 448.f : 1.f) / l_tot : 0.f;
        const bool have0 = n_total > 0 && f0 != 0.f, have1 = n_total > 1 && f1 != 0.f;
        constexpr int HC = D / 2;                        // output columns of this warpgroup
        // sum of the two partial P.V accumulators for 32 columns, scaled by 1/l
        auto o_sum = [&](int cc, float (&res)[32]) {
            uint32_t o0[32], o1[32];
            if (have0) tmem_ld32(tl + COL_O + cc, o0);
            if (have1) tmem_ld32(tl + COL_O + D + cc, o1);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x)
                res[x] = ((have0 ? f0 * __uint_as_float(o0[x]) : 0.f) +
                          (have1 ? f1 * __uint_as_float(o1[x]) : 0.f)) * inv_l;
        };
        if (PISA && a.first_order) {
            // global first-order term: + tau/(Nk Bk) * lc * (q . Hsum), with q . Hsum
            // on the tensor core (Hsum as bf16 hi + lo, MN-major boxes like the SLA
            // linear-branch operand; row r = c of Hsum, this warpgroup's columns)
            if (fin && r < D) {
                const float* hcol = a.hbar + static_cast<long long>(bh) * D * D + r;
                unsigned char* bhi = smem + L::OFF_K;
                unsigned char* blo = bhi + L::BBUF;
#pragma unroll 1
                for (int cc = h * HC; cc < (h + 1) * HC; cc += 8) {
                    uint32_t hi4[4], lo4[4];
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        const float v0 = __ldg(hcol + static_cast<long long>(cc + 2 * y) * D);
                        const float v1 = __ldg(hcol + static_cast<long long>(cc + 2 * y + 1) * D);
                        hi4[y] = pack_bf16(v0, v1);
                        lo4[y] = pack_bf16(v0 - bf16lo(hi4[y]), v1 - bf16hi(hi4[y]));
                    }
                    const uint32_t off = (cc >> 6) * L::BBOX + sw128(r, (cc & 63) >> 3);
                    *reinterpret_cast<uint4*>(bhi + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                    *reinterpret_cast<uint4*>(blo + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                }
            }
            fence_proxy_async_smem();                      // Hsum -> the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_ready);
            float res[HC];
            if (fin) {
#pragma unroll
                for (int x = 0; x < HC / 32; ++x) o_sum(h * HC + 32 * x, *reinterpret_cast<float(*)[32]>(&res[32 * x]));
            }
            const bool fo = fin && wwait(epi_ready, 0) && wwait(lin_done, 0);
            if (fin && !fo) fail();
            tc_fence_after();
            if (fo) {
                const float w1 = a.fo_scale * lc_tot * inv_l;
#pragma unroll
                for (int x = 0; x < HC / 32; ++x) {
                    const int cc = h * HC + 32 * x;
                    uint32_t fv[32];
                    tmem_ld32(tl + COL_G0 + cc, fv);
                    tmem_ld_wait();
                    float out32[32];
#pragma unroll
                    for (int y = 0; y < 32; ++y) out32[y] = res[32 * x + y] + w1 * __uint_as_float(fv[y]);
                    stage_row32(smem + L::OUT_OFF, a.out_f32, r, cc, out32);
                }
            }
        } else if (PISA) {
            if (fin) {
#pragma unroll 1
                for (int cc = h * HC; cc < (h + 1) * HC; cc += 32) {
                    float res[32];
                    o_sum(cc, res);
                    stage_row32(smem + L::OUT_OFF, a.out_f32, r, cc, res);
                }
            }
        } else {
            // (1) B_g = H - G_g (row r of the d x d matrices, this warpgroup's columns),
            //     bf16 hi + lo, MN-major 128-byte-swizzled boxes of 64 columns
            if (fin && r < D) {
                for (int gg = 0; gg < n_groups; ++gg) {
                    unsigned char* bhi = smem + L::OFF_K + (2 * gg) * L::BBUF;
                    unsigned char* blo = bhi + L::BBUF;
#pragma unroll 1
                    for (int cc = h * HC; cc < (h + 1) * HC; cc += 32) {
                        uint32_t gv[32];
                        tmem_ld32(tl + COL_G0 + gg * D + cc, gv);
                        tmem_ld_wait();
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint32_t hi4[4], lo4[4];
#pragma unroll
                            for (int y = 0; y < 4; ++y) {
                                const float v0 = __uint_as_float(gv[8 * x + 2 * y]);
                                const float v1 = __uint_as_float(gv[8 * x + 2 * y + 1]);
                                hi4[y] = pack_bf16(v0, v1);
                                lo4[y] = pack_bf16(v0 - bf16lo(hi4[y]), v1 - bf16hi(hi4[y]));
                            }
                            const int c8 = cc + 8 * x;
                            const uint32_t off = (c8 >> 6) * L::BBOX + sw128(r, (c8 & 63) >> 3);
                            *reinterpret_cast<uint4*>(bhi + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                            *reinterpret_cast<uint4*>(blo + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                        }
                    }
                }
            }
            // (2) phi(Q) over the query tile in shared memory (the A operand of the
            //     linear-branch product), this warpgroup's half of row r
            if (fin) {
#pragma unroll
                for (int x = 0; x < HC / 8; ++x) {
                    const int c8 = h * HC + 8 * x;               // first column of this chunk
                    unsigned char* p = smem + L::OFF_Q + (c8 >> 6) * L::QBOX + sw128(r, (c8 & 63) >> 3);
                    uint4 v = *reinterpret_cast<const uint4*>(p);
                    v.x = relu_bf16x2_u(v.x); v.y = relu_bf16x2_u(v.y);
                    v.z = relu_bf16x2_u(v.z); v.w = relu_bf16x2_u(v.w);
                    *reinterpret_cast<uint4*>(p) = v;
                }
            }
            fence_proxy_async_smem();                      // phi(Q), B_g -> the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_ready);
            // (3) the sparse part of the combine while the linear-branch product runs
            float res[HC];
            if (fin) {
#pragma unroll
                for (int x = 0; x < HC / 32; ++x) o_sum(h * HC + 32 * x, *reinterpret_cast<float(*)[32]>(&res[32 * x]));
            }
            const bool lin = fin && wwait(epi_ready, 0) && wwait(lin_done, 0);
            if (fin && !lin) fail();
            tc_fence_after();
            if (lin) {
                // denominator phi(q) . Zu_g, from warp 2 (written before its epi_ready arrival)
                const float den = xd[r];
                const float inv_den = den > 0.f ? 1.f / den : 0.f;
                const uint32_t col_lin = COL_G0 + (g < n_groups ? g : 0) * D;
#pragma unroll
                for (int x = 0; x < HC / 32; ++x) {
                    const int cc = h * HC + 32 * x;
                    uint32_t lv[32];
                    tmem_ld32(tl + col_lin + cc, lv);
                    tmem_ld_wait();
                    float out32[32];
#pragma unroll
                    for (int y = 0; y < 32; ++y)
                        out32[y] = al * res[32 * x + y] + (1.f - al) * (__uint_as_float(lv[y]) * inv_den);
                    stage_row32(smem + L::OUT_OFF, a.out_f32, r, cc, out32);
                }
            }
        }
    }

    // ------------------------------------------------------------ output store
    if (warp >= 4) {
        // all 8 softmax warps have staged their rows; one thread stores the valid
        // 64-row groups of the tile with the tensor engine
        fence_proxy_async_smem();
        named_bar(1, 256);
        if (warp == 4 && lane == 0 && !*abort_flag) {
            const CUtensorMap* tmOut = &tm.out;
            const int nb = a.out_f32 ? D / 32 : D / 64;
            const int bc = a.out_f32 ? 32 : 64;
            for (int k = 0; k < 2; ++k) {
                if (64 * k >= n_groups * a.Bq || row0 + 64 * k + 64 > a.N) continue;
                for (int b = 0; b < nb; ++b)
                    tma_store_2d(tmOut, smem + L::OUT_OFF + b * 16384 + k * 64 * 128, b * bc,
                                 bh * a.N + row0 + 64 * k);
            }
            tma_store_commit();
            tma_store_wait_read();
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, NCOLS);
}

}  // namespace sla

// attn.cuh -- block-sparse attention on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA owns 128 query rows = 128/Bq query blocks ("groups") of one head.
// It walks the union of its groups' selected KV blocks in ascending order
// (each entry tagged with the groups that selected it) and, in PISA mode,
// then the head's centroid pseudo-tiles.  Per entry:
//   S  = Q K_j^T                        tcgen05.mma M=128 N=64  -> TMEM (2 buffers)
//   P  = exp2(S*tau*log2e - m)          softmax warps, one row per thread,
//                                       online max with lazy rescale of O;
//                                       P is stored as fp16
//   O += P V_j                          tcgen05.mma M=128 N=d   -> TMEM (fp16 V copy)
//   G_g += phi(K_j)^T V_j  (SLA only)   tcgen05.mma M=128 N=d   -> TMEM, per group;
//                                       phi(K_j) written in place as fp16
// Linear branch (SALAD ReLU kernel; SLA2 combine): after the loop,
//   O_l = phi(Q) (H - G_g) / (phi(q) . (Z - sum_{j in S_g} z_j))
// with (H - G_g) split into bf16 hi + lo and multiplied on the tensor core,
// then out = alpha O_s + (1 - alpha) O_l.
// PISA (zero-order "exact-or-approximate"): a centroid pseudo-tile holds 64
// block centroids kbar_j and value means vbar_j; its logits get + log2(Bk)
// (the block multiplicity) and the groups' own selected blocks are masked, so
// e^{q.kbar_j - m} (sum_n v_n) enters N_t and Bk e^{q.kbar_j - m} enters D_t in
// the same online softmax; out = N_t / D_t.
//
// Warp roles (256 threads): w0 TMA producer, w1 MMA issuer (+ TMEM owner),
// w2-3 phi(K) transform + z sums (SLA), w4-7 softmax and epilogue.
// Every wait is bounded; a wait that runs out sets the device status word and
// the CTA unwinds after draining its own TMA loads and MMAs.
#pragma once
#include "common.cuh"

namespace sla {

constexpr int kStages = 3;
constexpr float kRescaleLog2 = 8.0f;    // lazy O rescale threshold (log2 units)

struct AttnArgs {
    int N, Nq, Nk, Bq, topk, tiles_per_head;
    float scale_log2;              // tau * log2(e)
    float log2_bk;                 // log2(Bk), PISA pseudo-tile bias
    const int32_t* lut;            // [BH][Nq][topk]
    const float* alpha;            // [BH][N]        (SLA)
    const float* hsum;             // [BH][D][D]     (SLA), transposed: H^T[e][c]
    const float* zsum;             // [BH][D]        (SLA)
    const float* zj;               // [BH][Nk][D]    (SLA)
    void* out;                     // [BH][N][D] bf16 or fp32
    int out_f32;
    unsigned long long wait_ns;
};

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 32 consecutive output values of one row: bf16 (four 16-byte stores) or fp32.
__device__ __forceinline__ void store_row32(void* out, int f32, long long off, const float (&v)[32]) {
    if (f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
#pragma unroll
        for (int x = 0; x < 8; ++x) dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + off);
#pragma unroll
        for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(pack_bf16(v[8 * x], v[8 * x + 1]), pack_bf16(v[8 * x + 2], v[8 * x + 3]),
                                pack_bf16(v[8 * x + 4], v[8 * x + 5]), pack_bf16(v[8 * x + 6], v[8 * x + 7]));
    }
}

template <int D>
struct AttnLayout {
    static constexpr int QB = 128 * D * 2;           // Q tile bytes
    static constexpr int KT = 64 * D * 2;            // K (or V) tile bytes
    static constexpr int KBOX = 64 * 128;            // one 64-row x 128-byte box
    static constexpr int QBOX = 128 * 128;           // one 128-row x 128-byte box
    static constexpr int PT = 128 * 128;             // P tile: 128 rows x 64 bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGE = OFF_Q + QB;
    static constexpr int OFF_P = OFF_STAGE + kStages * 2 * KT;
    static constexpr int OFF_MISC = OFF_P + 2 * PT;
    static constexpr int BBUF = D * D * 2;           // one (H - G) hi or lo buffer
    static constexpr int BBOX = D * 128;             // one 64-column box of it
};

template <int D, bool PISA>
__global__ void __launch_bounds__(256, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, const AttnArgs a) {
    using L = AttnLayout<D>;
    constexpr bool SLA = !PISA;
    constexpr int NBOX = D / 64;
    constexpr uint32_t NCOLS = (PISA ? (128 + D) : (128 + 3 * D)) <= 256 ? 256 : 512;
    constexpr uint32_t COL_O = 128;
    constexpr uint32_t COL_G0 = 128 + D;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);

    // misc region
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_MISC);
    uint64_t* q_full = bars + 0;
    uint64_t* kv_full = bars + 1;                 // [kStages]
    uint64_t* kv_empty = kv_full + kStages;       // [kStages]
    uint64_t* kdone = kv_empty + kStages;         // [kStages]  S_e done -> K_j reusable
    uint64_t* k_relu = kdone + kStages;           // [kStages]  phi(K_j) written
    uint64_t* s_full = k_relu + kStages;          // [2]
    uint64_t* s_empty = s_full + 2;               // [2]
    uint64_t* p_full = s_empty + 2;               // [2]
    uint64_t* p_empty = p_full + 2;               // [2]
    uint64_t* final_bar = p_empty + 2;
    uint64_t* epi_ready = final_bar + 1;
    uint64_t* lin_done = epi_ready + 1;
    uint64_t* drain_bar = lin_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
    int* n_exact_s = reinterpret_cast<int*>(tmem_slot + 1);
    volatile int* abort_flag = n_exact_s + 1;
    int* g_any = n_exact_s + 2;                   // [2] group selected >= 1 block
    float* zu = reinterpret_cast<float*>(smem + L::OFF_MISC + 256);       // [2][D]
    uint32_t* mark = reinterpret_cast<uint32_t*>(zu + 2 * D);            // [ceil(Nk/16)]
    const int nwords = (a.Nk + 15) >> 4;
    int32_t* sched = reinterpret_cast<int32_t*>(mark + ((nwords + 3) & ~3));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / a.tiles_per_head;
    const int tile = blockIdx.x % a.tiles_per_head;
    const int GR = 128 / a.Bq;
    const int qb0 = tile * GR;
    const int n_groups = min(GR, a.Nq - qb0);

    // ------------------------------------------------------------ set-up
    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&kdone[s], 1);
            mbar_init(&k_relu[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 4);
            mbar_init(&p_full[b], 4);
            mbar_init(&p_empty[b], 1);
        }
        mbar_init(final_bar, 1);
        mbar_init(epi_ready, 6);
        mbar_init(lin_done, 1);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, NCOLS);
        tmem_relinquish();
    }
    for (int w = tid; w < nwords; w += 256) mark[w] = 0u;
    __syncthreads();
    for (int x = tid; x < n_groups * a.topk; x += 256) {
        const int g = x / a.topk;
        const int j = a.lut[(static_cast<long long>(bh) * a.Nq + qb0 + g) * a.topk + x % a.topk];
        if (j < 0 || j >= a.Nk) { report(kStatusBadData); continue; }
        const uint32_t bit = (1u << g) << (2 * (j & 15));
        const uint32_t old = atomicOr(&mark[j >> 4], bit);
        if (old & bit) report(kStatusBadData);
    }
    __syncthreads();
    if (warp == 0) {
        int cnt = 0;
        uint32_t any = 0u;
        const uint32_t lt = (1u << lane) - 1u;
        for (int j0 = 0; j0 < a.Nk; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t bits = j < a.Nk ? (mark[j >> 4] >> (2 * (j & 15))) & 3u : 0u;
            const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
            if (bits) sched[cnt + __popc(bal & lt)] = j | static_cast<int>(bits << 16);
            cnt += __popc(bal);
            any |= bits;
        }
        any = __reduce_or_sync(0xffffffffu, any);
        if (lane == 0) {
            *n_exact_s = cnt;
            g_any[0] = any & 1u;
            g_any[1] = (any >> 1) & 1u;
        }
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

    const uint32_t sQ = sbase + L::OFF_Q;
    auto sK = [&](int s) { return sbase + L::OFF_STAGE + s * 2 * L::KT; };
    auto sV = [&](int s) { return sbase + L::OFF_STAGE + s * 2 * L::KT + L::KT; };
    auto sP = [&](int b) { return sbase + L::OFF_P + b * L::PT; };

    auto fail = [&]() {
        *abort_flag = 1;
        report(kStatusTimeout);
    };

    if (warp == 0) {
        // ======================================================== TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const int qrow = bh * a.N + tile * 128;
            mbar_arrive_expect_tx(q_full, L::QB);
            for (int b = 0; b < NBOX; ++b)
                tma_load_2d(smem + L::OFF_Q + b * L::QBOX, &tmQ, q_full, b * 64, qrow);
            int issued = 0;
            for (int e = 0; e < n_total; ++e) {
                const int s = e % kStages, r = e / kStages;
                if (!mbar_wait(&kv_empty[s], (r & 1) ^ 1, abort_flag, lim)) { fail(); break; }
                mbar_arrive_expect_tx(&kv_full[s], 2 * L::KT);
                unsigned char* kd = smem + L::OFF_STAGE + s * 2 * L::KT;
                unsigned char* vd = kd + L::KT;
                if (e < n_exact) {
                    const int row = bh * a.N + (sched[e] & 0xFFFF) * 64;
                    for (int b = 0; b < NBOX; ++b) {
                        tma_load_2d(kd + b * L::KBOX, &tmK, &kv_full[s], b * 64, row);
                        tma_load_2d(vd + b * L::KBOX, &tmV, &kv_full[s], b * 64, row);
                    }
                } else {
                    const int row = bh * a.Nk + (e - n_exact) * 64;
                    for (int b = 0; b < NBOX; ++b) {
                        tma_load_2d(kd + b * L::KBOX, &tmKc, &kv_full[s], b * 64, row);
                        tma_load_2d(vd + b * L::KBOX, &tmVc, &kv_full[s], b * 64, row);
                    }
                }
                issued = e + 1;
            }
            // drain: every load this thread issued has landed before the CTA exits
            mbar_wait(q_full, 0, abort_flag, drain_lim);
            for (int e = max(0, issued - kStages); e < issued; ++e)
                mbar_wait(&kv_full[e % kStages], (e / kStages) & 1, abort_flag, drain_lim);
        }
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t ID_PV = idesc_f16(128, D, 0, 1);
            constexpr uint32_t ID_G = idesc_f16(128, D, 1, 1);
            bool ok = mbar_wait(q_full, 0, abort_flag, lim);
            tc_fence_after();
            int g_started[2] = {0, 0};                // accumulate flag of G_g
            auto issue_pv = [&](int e) -> bool {
                const int s = e % kStages, b = e & 1, u = e >> 1;
                if (!mbar_wait(&p_full[b], u & 1, abort_flag, lim)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = sdesc(sP(b) + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = sdesc(sV(s) + kk * 2048, L::KBOX, 1024, kSwizzle128B);
                    umma_f16_ss(tmem + COL_O, ad, bd, ID_PV, (e > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&p_empty[b]);
                if (SLA) {
                    if (!mbar_wait(&k_relu[s], (e / kStages) & 1, abort_flag, lim)) return false;
                    tc_fence_after();
                    const int bits = (sched[e] >> 16) & 3;
                    for (int g = 0; g < 2; ++g) {
                        if (!((bits >> g) & 1)) continue;
                        const uint32_t lbo = D == 128 ? L::KBOX : 0;   // D = 64: M rows 64-127 repeat
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = sdesc(sK(s) + kk * 2048, lbo, 1024, kSwizzle128B);
                            const uint64_t bd = sdesc(sV(s) + kk * 2048, L::KBOX, 1024, kSwizzle128B);
                            umma_f16_ss(tmem + COL_G0 + g * D, ad, bd, ID_G,
                                        (g_started[g] || kk > 0) ? 1u : 0u);
                        }
                        g_started[g] = 1;
                    }
                }
                umma_commit(&kv_empty[s]);
                return true;
            };
            for (int e = 0; ok && e < n_total; ++e) {
                const int s = e % kStages, r = e / kStages, b = e & 1, u = e >> 1;
                if (!mbar_wait(&kv_full[s], r & 1, abort_flag, lim) ||
                    !mbar_wait(&s_empty[b], (u & 1) ^ 1, abort_flag, lim)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc(sQ + (kk >> 2) * L::QBOX + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = sdesc(sK(s) + (kk >> 2) * L::KBOX + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                    umma_f16_ss(tmem + b * 64, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[b]);
                if (SLA) umma_commit(&kdone[s]);
                if (e > 0 && !issue_pv(e - 1)) { ok = false; break; }
            }
            if (ok && n_total > 0 && !issue_pv(n_total - 1)) ok = false;
            if (!ok) fail();
            umma_commit(final_bar);
            if (SLA && ok) {
                // linear branch: D_lin_g = phi(Q) (H - G_g), hi + lo, into G_g's columns
                if (mbar_wait(epi_ready, 0, abort_flag, lim)) {
                    tc_fence_after();
                    constexpr uint32_t ID_L = idesc_bf16(128, D, 0, 1);
                    for (int g = 0; g < n_groups; ++g) {
                        for (int part = 0; part < 2; ++part) {
                            const uint32_t bb = sbase + L::OFF_STAGE + (2 * g + part) * L::BBUF;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t ad = sdesc(sQ + (kk >> 2) * L::QBOX + (kk & 3) * 32, 16, 1024, kSwizzle128B);
                                const uint64_t bd = sdesc(bb + kk * 2048, L::BBOX, 1024, kSwizzle128B);
                                umma_f16_ss(tmem + COL_G0 + g * D, ad, bd, ID_L,
                                            (part > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    }
                    umma_commit(lin_done);
                } else {
                    fail();
                }
            }
            // drain: all MMAs of this CTA complete before TMEM is released
            umma_commit(drain_bar);
            mbar_wait(drain_bar, 0, abort_flag, drain_lim);
        }
    } else if (warp < 4) {
        // ======================================================== phi(K) transform (SLA)
        if (SLA) {
            const int t = tid - 64;                      // 0..63
            float zacc[2][D / 64];
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
                for (int c = 0; c < D / 64; ++c) zacc[g][c] = 0.f;
            const float* zjh = a.zj + static_cast<long long>(bh) * a.Nk * D;
            bool ok = true;
            for (int e = 0; e < n_exact; ++e) {
                const int s = e % kStages, r = e / kStages;
                if (!mbar_wait(&kv_full[s], r & 1, abort_flag, lim) ||
                    !mbar_wait(&kdone[s], r & 1, abort_flag, lim)) { ok = false; break; }
                uint4* kp = reinterpret_cast<uint4*>(smem + L::OFF_STAGE + s * 2 * L::KT);
                constexpr int PER = L::KT / 16 / 64;     // uint4 per thread
#pragma unroll
                for (int x = 0; x < PER; ++x) {
                    // phi(k) = max(k, 0), bf16 -> fp16 (exact inside the fp16 range);
                    // consecutive threads touch consecutive 16-byte chunks (no bank conflicts)
                    uint4 v = kp[x * 64 + t];
                    v.x = pack_half2(fmaxf(bf16lo(v.x), 0.f), fmaxf(bf16hi(v.x), 0.f));
                    v.y = pack_half2(fmaxf(bf16lo(v.y), 0.f), fmaxf(bf16hi(v.y), 0.f));
                    v.z = pack_half2(fmaxf(bf16lo(v.z), 0.f), fmaxf(bf16hi(v.z), 0.f));
                    v.w = pack_half2(fmaxf(bf16lo(v.w), 0.f), fmaxf(bf16hi(v.w), 0.f));
                    kp[x * 64 + t] = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&k_relu[s]);
                const int ent = sched[e];
                const int j = ent & 0xFFFF;
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    if (!((ent >> (16 + g)) & 1)) continue;
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) zacc[g][c] += zjh[static_cast<long long>(j) * D + t + 64 * c];
                }
            }
            if (!ok) fail();
            const float* zs = a.zsum + static_cast<long long>(bh) * D;
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
                for (int c = 0; c < D / 64; ++c) zu[g * D + t + 64 * c] = zs[t + 64 * c] - zacc[g][c];
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_ready);
        }
    } else {
        // ======================================================== softmax + epilogue
        const int q4 = warp - 4;
        const int r = q4 * 32 + lane;                    // row within the tile
        const int g = r / a.Bq;
        const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        // warp-uniform bounded wait: if any lane gives up, the whole warp does
        auto wwait = [&](uint64_t* bar, uint32_t par) {
            return __all_sync(0xffffffffu, mbar_wait(bar, par, abort_flag, lim) ? 1 : 0) != 0;
        };
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        uint32_t sv[64];
        for (int e = 0; e < n_total; ++e) {
            const int b = e & 1, u = e >> 1;
            if (!wwait(&s_full[b], u & 1)) { ok = false; break; }
            tc_fence_after();
            tmem_ld32(tl + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(tl + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[b]);

            float mx = -INFINITY;
            if (e < n_exact) {
                const bool act = (sched[e] >> (16 + g)) & 1;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const float x = act ? __uint_as_float(sv[j]) * a.scale_log2 : -INFINITY;
                    sv[j] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
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
                        const float x = masked ? -INFINITY
                                               : fmaf(__uint_as_float(sv[j]), a.scale_log2, a.log2_bk);
                        sv[j] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
                }
            }
            // P buffer b is free once PV_{e-2} completed
            if (!wwait(&p_empty[b], (u & 1) ^ 1)) { ok = false; break; }
            const bool need = mx > m_run + kRescaleLog2;
            const float m_new = need ? mx : m_run;
            const bool rescale_o = need && m_run != -INFINITY;
            if (__any_sync(0xffffffffu, rescale_o)) {
                // O holds PV_{0..e-1}: wait for PV_{e-1} (its P buffer's release)
                if (e > 0 && !wwait(&p_empty[b ^ 1], ((e - 1) >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const float f = rescale_o ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ov[32];
                    tmem_ld32(tl + COL_O + c, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * f);
                    tmem_st32(tl + COL_O + c, ov);
                }
                tmem_st_wait();
                l_run *= f;
            }
            m_run = m_new;
            // P = exp2(x - m), fp16, into P buffer b (row r, 128-byte swizzle)
            unsigned char* prow = smem + L::OFF_P + b * L::PT;
            float ls = 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t w4[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int j = ch * 8 + 2 * x;
                    const float p0 = m_run == -INFINITY ? 0.f : fast_exp2(__uint_as_float(sv[j]) - m_run);
                    const float p1 = m_run == -INFINITY ? 0.f : fast_exp2(__uint_as_float(sv[j + 1]) - m_run);
                    w4[x] = pack_half2(p0, p1);
                    ls += half_lo(w4[x]) + half_hi(w4[x]);
                }
                *reinterpret_cast<uint4*>(prow + sw128(r, ch)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            l_run += ls;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
        }
        if (!ok) fail();

        // ------------------------------------------------ epilogue
        const bool fin = ok && wwait(final_bar, 0);
        tc_fence_after();
        const long long grow = static_cast<long long>(bh) * a.N + static_cast<long long>(tile) * 128 + r;
        const bool row_ok = tile * 128 + r < a.N;
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        const bool have_o = n_total > 0;
        if (PISA) {
            if (fin) {
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ov[32];
                    if (have_o) {
                        tmem_ld32(tl + COL_O + c, ov);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int x = 0; x < 32; ++x) ov[x] = 0u;
                    }
                    if (row_ok) {
                        float res[32];
#pragma unroll
                        for (int x = 0; x < 32; ++x) res[x] = __uint_as_float(ov[x]) * inv_l;
                        store_row32(a.out, a.out_f32, grow * D + c, res);
                    }
                }
            }
        } else {
            // (1) B_g = H - G_g (row c = r of the d x d matrices), bf16 hi + lo,
            //     MN-major 128-byte-swizzled boxes of 64 columns
            if (fin && r < D) {
                // H is stored transposed per head, H^T[e][c]: lane r reads column r, coalesced
                const float* hcol = a.hsum + static_cast<long long>(bh) * D * D + r;
                for (int gg = 0; gg < n_groups; ++gg) {
                    unsigned char* bhi = smem + L::OFF_STAGE + (2 * gg) * L::BBUF;
                    unsigned char* blo = bhi + L::BBUF;
                    const bool gs = g_any[gg] != 0;
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t gv[32];
                        if (gs) {
                            tmem_ld32(tl + COL_G0 + gg * D + c, gv);
                            tmem_ld_wait();
                        }
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint32_t hi4[4], lo4[4];
#pragma unroll
                            for (int y = 0; y < 4; ++y) {
                                const int cc = c + 8 * x + 2 * y;
                                const float v0 = hcol[cc * D] - (gs ? __uint_as_float(gv[8 * x + 2 * y]) : 0.f);
                                const float v1 = hcol[(cc + 1) * D] - (gs ? __uint_as_float(gv[8 * x + 2 * y + 1]) : 0.f);
                                hi4[y] = pack_bf16(v0, v1);
                                lo4[y] = pack_bf16(v0 - bf16lo(hi4[y]), v1 - bf16hi(hi4[y]));
                            }
                            const int cc = c + 8 * x;
                            const uint32_t off = (cc >> 6) * L::BBOX + sw128(r, (cc & 63) >> 3);
                            *reinterpret_cast<uint4*>(bhi + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                            *reinterpret_cast<uint4*>(blo + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                        }
                    }
                }
            }
            // (2) phi(Q) in place (row r of each 64-column box)
            {
#pragma unroll
                for (int bx = 0; bx < NBOX; ++bx) {
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint4* p = reinterpret_cast<uint4*>(smem + L::OFF_Q + bx * L::QBOX + sw128(r, ch));
                        uint4 v = *p;
                        v.x = relu_bf16x2_u(v.x); v.y = relu_bf16x2_u(v.y);
                        v.z = relu_bf16x2_u(v.z); v.w = relu_bf16x2_u(v.w);
                        *p = v;
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_ready);
            const bool lin = fin && wwait(epi_ready, 0) &&
                             wwait(lin_done, 0);
            if (fin && !lin) fail();
            tc_fence_after();
            if (lin) {
                // denominator phi(q) . Zu_g
                float den = 0.f;
#pragma unroll
                for (int bx = 0; bx < NBOX; ++bx)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 v = *reinterpret_cast<const uint4*>(smem + L::OFF_Q + bx * L::QBOX + sw128(r, ch));
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                        const float* z = zu + g * D + bx * 64 + ch * 8;
#pragma unroll
                        for (int y = 0; y < 4; ++y) den += bf16lo(w[y]) * z[2 * y] + bf16hi(w[y]) * z[2 * y + 1];
                    }
                const float inv_den = den > 0.f ? 1.f / den : 0.f;
                const float al = row_ok ? a.alpha[grow] : 0.f;
                const uint32_t col_lin = COL_G0 + (g < n_groups ? g : 0) * D;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ov[32], lv[32];
                    tmem_ld32(tl + col_lin + c, lv);
                    if (have_o) {
                        tmem_ld32(tl + COL_O + c, ov);
                    }
                    tmem_ld_wait();
                    if (!have_o) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) ov[x] = 0u;
                    }
                    if (row_ok) {
                        float res[32];
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            res[x] = al * (__uint_as_float(ov[x]) * inv_l) +
                                     (1.f - al) * (__uint_as_float(lv[x]) * inv_den);
                        store_row32(a.out, a.out_f32, grow * D + c, res);
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, NCOLS);
}

}  // namespace sla

// cocluster.cuh -- SVOO online bidirectional Q-K co-clustering ("Training-Free
// Sparse Attention for Fast Video Generation via Offline Layer-Wise Sparsity
// Profiling and Online Bidirectional Co-Clustering", sec. 2.B): keys are
// assigned to the cluster whose query centroid they have the largest affinity
// (dot product) with, then queries to the cluster of the largest affinity with
// the updated key centroids, alternately; the tokens are then ordered stably by
// cluster, so that the block-sparse path's contiguous blocks group tokens of one
// cluster.  Everything is fp64 from the bf16 inputs (centroid sums of bf16
// values are exact in fp64, so a centroid does not depend on summation order).
//
// Per head and per half-step:
//   cc_assign_kernel    label[n] = argmax over non-empty clusters c of x_n . cent_c
//                       (ties to the lower c), two tokens per thread, 16 centroids
//                       at a time in shared memory;
//   cc_count_kernel     per chunk of 1024 tokens, the tokens per label;
//   cc_scan_kernel      each chunk's first sorted position per label;
//   cc_scatter_kernel   perm[pos] = n, stable within a label (one warp per chunk,
//                       tokens in order);
//   cc_means_kernel     cent_c = mean of the label's tokens, in sorted order (a
//                       cluster without tokens is marked empty).
#pragma once
#include "common.cuh"

namespace sla {

constexpr int kCcChunk = 1024;     // tokens per counting-sort chunk
constexpr int kCcTile = 16;        // centroids per shared-memory tile of the assignment

// Initial query centroids: means of C contiguous chunks of N/C rows.
// grid (C, BH), D threads.
template <int D>
__global__ void __launch_bounds__(128) cc_chunk_mean_kernel(const __nv_bfloat16* __restrict__ x, int N, int C,
                                                            double* __restrict__ cent, int* __restrict__ valid) {
    const int c = blockIdx.x;
    const long long bh = blockIdx.y;
    const int rows = N / C;
    const __nv_bfloat16* xr = x + (bh * N + static_cast<long long>(c) * rows) * D + threadIdx.x;
    double s = 0.0;
    for (int r = 0; r < rows; ++r) s += static_cast<double>(__bfloat162float(xr[static_cast<long long>(r) * D]));
    cent[(bh * C + c) * D + threadIdx.x] = s / rows;
    if (threadIdx.x == 0) valid[bh * C + c] = 1;
}

// label[bh][n] = argmax over valid c of x[bh][n] . cent[bh][c].
// grid (ceil(N/256), BH), 128 threads, each with two tokens (t and t + 128 of
// the CTA's 256), so that every centroid coordinate read from shared memory
// serves two FMAs; dynamic shared memory: the CTA's tokens transposed (bf16
// [D][kCcPitch]), a tile of kCcTile centroids transposed (fp64 [D][kCcTile]: one
// 16-byte read gives two centroids' coordinate) and their empty flags.  The
// tokens arrive in 16-byte loads, eight in flight per thread; the next centroid
// tile is loaded into registers while the current one is in use.  Each dot
// product is summed over the coordinates in order.
constexpr int kCcPitch = 260;
constexpr int kCcTok = 256;        // tokens per CTA
template <int D>
constexpr size_t cc_assign_smem() { return static_cast<size_t>(D) * kCcPitch * 2 + kCcTile * D * 8 + kCcTile * 4; }

template <int D>
__global__ void __launch_bounds__(128) cc_assign_kernel(const __nv_bfloat16* __restrict__ x, int N, int C,
                                                        const double* __restrict__ cent,
                                                        const int* __restrict__ valid, int* __restrict__ label) {
    extern __shared__ __align__(16) unsigned char cc_smem[];
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(cc_smem);                       // [D][kCcPitch]
    double* cs = reinterpret_cast<double*>(cc_smem + static_cast<size_t>(D) * kCcPitch * 2);   // [D][kCcTile]
    int* vs = reinterpret_cast<int*>(cs + kCcTile * D);                                   // [kCcTile]
    constexpr int kPer = kCcTile * D / 128;                                                // tile values per thread
    const long long bh = blockIdx.y;
    const int n0 = blockIdx.x * kCcTok;
    const int t = threadIdx.x;
    // the first centroid tile into registers (consecutive threads: consecutive centroids)
    double pre[kPer];
    int pre_v = 0;
    auto fetch = [&](int c0) {
        const int nt = min(kCcTile, C - c0);
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = t + 128 * u;
            const int jc = i % kCcTile, dd = i / kCcTile;
            pre[u] = jc < nt ? cent[(bh * C + c0 + jc) * D + dd] : 0.0;
        }
        pre_v = t < nt ? valid[bh * C + c0 + t] : 0;
    };
    fetch(0);
    // stage the CTA's tokens, transposed so that thread t reads columns t and t + 128:
    // unit u of 16 bytes is row r = u % 256, coordinates 8 (u / 256) .. + 7
    constexpr int kUnits = kCcTok * D / 8 / 128;                                           // per thread
    static_assert(kUnits % 8 == 0, "eight loads in flight");
#pragma unroll 1
    for (int u0 = 0; u0 < kUnits; u0 += 8) {
        uint4 buf[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int u = t + 128 * (u0 + j);
            const int r = u % kCcTok, n = n0 + r;
            buf[j] = n < N ? *reinterpret_cast<const uint4*>(x + (bh * N + n) * D + (u / kCcTok) * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int u = t + 128 * (u0 + j);
            const int r = u % kCcTok, d0 = (u / kCcTok) * 8;
            const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&buf[j]);
#pragma unroll
            for (int q = 0; q < 8; ++q) xs[(d0 + q) * kCcPitch + r] = e[q];
        }
    }
    double best[2] = {-INFINITY, -INFINITY};
    int arg[2] = {-1, -1};
    for (int c0 = 0; c0 < C; c0 += kCcTile) {
        __syncthreads();
        const int nt = min(kCcTile, C - c0);
#pragma unroll
        for (int u = 0; u < kPer; ++u) cs[t + 128 * u] = pre[u];
        if (t < kCcTile) vs[t] = pre_v;
        __syncthreads();
        if (c0 + kCcTile < C) fetch(c0 + kCcTile);
        double a0[kCcTile], a1[kCcTile];
#pragma unroll
        for (int j = 0; j < kCcTile; ++j) a0[j] = a1[j] = 0.0;
#pragma unroll 2
        for (int dd = 0; dd < D; ++dd) {
            const double x0 = static_cast<double>(__bfloat162float(xs[dd * kCcPitch + t]));
            const double x1 = static_cast<double>(__bfloat162float(xs[dd * kCcPitch + t + 128]));
            const double2* c2 = reinterpret_cast<const double2*>(cs + dd * kCcTile);
#pragma unroll
            for (int j = 0; j < kCcTile / 2; ++j) {
                const double2 cc = c2[j];
                a0[2 * j] = fma(x0, cc.x, a0[2 * j]);
                a0[2 * j + 1] = fma(x0, cc.y, a0[2 * j + 1]);
                a1[2 * j] = fma(x1, cc.x, a1[2 * j]);
                a1[2 * j + 1] = fma(x1, cc.y, a1[2 * j + 1]);
            }
        }
#pragma unroll
        for (int j = 0; j < kCcTile; ++j) {
            if (j < nt && vs[j]) {
                if (arg[0] < 0 || a0[j] > best[0]) { best[0] = a0[j]; arg[0] = c0 + j; }
                if (arg[1] < 0 || a1[j] > best[1]) { best[1] = a1[j]; arg[1] = c0 + j; }
            }
        }
    }
    if (n0 + t < N) label[bh * N + n0 + t] = arg[0] < 0 ? 0 : arg[0];
    if (n0 + t + 128 < N) label[bh * N + n0 + t + 128] = arg[1] < 0 ? 0 : arg[1];
}

// counts[bh][chunk][c] = tokens of the chunk with label c.  grid (nchunk, BH), 256 threads.
__global__ void __launch_bounds__(256) cc_count_kernel(const int* __restrict__ label, int N, int C, int nchunk,
                                                       int* __restrict__ counts) {
    extern __shared__ int hist[];
    const long long bh = blockIdx.y;
    const int chunk = blockIdx.x;
    for (int c = threadIdx.x; c < C; c += 256) hist[c] = 0;
    __syncthreads();
    const int n0 = chunk * kCcChunk, n1 = min(N, n0 + kCcChunk);
    for (int n = n0 + threadIdx.x; n < n1; n += 256) {
        const int l = label[bh * N + n];
        if (l >= 0 && l < C) atomicAdd(&hist[l], 1);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += 256) counts[(bh * nchunk + chunk) * C + c] = hist[c];
}

// base[bh][chunk][c] = first sorted position of the chunk's label-c tokens;
// start[bh][c], count[bh][c] = the label's range.  grid (BH), 1024 threads.
__global__ void __launch_bounds__(1024) cc_scan_kernel(const int* __restrict__ counts, int C, int nchunk,
                                                       int* __restrict__ base, int* __restrict__ start,
                                                       int* __restrict__ count) {
    __shared__ int tot[1024];
    const long long bh = blockIdx.x;
    const int c = threadIdx.x;
    int run = 0;
    if (c < C)
        for (int k = 0; k < nchunk; ++k) {
            base[(bh * nchunk + k) * C + c] = run;
            run += counts[(bh * nchunk + k) * C + c];
        }
    tot[c] = c < C ? run : 0;
    __syncthreads();
    // exclusive scan of the totals over the labels (Hillis-Steele, 1024 entries)
    for (int off = 1; off < 1024; off <<= 1) {
        const int v = c >= off ? tot[c - off] : 0;
        __syncthreads();
        tot[c] += v;
        __syncthreads();
    }
    if (c < C) {
        const int st = tot[c] - run;
        start[bh * C + c] = st;
        count[bh * C + c] = run;
        for (int k = 0; k < nchunk; ++k) base[(bh * nchunk + k) * C + c] += st;
    }
}

// perm[bh][pos] = n for the chunk's tokens, stable within each label.
// grid (nchunk, BH), 32 threads (one warp walks the chunk in order).
__global__ void __launch_bounds__(32) cc_scatter_kernel(const int* __restrict__ label, int N, int C, int nchunk,
                                                        const int* __restrict__ base, int* __restrict__ perm) {
    extern __shared__ int run[];
    const long long bh = blockIdx.y;
    const int chunk = blockIdx.x;
    const int lane = threadIdx.x;
    for (int c = lane; c < C; c += 32) run[c] = base[(bh * nchunk + chunk) * C + c];
    __syncwarp();
    const int n0 = chunk * kCcChunk, n1 = min(N, n0 + kCcChunk);
    const uint32_t lt = (1u << lane) - 1u;
    for (int nb = n0; nb < n1; nb += 32) {
        const int n = nb + lane;
        const bool in = n < n1;
        const int l = in ? label[bh * N + n] : -1;
        const bool ok = in && l >= 0 && l < C;
        const uint32_t act = __ballot_sync(0xffffffffu, ok);
        const uint32_t same = __match_any_sync(0xffffffffu, ok ? l : -1) & act;
        if (ok) {
            const int rank = __popc(same & lt);
            const int pos = run[l] + rank;
            if (pos >= 0 && pos < N) perm[bh * N + pos] = n;
            else report(kStatusBadData);
        }
        __syncwarp();
        if (ok && (same & lt) == 0) run[l] += __popc(same);   // the label's first lane advances it
        __syncwarp();
    }
}

// cent[bh][c] = mean of rows perm[start_c .. start_c + count_c); a label
// without tokens is marked empty and keeps its old centroid.  D/8 threads share
// a row (16-byte loads of eight coordinates), so kCcMeanThreads*8/D rows are
// read at a time, four per thread in flight.  Sums of bf16 values in fp64 are
// exact while the values' binary exponents span less than 53 - 8 - log2(rows)
// bits, so the row groups and their combination in a fixed order give the
// value of any order.  grid (C, BH), kCcMeanThreads threads.
constexpr int kCcMeanThreads = 512;
template <int D>
__global__ void __launch_bounds__(kCcMeanThreads) cc_means_kernel(const __nv_bfloat16* __restrict__ x, int N, int C,
                                                                 const int* __restrict__ perm,
                                                                 const int* __restrict__ start,
                                                                 const int* __restrict__ count,
                                                                 double* __restrict__ cent,
                                                                 int* __restrict__ valid) {
    constexpr int L = D / 8, R = kCcMeanThreads / L;      // threads per row, rows at a time
    __shared__ double part[R][D];
    const int c = blockIdx.x;
    const long long bh = blockIdx.y;
    const int k8 = (threadIdx.x % L) * 8, grp = threadIdx.x / L;
    const int st = start[bh * C + c], cnt = count[bh * C + c];
    if (cnt <= 0) {
        if (threadIdx.x == 0) valid[bh * C + c] = 0;
        return;
    }
    double s[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) s[q] = 0.0;
    for (int i0 = grp; i0 < cnt; i0 += 4 * R) {
        int n[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) n[u] = i0 + u * R < cnt ? perm[bh * N + st + i0 + u * R] : -1;
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            v[u] = n[u] >= 0 ? *reinterpret_cast<const uint4*>(x + (bh * N + n[u]) * D + k8) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v[u]);
#pragma unroll
            for (int q = 0; q < 8; ++q) s[q] += static_cast<double>(__bfloat162float(e[q]));
        }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) part[grp][k8 + q] = s[q];
    __syncthreads();
    if (threadIdx.x < D) {
        const int col = threadIdx.x;
        double t = part[0][col];
        for (int g2 = 1; g2 < R; ++g2) t += part[g2][col];
        cent[(bh * C + c) * D + col] = t / cnt;
        if (col == 0) valid[bh * C + c] = 1;
    }
}

// dst row (bh, i) = src row (bh, perm[bh][i]) (inverse: dst row (bh, perm[bh][i])
// = src row (bh, i)); rows of row_words 32-bit words (VEC: 16-byte words).
// A perm entry outside [0, N) is skipped and flagged.  Grid-stride over rows,
// kPermRows rows per thread at a time (their perm entries first, then their
// loads), so that several loads are in flight behind each index load.
constexpr int kPermRows = 4;
template <typename T>
__global__ void __launch_bounds__(256) permute_rows_kernel(const T* __restrict__ src, const int* __restrict__ perm,
                                                           T* __restrict__ dst, long long BH, int N, int row_words,
                                                           int inverse) {
    const long long rows = BH * N;
    const int per_row = max(1, 256 / row_words);      // rows handled by one CTA pass
    const int rr = threadIdx.x / row_words, w = threadIdx.x % row_words;
    if (rr >= per_row) return;
    const long long step = static_cast<long long>(gridDim.x) * per_row;
    for (long long r0 = static_cast<long long>(blockIdx.x) * per_row + rr; r0 < rows; r0 += kPermRows * step) {
        int p[kPermRows];
#pragma unroll
        for (int u = 0; u < kPermRows; ++u) {
            const long long r = r0 + u * step;
            p[u] = r < rows ? perm[r] : -1;
        }
        T v[kPermRows] = {};
#pragma unroll
        for (int u = 0; u < kPermRows; ++u) {
            const long long r = r0 + u * step;
            if (r < rows && p[u] >= 0 && p[u] < N)
                v[u] = src[(inverse ? r : (r / N) * N + p[u]) * row_words + w];
        }
#pragma unroll
        for (int u = 0; u < kPermRows; ++u) {
            const long long r = r0 + u * step;
            if (r >= rows) continue;
            if (p[u] < 0 || p[u] >= N) { if (w == 0) report(kStatusBadData); continue; }
            dst[(inverse ? (r / N) * N + p[u] : r) * row_words + w] = v[u];
        }
    }
}

}  // namespace sla

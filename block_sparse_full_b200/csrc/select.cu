// Block selection of the SSA sparse stream: mean-pooled block scores and a
// top-k block budget per query block ("Sintesi Tecnica: SSA", section 2,
// Sparse Attention Stream = block-sparse attention; section 4, "Efficienza":
// the same operations as MoBA at inference).
//
// Two steps, on CUDA cores in float64 (the decision is an integer set, so it
// is taken in the precision the definition fixes):
//   pool_kernel       reads Q and K once (HBM-bound) and writes the exact
//                     float64 block means Qbar, Kbar to the workspace;
//   score_topk_kernel one CTA per 8 query blocks of one (b, h), two CTAs per
//                     SM: scores s_ij for j < i (tiled over 8 rows x 4 keys
//                     per warp, fixed summation order), then one warp per
//                     row fills the free slots by warp-argmax rounds under
//                     (score desc, index asc) and writes the ascending
//                     index list by popcount prefix of the set bitmask;
//   score_topk_row_kernel the same selection one CTA per query block, for
//                     rows longer than 1024 blocks.
#include <cstdio>

#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelThreads = 256;
constexpr int kMaxBlocksPerRow = 4096;  // n = T / block limit (score row in smem)

// Units are the B*H*n query blocks followed by the B*H*n key blocks; the
// rows of unit (b,h,i) are contiguous because T = n * block.  A CTA pools U
// consecutive units: every thread first issues all its 16-byte loads (V
// consecutive columns of rows g, g + G, ... of each unit; a warp covers
// whole rows, so they coalesce), then the units are reduced one at a time
// through shared memory in a fixed order.  Each thread keeps 8 to 16 loads
// in flight.  The base pointers are 16-byte aligned (host-checked).
template <typename T, int D, int BLOCK>
struct PoolShape {
    static constexpr int V = 16 / (int)sizeof(T);  // columns per load
    static constexpr int TPR = D / V;               // threads per row
    static constexpr int G = kPoolThreads / TPR;    // row groups
    static constexpr int PER = BLOCK / G;           // rows per thread per unit
    // units per CTA: 8 loads in flight per thread for short rows (more CTAs
    // per SM), 16 for long ones
    static constexpr int U = PER >= 16 ? 1 : (PER >= 8 ? 16 / PER : 8 / PER);
    static_assert(BLOCK % G == 0, "block rows must split evenly over row groups");
};

template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const T* __restrict__ q, const T* __restrict__ k, double* __restrict__ qbar,
            double* __restrict__ kbar, int units_q) {
    using S = PoolShape<T, D, BLOCK>;
    constexpr int V = S::V, TPR = S::TPR, G = S::G, PER = S::PER, U = S::U;
    const int c0 = (threadIdx.x % TPR) * V;
    const int g = threadIdx.x / TPR;
    const int total = 2 * units_q;
    const int unit0 = blockIdx.x * U;

    uint4 raw[U][PER];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int unit = unit0 + u;
        if (unit < total) {
            const T* src = unit < units_q ? q + (size_t)unit * BLOCK * D
                                          : k + (size_t)(unit - units_q) * BLOCK * D;
#pragma unroll
            for (int r = 0; r < PER; ++r)
                raw[u][r] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(g + G * r) * D + c0));
        }
    }

    __shared__ double part[G * D];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int unit = unit0 + u;
        if (unit >= total) break;  // uniform over the CTA
        double acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0;
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const T* x = reinterpret_cast<const T*>(&raw[u][r]);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += (double)to_f32(x[e]);
        }
        if (u > 0) __syncthreads();  // the previous unit's readers are done
#pragma unroll
        for (int e = 0; e < V; ++e) part[g * D + c0 + e] = acc[e];
        __syncthreads();
        double* dst = unit < units_q ? qbar + (size_t)unit * D : kbar + (size_t)(unit - units_q) * D;
        for (int c = threadIdx.x; c < D; c += kPoolThreads) {
            double s = 0.0;
            for (int j = 0; j < G; ++j) s += part[j * D + c];
            dst[c] = s / (double)BLOCK;  // block is a power of two: exact
        }
    }
}

// Rows of R = 8 consecutive query blocks i0 .. i0+7 of one (b, h) per CTA
// (n <= kRowsKernelMaxN).  Scores: warp w takes keys j0 + 4w .. j0 + 4w + 3
// of each group of 32 for all 8 rows at once; the 8 query block means sit in
// shared memory (lane l reads columns l, l+32, ...), so one read of a key
// block mean serves 8 rows, and ~120 registers leave room for two CTAs per SM
// (twice the warps to hide the float64 latencies).  The 32 partial dot
// products of a lane (4 keys x 8 rows) are summed over the warp by a
// transpose-reduce (31 double exchanges), after which lane l owns one
// complete score.  Top-k: warp w alone handles row i0 + w (selection, index
// list, mask, count), with no CTA-wide barrier.  dynamic smem: scores [8][n]
// f64, bits [8][32] u32; static: the 8 query block means.
constexpr int kRowsPerCta = 8;
constexpr int kRowsKernelMaxN = 1024;

template <int D>
__global__ void __launch_bounds__(kSelThreads, 2)
score_topk_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar, int n,
                  int topk, int force_sink, int words, int32_t* __restrict__ idx,
                  int32_t* __restrict__ cnt, uint32_t* __restrict__ mask) {
    constexpr int M = D / 32;
    constexpr int R = kRowsPerCta;
    constexpr int KPW = 32 / R;                   // keys per warp per group
    constexpr int GROUP = (kSelThreads / 32) * KPW;  // keys per group
    static_assert(KPW * R == 32, "one partial per lane after the transpose-reduce");
    extern __shared__ double smem[];
    double* sc = smem;                                                      // [R][n]
    uint32_t* bits_all = reinterpret_cast<uint32_t*>(sc + (size_t)R * n);  // [R][32]

    const int nrb = (n + R - 1) / R;
    const size_t bh = blockIdx.x / nrb;
    const int i0 = (blockIdx.x % nrb) * R;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double* kb = kbar + bh * (size_t)n * D;
    const int kend = min(i0 + R, n) - 1;  // keys j < kend cover every row's j < i

    __shared__ double qs[R * D];  // the R query-block means
    for (int e = threadIdx.x; e < R * D; e += kSelThreads) {
        const int r = e / D, c = e % D;
        qs[e] = qbar[(bh * n + min(i0 + r, n - 1)) * D + c];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < R * 32; t += kSelThreads) bits_all[t] = 0u;

    auto load_group = [&](int j0, double (&kv)[KPW][M]) {
#pragma unroll
        for (int kk = 0; kk < KPW; ++kk) {
            const int j = max(min(j0 + KPW * warp + kk, kend - 1), 0);  // past the end: result unused
            const double* kr = kb + (size_t)j * D + lane;
#pragma unroll
            for (int m = 0; m < M; ++m) kv[kk][m] = kr[32 * m];
        }
    };
    if (kend > 0) {
        double kv[KPW][M];
        for (int j0 = 0; j0 < kend; j0 += GROUP) {
            load_group(j0, kv);
            double v[32];
#pragma unroll
            for (int kk = 0; kk < KPW; ++kk)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    double acc = 0.0;
#pragma unroll
                    for (int m = 0; m < M; ++m) acc = fma(qs[r * D + lane + 32 * m], kv[kk][m], acc);
                    v[kk * R + r] = acc;
                }
            // transpose-reduce: after the step of width s, v[t] (t < s) holds
            // entry t + s * (lane bit s) + (the bits kept before), summed
            // over the lanes that differ in that bit
#pragma unroll
            for (int s = 16; s >= 1; s >>= 1) {
                const bool upper = (lane & s) != 0;
#pragma unroll
                for (int t = 0; t < s; ++t) {
                    const double send = upper ? v[t] : v[t + s];
                    const double keep = upper ? v[t + s] : v[t];
                    v[t] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            }
            const int kk = lane / R, r = lane % R;
            const int j = j0 + KPW * warp + kk;
            if (j < kend) sc[(size_t)r * n + j] = v[0];
        }
    }
    __syncthreads();  // all rows' scores and cleared bits visible

    if (warp >= R) return;
    const int i = i0 + warp;
    if (i >= n) return;
    const size_t row = bh * n + i;
    const double* srow = sc + (size_t)warp * n;
    uint32_t* bits = bits_all + warp * 32;
    const bool sink = force_sink && i > 0;
    if (lane == 0) {
        bits[i >> 5] |= 1u << (i & 31);
        if (sink) bits[0] |= 1u;
    }
    __syncwarp();
    const int first = sink ? 1 : 0;          // candidates are first .. i-1
    const int ncand = i - first;
    const int r = topk - (sink ? 2 : 1);     // free slots (>= 0, host-checked)
    if (ncand <= r) {
        for (int j = first + lane; j < i; j += 32) atomicOr(&bits[j >> 5], 1u << (j & 31));
    } else {
        warp_topk_rounds(srow, first, i, r, bits, lane);
    }
    __syncwarp();
    // ascending index list: lane l owns mask word l (words <= 32)
    const uint32_t wv = lane < words ? bits[lane] : 0u;
    const int c = __popc(wv);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int32_t* irow = idx + row * topk;
    int pos = incl - c;
    for (uint32_t b = wv; b != 0u; b &= b - 1u, ++pos)
        if (pos < topk) irow[pos] = lane * 32 + __ffs(b) - 1;  // NaN scores: stay in bounds
    for (int p = total + lane; p < topk; p += 32) irow[p] = -1;
    if (lane < words) mask[row * words + lane] = wv;
    if (lane == 0) cnt[row] = total < topk ? total : topk;
}

// n > kRowsKernelMaxN: one CTA per (b, h, query block i).
// grid B*H*n; dynamic smem: scores[n] f64, bits[words] u32, prefix[words + 1] i32.
//
// Scores: warp per key block, lane l owns columns l, l + 32, ... (the query
// block mean sits in registers), fixed butterfly sum; each warp keeps the
// loads of U key blocks in flight.  Top-k by warp 0 (warp_topk_rounds).
template <int D>
__global__ void __launch_bounds__(kSelThreads)
score_topk_row_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar, int n,
                  int topk, int force_sink, int words, int32_t* __restrict__ idx,
                  int32_t* __restrict__ cnt, uint32_t* __restrict__ mask) {
    constexpr int M = D / 32;
    constexpr int U = 4;
    extern __shared__ double smem[];
    double* sc = smem;
    uint32_t* bits = reinterpret_cast<uint32_t*>(sc + n);
    int* prefix = reinterpret_cast<int*>(bits + words);

    const int row = blockIdx.x;  // (b*H + h) * n + i
    const int i = row % n;
    const size_t bh = row / n;
    const double* kb = kbar + bh * (size_t)n * D;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    double qr[M];
#pragma unroll
    for (int m = 0; m < M; ++m) qr[m] = qbar[(size_t)row * D + lane + 32 * m];
    for (int w = tid; w < words; w += kSelThreads) bits[w] = 0u;

    for (int j0 = warp * U; j0 < i; j0 += (kSelThreads / 32) * U) {
        double a[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = min(j0 + u, i - 1);  // past the end: a valid row, result unused
            const double* kr = kb + (size_t)j * D + lane;
            double acc = 0.0;
#pragma unroll
            for (int m = 0; m < M; ++m) acc = fma(qr[m], kr[32 * m], acc);
            a[u] = acc;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) a[u] = warp_sum(a[u]);
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (j0 + u < i) sc[j0 + u] = a[u];
        }
    }
    const bool sink = force_sink && i > 0;
    __syncthreads();  // scores and cleared bits visible
    if (tid == 0) {
        bits[i >> 5] |= 1u << (i & 31);
        if (sink) bits[0] |= 1u;
    }
    __syncthreads();

    const int first = sink ? 1 : 0;          // candidates are first .. i-1
    const int ncand = i - first;
    const int r = topk - (sink ? 2 : 1);     // free slots (>= 0, host-checked)
    if (ncand <= r) {
        for (int j = first + tid; j < i; j += kSelThreads) atomicOr(&bits[j >> 5], 1u << (j & 31));
    } else if (warp == 0) {
        warp_topk_rounds(sc, first, i, r, bits, lane);
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int w = 0; w < words; ++w) {
            prefix[w] = acc;
            acc += __popc(bits[w]);
        }
        prefix[words] = acc;
    }
    __syncthreads();
    const int total = prefix[words];
    int32_t* irow = idx + (size_t)row * topk;
    for (int j = tid; j <= i; j += kSelThreads) {
        const uint32_t wv = bits[j >> 5];
        if ((wv >> (j & 31)) & 1u) {
            const int pos = prefix[j >> 5] + __popc(wv & ((1u << (j & 31)) - 1u));
            if (pos < topk) irow[pos] = j;
        }
    }
    for (int p = total + tid; p < topk; p += kSelThreads) irow[p] = -1;
    for (int w = tid; w < words; w += kSelThreads) mask[(size_t)row * words + w] = bits[w];
    if (tid == 0) cnt[row] = total < topk ? total : topk;
}

template <typename T, int D, int BLOCK>
int launch_pool(const void* q, const void* k, double* qbar, double* kbar, size_t units_q,
                cudaStream_t s) {
    constexpr int U = PoolShape<T, D, BLOCK>::U;
    const size_t grid = (2 * units_q + U - 1) / U;
    pool_kernel<T, D, BLOCK><<<(unsigned)grid, kPoolThreads, 0, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), qbar, kbar, (int)units_q);
    return check_launch("pool_kernel");
}

template <typename T>
int launch_pool_t(const ssa_params_t& p, const void* q, const void* k, double* qbar, double* kbar,
                  size_t units_q, cudaStream_t s) {
    if (p.D == 64)
        return p.block == 64 ? launch_pool<T, 64, 64>(q, k, qbar, kbar, units_q, s)
                             : launch_pool<T, 64, 128>(q, k, qbar, kbar, units_q, s);
    return p.block == 64 ? launch_pool<T, 128, 64>(q, k, qbar, kbar, units_q, s)
                         : launch_pool<T, 128, 128>(q, k, qbar, kbar, units_q, s);
}

template <int D>
int launch_score(const ssa_params_t& p, const double* qbar, const double* kbar, size_t rows,
                 int32_t* idx, int32_t* cnt, uint32_t* mask, cudaStream_t s) {
    const int n = num_blocks(p);
    const int words = mask_words(p);
    const int sink = (p.flags & SSA_FLAG_FORCE_SINK) ? 1 : 0;
    if (n <= kRowsKernelMaxN) {
        const size_t smem = (size_t)kRowsPerCta * n * 8 + kRowsPerCta * 32 * 4;
        int st = opt_in_max_smem<score_topk_kernel<D>>("score_topk_kernel");
        if (st != SSA_OK) return st;
        const size_t grid = (size_t)p.B * p.H * ((n + kRowsPerCta - 1) / kRowsPerCta);
        score_topk_kernel<D><<<(unsigned)grid, kSelThreads, smem, s>>>(qbar, kbar, n, p.topk, sink,
                                                                       words, idx, cnt, mask);
        return check_launch("score_topk_kernel");
    }
    const size_t smem = (size_t)n * 8 + (size_t)words * 4 + (size_t)(words + 1) * 4;
    int st = opt_in_max_smem<score_topk_row_kernel<D>>("score_topk_row_kernel");
    if (st != SSA_OK) return st;
    score_topk_row_kernel<D><<<(unsigned)rows, kSelThreads, smem, s>>>(qbar, kbar, n, p.topk, sink,
                                                                       words, idx, cnt, mask);
    return check_launch("score_topk_row_kernel");
}

}  // namespace

size_t select_workspace(const ssa_params_t& p) {
    // Qbar and Kbar, float64 [B, H, n, D] each
    return 2 * align_up((size_t)p.B * p.H * num_blocks(p) * p.D * sizeof(double), 256);
}

int launch_select(const ssa_params_t& p, const void* q, const void* k, int32_t* idx,
                  int32_t* cnt, uint32_t* mask, void* ws, cudaStream_t s) {
    const int n = num_blocks(p);
    if (n > kMaxBlocksPerRow)
        return fail(SSA_ERR_UNSUPPORTED, "select: T/block = %d exceeds %d", n, kMaxBlocksPerRow);
    const size_t rows = (size_t)p.B * p.H * n;
    if (2 * rows > 0x7fffffffull) return fail(SSA_ERR_UNSUPPORTED, "select: B*H*n too large");
    if ((p.D != 64 && p.D != 128) || (p.block != 64 && p.block != 128))
        return fail(SSA_ERR_UNSUPPORTED, "select: D and block must be 64 or 128");
    double* qbar = static_cast<double*>(ws);
    double* kbar = reinterpret_cast<double*>(static_cast<char*>(ws) + select_workspace(p) / 2);

    int st = p.dtype == SSA_F32 ? launch_pool_t<float>(p, q, k, qbar, kbar, rows, s)
                                : launch_pool_t<__nv_bfloat16>(p, q, k, qbar, kbar, rows, s);
    if (st != SSA_OK) return st;
    return p.D == 64 ? launch_score<64>(p, qbar, kbar, rows, idx, cnt, mask, s)
                     : launch_score<128>(p, qbar, kbar, rows, idx, cnt, mask, s);
}

}  // namespace ssa

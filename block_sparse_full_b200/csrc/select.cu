// Block selection of the SSA sparse stream: mean-pooled block scores and a
// top-k block budget per query block ("Sintesi Tecnica: SSA", section 2,
// Sparse Attention Stream = block-sparse attention; section 4, "Efficienza":
// the same operations as MoBA at inference).
//
// Two steps in float64 (the decision is an integer set, so it is taken in the
// precision the definition fixes):
//   pool_ring_kernel  (bf16; pool_kernel for f32) reads Q and K once
//                     (HBM-bound) and writes the exact float64 block means
//                     Qbar, Kbar to the workspace;
//   score_topk_kernel one CTA per 8 query blocks of one (b, h), four CTAs per
//                     SM: scores s_ij for j < i on the float64 tensor cores
//                     (8 rows x 8 keys per DMMA tile, fixed summation
//                     order), then one warp per row fills the free slots by
//                     warp rounds under (score desc, index asc) and writes
//                     the ascending index list by popcount prefix of the
//                     set bitmask;
//   score_topk_row_kernel the same selection one CTA per query block, for
//                     rows longer than 1024 blocks.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "device_util.cuh"
#include "ssa_internal.h"
#include "tc_util.cuh"

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

using tc::fence_mbar_init;
using tc::kDrainLimitNs;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_try_wait;
using tc::smem_u32;
using tc::globaltimer;

// one-dimensional bulk copy global -> this CTA's shared memory, completing on `bar`
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}
// wait for the phase of parity `parity` (wall-clock bound); false if it expired
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > limit_ns) return false;
    return true;
}

__device__ unsigned int g_select_status;

// bf16 pooling as a persistent stream: CTA c takes units c, c + G, ... (G =
// grid size); one thread keeps NS units in flight with bulk copies (a unit is
// BLOCK contiguous rows, 8 to 32 KB) into a ring of shared-memory stages, and
// all threads reduce each landed unit: thread (column pair, row group) sums its
// rows in float64, the row groups are added in a fixed order.  The copies of
// the next units overlap the conversions of this one, so HBM stays busy.
template <int D, int BLOCK>
struct RingShape {
    static constexpr int UB = BLOCK * D * 2;                     // bytes per unit
    static constexpr int NS = UB <= 16384 ? 6 : 3;               // stages in flight
    static constexpr int CP = D / 2;                             // column pairs
    static constexpr int RG = kPoolThreads / CP;                 // row groups
    static constexpr size_t SMEM = (size_t)NS * UB + 2 * (size_t)RG * D * 8 + 1024;
};

template <int D, int BLOCK>
__global__ void __launch_bounds__(kPoolThreads, 2)
pool_ring_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                 double* __restrict__ qbar, double* __restrict__ kbar, int units_q, int total,
                 unsigned long long limit_ns) {
    using S = RingShape<D, BLOCK>;
    constexpr int UB = S::UB, NS = S::NS, CP = S::CP, RG = S::RG;
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ __align__(8) uint64_t full[NS];
    double* part = reinterpret_cast<double*>(sm + (size_t)NS * UB);  // [2][RG][D]
    const int tid = threadIdx.x;
    const int G = gridDim.x;
    const int mine = blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / G + 1 : 0;
    auto src_of = [&](int l) -> const void* {
        const int u = (int)blockIdx.x + l * G;
        return u < units_q ? (const void*)(q + (size_t)u * BLOCK * D)
                           : (const void*)(k + (size_t)(u - units_q) * BLOCK * D);
    };
    if (tid == 0) {
        for (int st = 0; st < NS; ++st) mbar_init(smem_u32(&full[st]), 1);
        fence_mbar_init();
        for (int l = 0; l < NS && l < mine; ++l) {
            mbar_expect_tx(smem_u32(&full[l]), UB);
            bulk_load_1d(smem_u32(sm + (size_t)l * UB), src_of(l), UB, smem_u32(&full[l]));
        }
    }
    __syncthreads();
    const int cp = tid % CP, rg = tid / CP;
    int l = 0;
    for (; l < mine; ++l) {
        const int st = l % NS;
        if (!__syncthreads_and(mbar_wait_bounded(smem_u32(&full[st]), (l / NS) & 1, limit_ns))) {
            atomicOr(&g_select_status, 1u);
            break;
        }
        const uint32_t* unit = reinterpret_cast<const uint32_t*>(sm + (size_t)st * UB);
        double a0 = 0.0, a1 = 0.0;
#pragma unroll 8
        for (int r = rg; r < BLOCK; r += RG) {
            const uint32_t w = unit[r * CP + cp];  // columns 2 cp, 2 cp + 1 of row r
            a0 += (double)__uint_as_float(w << 16);
            a1 += (double)__uint_as_float(w & 0xffff0000u);
        }
        double* pp = part + (size_t)(l & 1) * RG * D;
        pp[rg * D + 2 * cp] = a0;
        pp[rg * D + 2 * cp + 1] = a1;
        __syncthreads();  // the stage is read and the partials are written
        if (tid == 0 && l + NS < mine) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_expect_tx(smem_u32(&full[st]), UB);
            bulk_load_1d(smem_u32(sm + (size_t)st * UB), src_of(l + NS), UB, smem_u32(&full[st]));
        }
        if (tid < D) {
            double sum = 0.0;
#pragma unroll
            for (int g = 0; g < RG; ++g) sum += pp[g * D + tid];
            const int u = (int)blockIdx.x + l * G;
            double* dst = u < units_q ? qbar + (size_t)u * D : kbar + (size_t)(u - units_q) * D;
            dst[tid] = sum / (double)BLOCK;  // block is a power of two: exact
        }
    }
    if (l < mine && tid == 0) {
        // a wait expired: let the copies already issued land before the CTA exits
        for (int l2 = l; l2 < mine && l2 < l + NS; ++l2)
            mbar_wait_bounded(smem_u32(&full[l2 % NS]), (l2 / NS) & 1, kDrainLimitNs);
    }
}

// The selection order (score desc, index asc) on integers: the float64 score
// mapped to a u64 whose unsigned order is the score's order (-0 taken as +0,
// so that equal scores give equal keys).
__device__ __forceinline__ uint64_t order_key(double x) {
    const uint64_t b = (uint64_t)__double_as_longlong(x == 0.0 ? 0.0 : x);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ void dmma8(double (&c)[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(c[0]), "+d"(c[1])
                 : "d"(a), "d"(b));
}

// (key, index) a ranks ahead of b: larger key, or equal key and lower index
__device__ __forceinline__ bool ahead(uint64_t ka, int ja, uint64_t kb, int jb) {
    return ka > kb || (ka == kb && ja < jb);
}

// Top r of at most 128 candidates first .. i-1 of one row: each lane holds
// its (up to four) candidates sorted in registers; a round takes the largest
// head with one warp max-reduction of the high key words when that maximum
// is held by one lane (the common case), else by the full (high, low, index)
// reductions; the winning lane shifts its list.
__device__ __forceinline__ void warp_topk_keys_small(const uint64_t* key, int first, int i, int r,
                                                     uint32_t* bits, int lane) {
    uint64_t k4[4];
    int j4[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int j = first + lane + 32 * m;
        j4[m] = j < i ? j : 0x7fffffff;
        k4[m] = j < i ? key[j] : 0ull;
    }
    auto cswap = [&](int a, int b) {  // sorting network step: list order (key desc, index asc)
        if (ahead(k4[b], j4[b], k4[a], j4[a])) {
            const uint64_t tk = k4[a];
            k4[a] = k4[b];
            k4[b] = tk;
            const int tj = j4[a];
            j4[a] = j4[b];
            j4[b] = tj;
        }
    };
    cswap(0, 1);
    cswap(2, 3);
    cswap(0, 2);
    cswap(1, 3);
    cswap(1, 2);
    for (int round = 0; round < r; ++round) {
        const bool have = j4[0] != 0x7fffffff;
        const uint32_t hi = have ? (uint32_t)(k4[0] >> 32) : 0u;
        const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
        const uint32_t tie = __ballot_sync(0xffffffffu, have && hi == mhi);
        if (tie == 0u) break;  // no candidate left
        int wl;
        if (__popc(tie) == 1) {
            wl = __ffs(tie) - 1;
        } else {
            const bool top = (tie >> lane) & 1u;
            const uint32_t mlo = __reduce_max_sync(0xffffffffu, top ? (uint32_t)k4[0] : 0u);
            const bool win = top && (uint32_t)k4[0] == mlo;
            const uint32_t wj = __reduce_min_sync(0xffffffffu, win ? (uint32_t)j4[0] : 0xffffffffu);
            wl = __ffs(__ballot_sync(0xffffffffu, win && (uint32_t)j4[0] == wj)) - 1;
        }
        if (lane == wl) {
            atomicOr(&bits[j4[0] >> 5], 1u << (j4[0] & 31));
            k4[0] = k4[1];
            j4[0] = j4[1];
            k4[1] = k4[2];
            j4[1] = j4[2];
            k4[2] = k4[3];
            j4[2] = j4[3];
            k4[3] = 0ull;
            j4[3] = 0x7fffffff;
        }
    }
}

// Top r of the candidates first .. i-1 of one row (order keys in shared memory)
// by warp rounds: each lane holds its best remaining candidate; a round finds
// the largest key with two warp max-reductions (high and low word) and the
// lowest index holding it with a min-reduction; the winner's lane rescans its
// own candidates for the best one below the winner.
__device__ __forceinline__ void warp_topk_keys(const uint64_t* key, int first, int i, int r,
                                               uint32_t* bits, int lane) {
    uint64_t bk = 0;
    int bj = -1;
    for (int j = first + lane; j < i; j += 32) {
        const uint64_t x = key[j];
        if (bj < 0 || x > bk) {  // ascending j: equal keys keep the lower index
            bk = x;
            bj = j;
        }
    }
    for (int round = 0; round < r; ++round) {
        const uint32_t hi = bj < 0 ? 0u : (uint32_t)(bk >> 32);
        const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
        const bool top = bj >= 0 && hi == mhi;
        const uint32_t mlo = __reduce_max_sync(0xffffffffu, top ? (uint32_t)bk : 0u);
        const bool win = top && (uint32_t)bk == mlo;
        const uint32_t wj = __reduce_min_sync(0xffffffffu, win ? (uint32_t)bj : 0xffffffffu);
        if (wj == 0xffffffffu) break;  // no candidate left
        if ((uint32_t)bj == wj) {
            atomicOr(&bits[wj >> 5], 1u << (wj & 31));
            const uint64_t wk = bk;
            bj = -1;
            for (int j = first + lane; j < i; j += 32) {
                const uint64_t x = key[j];
                if (!(x < wk || (x == wk && j > (int)wj))) continue;  // taken already
                if (bj < 0 || x > bk) {
                    bk = x;
                    bj = j;
                }
            }
        }
    }
}

// Rows of R = 8 consecutive query blocks i0 .. i0+7 of one (b, h) per CTA
// (n <= kRowsKernelMaxN).  Scores on the float64 tensor cores: warp w takes
// the 8-key tiles j0 = 8 w, 8 (w + 8), ...; one DMMA (m8n8k4) per 4 columns
// with A = the 8 query-block means (shared memory, rows padded to D + 4
// doubles) and B = the tile's 8 key-block means (read from L2), so C holds
// the tile's 8 x 8 scores.  The column steps go to four accumulator chains
// (step mod 4, added pairwise at the end: a fixed order) so that a tile's
// MMAs overlap; 64 registers leave room for four CTAs per SM.  The scores'
// order keys go to shared memory.  Top-k: warp w alone handles row i0 + w
// (selection, index list, mask, count), with no CTA-wide barrier; rows of at
// most 128 candidates keep them sorted in registers.  dynamic smem: keys
// [8][n] u64, bits [8][32] u32; static: the 8 query block means.
constexpr int kRowsPerCta = 8;
constexpr int kRowsKernelMaxN = 1024;

template <int D>
__global__ void __launch_bounds__(kSelThreads, 4)
score_topk_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar, int n,
                  int topk, int force_sink, int words, int32_t* __restrict__ idx,
                  int32_t* __restrict__ cnt, uint32_t* __restrict__ mask) {
    constexpr int R = kRowsPerCta;
    constexpr int NW = kSelThreads / 32;
    constexpr int QS = D + 4;  // padded row of the query-block means
    static_assert(R == 8, "the DMMA tile has 8 rows");
    extern __shared__ uint64_t smem_u64[];
    uint64_t* sc = smem_u64;                                                // [R][n]
    uint32_t* bits_all = reinterpret_cast<uint32_t*>(sc + (size_t)R * n);  // [R][32]

    const int nrb = (n + R - 1) / R;
    const size_t bh = blockIdx.x / nrb;
    const int i0 = (blockIdx.x % nrb) * R;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double* kb = kbar + bh * (size_t)n * D;
    const int kend = min(i0 + R, n) - 1;  // keys j < kend cover every row's j < i

    __shared__ double qs[R * QS];  // the R query-block means
    for (int e = threadIdx.x; e < R * D; e += kSelThreads) {
        const int r = e / D, c = e % D;
        qs[r * QS + c] = qbar[(bh * n + min(i0 + r, n - 1)) * D + c];
    }
    for (int t = threadIdx.x; t < R * 32; t += kSelThreads) bits_all[t] = 0u;
    __syncthreads();

    {
        const int g = lane >> 2, t = lane & 3;  // fragment row / column of the DMMA
        const double* qr = qs + g * QS + t;
        // one tile at a time, summed in four chains (column steps s mod 4) so
        // that the float64 MMAs of a tile overlap
        for (int j0 = 8 * warp; j0 < kend; j0 += 8 * NW) {
            const double* kr = kb + (size_t)min(j0 + g, kend - 1) * D + t;  // past the end: unused
            double c[4][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
#pragma unroll 16
            for (int s4 = 0; s4 < D / 4; ++s4) dmma8(c[s4 & 3], qr[4 * s4], kr[4 * s4]);
            const int j = j0 + 2 * t;  // C[g][2t], C[g][2t + 1]: row i0 + g, keys j, j + 1
            if (j < kend) sc[(size_t)g * n + j] = order_key((c[0][0] + c[1][0]) + (c[2][0] + c[3][0]));
            if (j + 1 < kend) sc[(size_t)g * n + j + 1] = order_key((c[0][1] + c[1][1]) + (c[2][1] + c[3][1]));
        }
    }
    __syncthreads();  // all rows' keys visible

    if (warp >= R) return;
    const int i = i0 + warp;
    if (i >= n) return;
    const size_t row = bh * n + i;
    const uint64_t* srow = sc + (size_t)warp * n;
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
    } else if (ncand <= 128) {
        warp_topk_keys_small(srow, first, i, r, bits, lane);
    } else {
        warp_topk_keys(srow, first, i, r, bits, lane);
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
    // word by word, lane l places bit l: no lane walks its word's bits one by one
    for (int w = 0; w <= (i >> 5); ++w) {
        const uint32_t ww = __shfl_sync(0xffffffffu, wv, w);
        const int before = __shfl_sync(0xffffffffu, incl - c, w);
        if ((ww >> lane) & 1u) {
            const int pos = before + __popc(ww & ((1u << lane) - 1u));
            if (pos < topk) irow[pos] = w * 32 + lane;  // NaN scores: stay in bounds
        }
    }
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

template <int D, int BLOCK>
int launch_pool_ring(const void* q, const void* k, double* qbar, double* kbar, size_t units_q,
                     cudaStream_t s) {
    using S = RingShape<D, BLOCK>;
    static int sms = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    });
    int st = opt_in_max_smem<pool_ring_kernel<D, BLOCK>>("pool_ring_kernel");
    if (st != SSA_OK) return st;
    const size_t total = 2 * units_q;
    const size_t grid = std::min(total, (size_t)(sms > 0 ? sms : 148) * 2);
    pool_ring_kernel<D, BLOCK><<<(unsigned)grid, kPoolThreads, S::SMEM, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qbar, kbar,
        (int)units_q, (int)total, wait_limit_ns());
    return check_launch("pool_ring_kernel");
}

template <typename T>
int launch_pool_t(const ssa_params_t& p, const void* q, const void* k, double* qbar, double* kbar,
                  size_t units_q, cudaStream_t s) {
    if constexpr (sizeof(T) == 2) {
        if (p.D == 64)
            return p.block == 64 ? launch_pool_ring<64, 64>(q, k, qbar, kbar, units_q, s)
                                 : launch_pool_ring<64, 128>(q, k, qbar, kbar, units_q, s);
        return p.block == 64 ? launch_pool_ring<128, 64>(q, k, qbar, kbar, units_q, s)
                             : launch_pool_ring<128, 128>(q, k, qbar, kbar, units_q, s);
    } else {
        if (p.D == 64)
            return p.block == 64 ? launch_pool<T, 64, 64>(q, k, qbar, kbar, units_q, s)
                                 : launch_pool<T, 64, 128>(q, k, qbar, kbar, units_q, s);
        return p.block == 64 ? launch_pool<T, 128, 64>(q, k, qbar, kbar, units_q, s)
                             : launch_pool<T, 128, 128>(q, k, qbar, kbar, units_q, s);
    }
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

int select_take_status() {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_select_status, sizeof v);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_select_status, &zero, sizeof zero);
        return fail(SSA_ERR_TIMEOUT, "pooling: a wait for a bulk copy expired");
    }
    return SSA_OK;
}

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

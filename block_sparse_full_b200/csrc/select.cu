// Block selection of the SSA sparse stream: mean-pooled block scores and a
// top-k block budget per query block ("Sintesi Tecnica: SSA", section 2,
// Sparse Attention Stream = block-sparse attention; section 4, "Efficienza":
// the same operations as MoBA at inference).
//
// Two kernels, both on CUDA cores in float64 (the decision is an integer
// set, so it is taken in the precision the definition fixes):
//   pool_kernel       reads Q and K once (HBM-bound) and writes the exact
//                     float64 block means Qbar, Kbar to the workspace;
//   score_topk_kernel one CTA per (b, h, query block i): scores s_ij for
//                     j < i (warp per key block, lanes split d, fixed
//                     butterfly order), then each candidate's rank under
//                     (score desc, index asc) and the set bitmask, then the
//                     ascending index list by popcount prefix.
#include <cstdio>

#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelThreads = 256;
constexpr int kMaxBlocksPerRow = 4096;  // n = T / block limit (score row in smem)

// grid (B*H*n, 2): y = 0 pools q, y = 1 pools k.  Block (b,h,i) rows are
// contiguous because T = n * block.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const T* __restrict__ q, const T* __restrict__ k, double* __restrict__ qbar,
            double* __restrict__ kbar, int D, int block) {
    const T* src = (blockIdx.y == 0 ? q : k) + (size_t)blockIdx.x * block * D;
    double* dst = (blockIdx.y == 0 ? qbar : kbar) + (size_t)blockIdx.x * D;
    const int c = threadIdx.x % D;
    const int g = threadIdx.x / D;
    const int G = kPoolThreads / D;
    double acc = 0.0;
    for (int r = g; r < block; r += G) acc += (double)to_f32(src[(size_t)r * D + c]);
    __shared__ double part[kPoolThreads];
    part[threadIdx.x] = acc;
    __syncthreads();
    if (g == 0) {
        double s = 0.0;
        for (int j = 0; j < G; ++j) s += part[j * D + c];
        dst[c] = s / (double)block;  // block is a power of two: exact
    }
}

// grid B*H*n; dynamic smem: scores[n] f64, qrow[D] f64, bits[words] u32,
// prefix[words + 1] i32.
__global__ void __launch_bounds__(kSelThreads)
score_topk_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar, int n,
                  int D, int topk, int force_sink, int words, int32_t* __restrict__ idx,
                  int32_t* __restrict__ cnt, uint32_t* __restrict__ mask) {
    extern __shared__ double smem[];
    double* sc = smem;
    double* qrow = sc + n;
    uint32_t* bits = reinterpret_cast<uint32_t*>(qrow + D);
    int* prefix = reinterpret_cast<int*>(bits + words);

    const int row = blockIdx.x;  // (b*H + h) * n + i
    const int i = row % n;
    const size_t bh = row / n;
    const double* kb = kbar + bh * (size_t)n * D;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int c = tid; c < D; c += kSelThreads) qrow[c] = qbar[(size_t)row * D + c];
    for (int w = tid; w < words; w += kSelThreads) bits[w] = 0u;
    __syncthreads();

    for (int j = warp; j < i; j += kSelThreads / 32) {
        double acc = 0.0;
        for (int c = lane; c < D; c += 32) acc = fma(qrow[c], kb[(size_t)j * D + c], acc);
        acc = warp_sum(acc);
        if (lane == 0) sc[j] = acc;
    }
    const bool sink = force_sink && i > 0;
    if (tid == 0) {
        atomicOr(&bits[i >> 5], 1u << (i & 31));
        if (sink) atomicOr(&bits[0], 1u);
    }
    __syncthreads();

    const int first = sink ? 1 : 0;          // candidates are first .. i-1
    const int ncand = i - first;
    const int r = topk - (sink ? 2 : 1);     // free slots (>= 0, host-checked)
    for (int j = first + tid; j < i; j += kSelThreads) {
        bool take = true;
        if (ncand > r) {
            const double sj = sc[j];
            int rank = 0;
            for (int j2 = first; j2 < i; ++j2) {
                const double s2 = sc[j2];
                rank += (s2 > sj) || (s2 == sj && j2 < j);
            }
            take = rank < r;
        }
        if (take) atomicOr(&bits[j >> 5], 1u << (j & 31));
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
            if (pos < topk) irow[pos] = j;  // NaN scores can over-select; stay in bounds
        }
    }
    for (int p = total + tid; p < topk; p += kSelThreads) irow[p] = -1;
    for (int w = tid; w < words; w += kSelThreads) mask[(size_t)row * words + w] = bits[w];
    if (tid == 0) cnt[row] = total < topk ? total : topk;
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
    if (rows > 0x7fffffffull) return fail(SSA_ERR_UNSUPPORTED, "select: B*H*n too large");
    double* qbar = static_cast<double*>(ws);
    double* kbar = reinterpret_cast<double*>(static_cast<char*>(ws) + select_workspace(p) / 2);

    dim3 pgrid((unsigned)rows, 2);
    if (p.dtype == SSA_F32)
        pool_kernel<float><<<pgrid, kPoolThreads, 0, s>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), qbar, kbar, p.D, p.block);
    else
        pool_kernel<__nv_bfloat16><<<pgrid, kPoolThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qbar,
            kbar, p.D, p.block);
    int st = check_launch("pool_kernel");
    if (st != SSA_OK) return st;

    const int words = mask_words(p);
    const size_t smem = (size_t)n * 8 + (size_t)p.D * 8 + (size_t)words * 4 + (size_t)(words + 1) * 4;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(score_topk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "select: smem attribute: %s", cudaGetErrorString(e));
    }
    score_topk_kernel<<<(unsigned)rows, kSelThreads, smem, s>>>(
        qbar, kbar, n, p.D, p.topk, (p.flags & SSA_FLAG_FORCE_SINK) ? 1 : 0, words, idx, cnt, mask);
    return check_launch("score_topk_kernel");
}

}  // namespace ssa

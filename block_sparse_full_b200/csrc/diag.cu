// Attention diagnostics ("Sintesi Tecnica: SSA", section 1: the sparse
// stream's error grows with the discarded attention mass delta(t); the pages
// also discuss the first block as an attention sink and the sparsity of
// learned attention):
//   sink(t)       = sum_{s <= t, s < block} exp(sigma q_t . k_s - lse_full(t)),
//                   the full-softmax mass on block 0;
//   mean_delta[h] = mean over t of delta(t),  mean_sink[h] = mean over t of sink(t).
// Two launches: diag_sink_kernel (CUDA cores; K of block 0 staged transposed in
// shared memory, one warp per query row, lane = key) and diag_head_kernel (one
// CTA per head, fixed-order float64 sums: bitwise repeatable).  HBM-bound: the
// first pass reads Q once.
#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerCta = 64;

template <typename T>
__global__ void __launch_bounds__(kThreads)
diag_sink_kernel(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse,
                 int Tn, int D, int nkeys, float scale, float* __restrict__ sink) {
    extern __shared__ float sm[];
    float* kT = sm;                         // [D][nkeys]: lane j reads column j (no conflicts)
    float* qs = sm + (size_t)D * nkeys;     // [8 warps][D]
    const size_t bh = blockIdx.y;
    const T* kh = k + bh * (size_t)Tn * D;
    for (int e = threadIdx.x; e < nkeys * D; e += kThreads) {
        const int s = e / D, c = e % D;
        kT[c * nkeys + s] = to_f32(kh[(size_t)s * D + c]);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qw = qs + warp * D;
    const int r0 = blockIdx.x * kRowsPerCta;
    for (int r = r0 + warp; r < r0 + kRowsPerCta && r < Tn; r += kThreads / 32) {
        const size_t row = bh * (size_t)Tn + r;
        for (int c = lane; c < D; c += 32) qw[c] = to_f32(q[row * D + c]);
        __syncwarp();
        const float l = lse[row];
        float acc = 0.f;
        for (int s = lane; s < nkeys && s <= r; s += 32) {
            float x = 0.f;
            for (int c = 0; c < D; ++c) x = fmaf(qw[c], kT[c * nkeys + s], x);
            acc += expf(scale * x - l);
        }
        acc = warp_sum(acc);
        if (lane == 0) sink[row] = acc;
        __syncwarp();
    }
}

__global__ void __launch_bounds__(kThreads)
diag_head_kernel(const float* __restrict__ delta, const float* __restrict__ sink, int Tn,
                 float* __restrict__ stats) {
    __shared__ double part[2][kThreads / 32];
    const size_t base = (size_t)blockIdx.x * Tn;
    double a = 0.0, b = 0.0;
    for (int t = threadIdx.x; t < Tn; t += kThreads) {
        a += (double)delta[base + t];
        b += (double)sink[base + t];
    }
    a = warp_sum(a);
    b = warp_sum(b);
    if ((threadIdx.x & 31) == 0) {
        part[0][threadIdx.x >> 5] = a;
        part[1][threadIdx.x >> 5] = b;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double sa = 0.0, sb = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) {
            sa += part[0][w];
            sb += part[1][w];
        }
        stats[2 * blockIdx.x] = (float)(sa / Tn);
        stats[2 * blockIdx.x + 1] = (float)(sb / Tn);
    }
}

}  // namespace

int launch_diagnostics(const ssa_params_t& p, const void* q, const void* k, const float* lse_full,
                       const float* delta, float* sink, float* stats, cudaStream_t s) {
    const int BH = p.B * p.H;
    const int nkeys = p.block < p.T ? p.block : p.T;
    const size_t smem = ((size_t)p.D * nkeys + (kThreads / 32) * (size_t)p.D) * sizeof(float);
    const dim3 grid((unsigned)((p.T + kRowsPerCta - 1) / kRowsPerCta), (unsigned)BH);
    cudaError_t e;
    if (p.dtype == SSA_BF16) {
        e = cudaFuncSetAttribute(diag_sink_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            diag_sink_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
                static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                lse_full, p.T, p.D, nkeys, p.sm_scale, sink);
    } else {
        e = cudaFuncSetAttribute(diag_sink_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e == cudaSuccess)
            diag_sink_kernel<float><<<grid, kThreads, smem, s>>>(
                static_cast<const float*>(q), static_cast<const float*>(k), lse_full, p.T, p.D,
                nkeys, p.sm_scale, sink);
    }
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "diag: smem attribute: %s", cudaGetErrorString(e));
    int st = check_launch("diag_sink_kernel");
    if (st != SSA_OK) return st;
    diag_head_kernel<<<BH, kThreads, 0, s>>>(delta, sink, p.T, stats);
    return check_launch("diag_head_kernel");
}

}  // namespace ssa

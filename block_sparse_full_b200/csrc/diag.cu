// Attention diagnostics ("Sintesi Tecnica: SSA", section 1: the sparse
// stream's error grows with the discarded attention mass delta(t); the pages
// also discuss the first block as an attention sink and the sparsity of
// learned attention):
//   sink(t)       = sum_{s <= t, s < block} exp(sigma q_t . k_s - lse_full(t)),
//                   the full-softmax mass on block 0;
//   mean_delta[h] = mean over t of delta(t),  mean_sink[h] = mean over t of sink(t).
// Two launches: diag_sink_kernel (CUDA cores; block 0 of K staged transposed
// once per CTA, 64-row slabs of Q staged row-major, each warp register-tiles 8
// rows x its lane's 2 or 4 keys) and diag_head_kernel (one CTA per head, fixed-order
// float64 sums: bitwise repeatable).  The first pass reads Q once.
#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerCta = 64;

template <typename T, int KPL>  // KPL = keys of block 0 per lane (2 for block 64, 4 for 128)
__global__ void __launch_bounds__(kThreads)
diag_sink_kernel(const T* __restrict__ q, const T* __restrict__ k, const float* __restrict__ lse,
                 int Tn, int D, int nkeys, float scale, int slabs, float* __restrict__ sink) {
    extern __shared__ float sm[];
    constexpr int NK = 32 * KPL;                 // key slots (keys past nkeys are masked)
    constexpr int RW = kRowsPerCta / (kThreads / 32);  // rows per warp (8)
    const int QS = D + 4;                        // row stride of the Q slab (16-byte aligned)
    float* kT = sm;                              // [D][NK]: lane reads its KPL keys at once
    float* qs = sm + (size_t)D * NK;             // [kRowsPerCta][D + 4], row-major
    const size_t bh = blockIdx.y;
    const T* kh = k + bh * (size_t)Tn * D;
    // block 0 of K, transposed once per CTA (consecutive threads on consecutive shared
    // words; the strided global reads hit the same lines repeatedly in L1)
    for (int e = threadIdx.x; e < NK * D; e += kThreads) {
        const int s = e % NK, c = e / NK;
        kT[c * NK + s] = s < nkeys ? to_f32(kh[(size_t)s * D + c]) : 0.f;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int slab = 0; slab < slabs; ++slab) {
        const int r0 = (blockIdx.x * slabs + slab) * kRowsPerCta;
        if (r0 >= Tn) break;  // CTA-uniform
        __syncthreads();  // previous slab's reads of qs are done (and kT is staged)
        for (int e = threadIdx.x; e < kRowsPerCta * D; e += kThreads) {
            const int r = e / D, c = e % D;
            const int t = r0 + r;
            qs[r * QS + c] = t < Tn ? to_f32(q[(bh * (size_t)Tn + t) * D + c]) : 0.f;
        }
        __syncthreads();
        // acc[r][j] = q_(row r of this warp) . k_(key KPL*lane + j)
        float acc[RW][KPL];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int j = 0; j < KPL; ++j) acc[r][j] = 0.f;
        const float* qw = qs + (RW * warp) * QS;
        for (int c = 0; c < D; c += 4) {
            float kv[4][KPL];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if constexpr (KPL == 2) {
                    const float2 x = *reinterpret_cast<const float2*>(kT + (c + u) * NK + 2 * lane);
                    kv[u][0] = x.x;
                    kv[u][1] = x.y;
                } else {
                    const float4 x = *reinterpret_cast<const float4*>(kT + (c + u) * NK + 4 * lane);
                    kv[u][0] = x.x;
                    kv[u][1] = x.y;
                    kv[u][2] = x.z;
                    kv[u][3] = x.w;
                }
            }
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const float4 q4 = *reinterpret_cast<const float4*>(qw + r * QS + c);  // broadcast
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int j = 0; j < KPL; ++j) acc[r][j] = fmaf(qv[u], kv[u][j], acc[r][j]);
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int t = r0 + RW * warp + r;
            if (t >= Tn) break;  // warp-uniform
            const size_t row = bh * (size_t)Tn + t;
            const float l = lse[row];
            float m = 0.f;
#pragma unroll
            for (int j = 0; j < KPL; ++j) {
                const int s = KPL * lane + j;
                if (s < nkeys && s <= t) m += expf(scale * acc[r][j] - l);
            }
            m = warp_sum(m);
            if (lane == 0) sink[row] = m;
        }
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
    const int kpl = p.block > 64 ? 4 : 2;
    const size_t smem = ((size_t)p.D * 32 * kpl + (size_t)(p.D + 4) * kRowsPerCta) * sizeof(float);
    // enough CTAs to cover the SMs a few times; each loops over 64-row slabs
    // with block 0 of K staged once
    const int nslab = (p.T + kRowsPerCta - 1) / kRowsPerCta;
    int per_head = (4 * 148 + BH - 1) / BH;
    if (per_head > nslab) per_head = nslab;
    const int slabs = (nslab + per_head - 1) / per_head;
    const dim3 grid((unsigned)((nslab + slabs - 1) / slabs), (unsigned)BH);
    auto go = [&](auto kernel, auto qp, auto kp) -> int {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "diag: smem attribute: %s", cudaGetErrorString(e));
        kernel<<<grid, kThreads, smem, s>>>(qp, kp, lse_full, p.T, p.D, nkeys, p.sm_scale, slabs, sink);
        return check_launch("diag_sink_kernel");
    };
    int st;
    if (p.dtype == SSA_BF16) {
        auto qp = static_cast<const __nv_bfloat16*>(q);
        auto kp = static_cast<const __nv_bfloat16*>(k);
        st = kpl == 4 ? go(diag_sink_kernel<__nv_bfloat16, 4>, qp, kp)
                      : go(diag_sink_kernel<__nv_bfloat16, 2>, qp, kp);
    } else {
        auto qp = static_cast<const float*>(q);
        auto kp = static_cast<const float*>(k);
        st = kpl == 4 ? go(diag_sink_kernel<float, 4>, qp, kp) : go(diag_sink_kernel<float, 2>, qp, kp);
    }
    if (st != SSA_OK) return st;
    return launch_diag_heads(p, delta, sink, stats, s);
}

int launch_diag_heads(const ssa_params_t& p, const float* delta, const float* sink, float* stats,
                      cudaStream_t s) {
    diag_head_kernel<<<p.B * p.H, kThreads, 0, s>>>(delta, sink, p.T, stats);
    return check_launch("diag_head_kernel");
}

}  // namespace ssa

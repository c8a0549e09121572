// Dual-stream forward on CUDA cores (float32 arithmetic): the exact-fp32
// path for float32 inputs (where tf32 tensor cores would miss a 1e-4
// tolerance) and the comparator behind SSA_FLAG_FORCE_SIMT.
//
// One CTA = 16 query rows of one (b, h), a warp per row (a row's logit,
// softmax and P V chains are serial, so many warps with one row each overlap
// them, and small problems still give the GPU many CTAs).  K/V stream
// through shared memory in chunks of 32 keys; lane j owns key j of the chunk
// for the logits and dimension lane + 32u of the accumulators.  A chunk lies
// inside one key block and the CTA's rows inside one query block, so the
// selection test (sparse stream or not) is one mask bit per chunk.  The next
// chunk's loads are in flight while a chunk is computed.  Online
// softmax with one running max shared by both streams:
//   l_sel, l_uns  running sums over selected / unselected keys,
//   O_sel, O_uns  running weighted sums of v,
// and at the end h_full = (O_sel + O_uns) / (l_sel + l_uns),
// h_sparse = O_sel / l_sel, delta = l_uns / (l_sel + l_uns)
// ("Sintesi Tecnica: SSA", sections 1-2).
#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kRows = 16;  // query rows per CTA
constexpr int kKeys = 32;  // keys per chunk
constexpr int kThreads = 512;  // 16 warps of 1 row: the rows' dependency chains overlap
constexpr int kRowsPerWarp = kRows / (kThreads / 32);

template <int D>
struct FwdSmem {
    float q[kRows][D];
    float k[kKeys][D + 4];  // +4: lane j reads row j 16 bytes at a time, conflict-free
    float v[kKeys][D];
    uint32_t mrow[256];     // mask words of this CTA's query block
};

// a + x[0] y[0] + x[1] y[1] + ... + x[D-1] y[D-1], one fused multiply-add per
// column in column order (the rounding of a plain loop), four columns per
// shared-memory load; x and y are 16-byte aligned.
template <int D>
__device__ __forceinline__ float dot_seq(const float* x, const float* y, float a) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* y4 = reinterpret_cast<const float4*>(y);
#pragma unroll 4
    for (int c = 0; c < D / 4; ++c) {
        const float4 p = x4[c], q = y4[c];
        a = fmaf(p.x, q.x, a);
        a = fmaf(p.y, q.y, a);
        a = fmaf(p.z, q.z, a);
        a = fmaf(p.w, q.w, a);
    }
    return a;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const uint32_t* __restrict__ mask, int BH, int T_, int block, int words,
                float sm_scale, T* __restrict__ h_full, T* __restrict__ h_sparse,
                float* __restrict__ delta, float* __restrict__ lse_full,
                float* __restrict__ lse_sparse, float* __restrict__ sqdiff) {
    constexpr int DPL = D / 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(smem_raw);

    const int ntiles = T_ / kRows;
    const int L = blockIdx.x;
    const int tile = ntiles - 1 - L / BH;  // longest rows first
    const size_t bh = L % BH;
    const int t0 = tile * kRows;
    const int qblk = t0 / block;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t base = bh * (size_t)T_ * D;

    for (int e = tid; e < kRows * D; e += kThreads)
        sm.q[e / D][e % D] = to_f32(q[base + (size_t)t0 * D + e]);
    const uint32_t* mrow = mask + (bh * (T_ / block) + qblk) * (size_t)words;
    for (int w = tid; w < words; w += kThreads) sm.mrow[w] = mrow[w];

    float m[kRowsPerWarp], lsel[kRowsPerWarp], luns[kRowsPerWarp];
    float osel[kRowsPerWarp][DPL], ouns[kRowsPerWarp][DPL];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        m[r] = -INFINITY;
        lsel[r] = 0.f;
        luns[r] = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) osel[r][u] = ouns[r][u] = 0.f;
    }

    // chunk c + 1's keys and values are loaded into registers while chunk c
    // is computed, and stored to shared memory after it
    constexpr int NE = kKeys * D / kThreads;  // elements per thread per chunk and operand
    static_assert(NE * kThreads == kKeys * D, "whole chunks per CTA");
    T kn[NE], vn[NE];
    auto fetch = [&](int s0) {
#pragma unroll
        for (int x = 0; x < NE; ++x) {
            const size_t g = base + (size_t)s0 * D + tid + x * kThreads;
            kn[x] = k[g];
            vn[x] = v[g];
        }
    };
    const int send = t0 + kRows;  // chunks [s0, s0 + 32) with s0 < send end at or before T
    fetch(0);
    for (int s0 = 0; s0 < send; s0 += kKeys) {
        __syncthreads();
#pragma unroll
        for (int x = 0; x < NE; ++x) {
            const int e = tid + x * kThreads;
            sm.k[e / D][e % D] = to_f32(kn[x]);
            sm.v[e / D][e % D] = to_f32(vn[x]);
        }
        __syncthreads();
        if (s0 + kKeys < send) fetch(s0 + kKeys);
        const bool chunk_sel = mask_bit(sm.mrow, s0 / block);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int rr = warp * kRowsPerWarp + r;
            const int t = t0 + rr;
            float x = dot_seq<D>(sm.q[rr], sm.k[lane], 0.f);
            const bool valid = s0 + lane <= t;
            x = valid ? x * sm_scale : -INFINITY;
            const float mnew = fmaxf(m[r], warp_max(x));  // key s0 <= t always valid
            const float alpha = expf(m[r] - mnew);
            const float p = valid ? expf(x - mnew) : 0.f;
            const float psum = warp_sum(p);
            m[r] = mnew;
            lsel[r] *= alpha;
            luns[r] *= alpha;
#pragma unroll
            for (int u = 0; u < DPL; ++u) {
                osel[r][u] *= alpha;
                ouns[r][u] *= alpha;
            }
            if (chunk_sel) {
                lsel[r] += psum;
#pragma unroll 8
                for (int j = 0; j < kKeys; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
                    for (int u = 0; u < DPL; ++u) osel[r][u] = fmaf(pj, sm.v[j][lane + 32 * u], osel[r][u]);
                }
            } else {
                luns[r] += psum;
#pragma unroll 8
                for (int j = 0; j < kKeys; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
                    for (int u = 0; u < DPL; ++u) ouns[r][u] = fmaf(pj, sm.v[j][lane + 32 * u], ouns[r][u]);
                }
            }
        }
    }

#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int t = t0 + warp * kRowsPerWarp + r;
        const size_t row = bh * (size_t)T_ + t;
        const float l = lsel[r] + luns[r];
        const float inv_l = 1.f / l;
        const float inv_ls = lsel[r] > 0.f ? 1.f / lsel[r] : 0.f;
        float sq = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            const float hf = (osel[r][u] + ouns[r][u]) * inv_l;
            const float hs = osel[r][u] * inv_ls;
            const float df = hf - hs;
            sq = fmaf(df, df, sq);
            h_full[row * D + lane + 32 * u] = from_f32<T>(hf);
            h_sparse[row * D + lane + 32 * u] = from_f32<T>(hs);
        }
        sq = warp_sum(sq);
        if (lane == 0) {
            delta[row] = luns[r] * inv_l;
            lse_full[row] = m[r] + logf(l);
            lse_sparse[row] = lsel[r] > 0.f ? m[r] + logf(lsel[r]) : -INFINITY;
            sqdiff[row] = sq;
        }
    }
}

template <typename T, int D>
int launch_typed(const ssa_params_t& p, const void* q, const void* k, const void* v,
                 const uint32_t* mask, void* hf, void* hs, float* delta, float* lf, float* ls,
                 float* sq, cudaStream_t s) {
    const size_t smem = sizeof(FwdSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "fwd_simt: smem attribute: %s", cudaGetErrorString(e));
    const int BH = p.B * p.H;
    const size_t grid = (size_t)BH * (p.T / kRows);
    fwd_simt_kernel<T, D><<<(unsigned)grid, kThreads, smem, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), mask, BH,
        p.T, p.block, mask_words(p), p.sm_scale, static_cast<T*>(hf), static_cast<T*>(hs), delta,
        lf, ls, sq);
    return check_launch("fwd_simt_kernel");
}

}  // namespace

int launch_fwd_simt(const ssa_params_t& p, const void* q, const void* k, const void* v,
                    const uint32_t* mask, void* hf, void* hs, float* delta, float* lf, float* ls,
                    float* sq, cudaStream_t s) {
    if (mask_words(p) > 256) return fail(SSA_ERR_UNSUPPORTED, "fwd_simt: more than 8192 blocks");
    if ((size_t)p.B * p.H * (p.T / kRows) > 0x7fffffffull)
        return fail(SSA_ERR_UNSUPPORTED, "fwd_simt: grid too large");
    const bool bf = p.dtype == SSA_BF16;
    if (p.D == 64)
        return bf ? launch_typed<__nv_bfloat16, 64>(p, q, k, v, mask, hf, hs, delta, lf, ls, sq, s)
                  : launch_typed<float, 64>(p, q, k, v, mask, hf, hs, delta, lf, ls, sq, s);
    return bf ? launch_typed<__nv_bfloat16, 128>(p, q, k, v, mask, hf, hs, delta, lf, ls, sq, s)
              : launch_typed<float, 128>(p, q, k, v, mask, hf, hs, delta, lf, ls, sq, s);
}

}  // namespace ssa

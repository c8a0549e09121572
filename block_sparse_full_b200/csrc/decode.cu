// One generation step of the sparse stream over a key/value cache ("Sintesi
// Tecnica: SSA", section 4, "Efficienza": at inference SSA runs the same
// operations as MoBA).  The pages do not describe decoding itself; the
// reading here is MoBA's inference rule: the current query q_t is scored
// against the pooled keys Kbar_j of the completed blocks j < i = t / block
// (float64, like the training-time scores), the current block i is always
// attended (keys 0..t of it) and counts inside the budget k, block 0 is
// forced only with SSA_FLAG_FORCE_SINK, the remaining places go to the best
// scores (ties to the lower index), and the step attends over every key of
// the selected blocks up to t.
//
// Launches (CUDA cores: one query per head is matrix-vector work, bound by
// the key/value bytes it reads and by latency):
//   decode_pool_kernel     Kbar_j = mean of block j's keys (float64, exact)
//   decode_select_kernel   CTA per (32 completed blocks, head): scores (warp
//                          per block, lanes over d) to the workspace; the
//                          head's last CTA to finish (a counter in the
//                          workspace) fills the free slots by warp-argmax
//                          rounds and writes the ascending list
//   decode_attend_kernel   CTA per (head, selected block): scores with a
//                          warp per group of keys (lanes over d), softmax
//                          statistics CTA-wide, then P V with threads over
//                          (d, key group); the head's last CTA to finish
//                          merges the per-block partials into h and lse
// The counters are cleared before each step (one memset) and by the CTA that
// consumes them.
#include <type_traits>

#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxTopk = 64;

template <typename T>
__global__ void __launch_bounds__(kThreads)
decode_pool_kernel(const T* __restrict__ k, int Tcap, int D, int block, int j0,
                   double* __restrict__ kbar, int nb) {
    const int j = j0 + blockIdx.x;
    const size_t bh = blockIdx.y;
    const T* src = k + (bh * Tcap + (size_t)j * block) * D;
    for (int c = threadIdx.x; c < D; c += kThreads) {
        double acc = 0.0;
        for (int r = 0; r < block; ++r) acc += (double)to_f32(src[(size_t)r * D + c]);
        kbar[(bh * nb + j) * D + c] = acc / (double)block;  // block is a power of two: exact
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_select_kernel(const T* __restrict__ q, const double* __restrict__ kbar, int nb, int i,
                     int topk, bool force_sink, double* __restrict__ score_g,
                     unsigned int* __restrict__ counter, int32_t* __restrict__ sel,
                     int32_t* __restrict__ idx_out) {
    constexpr int M = D / 32;  // query columns per lane
    constexpr int U = 4;       // key blocks in flight per warp
    constexpr int CHUNK = (kThreads / 32) * U;  // completed blocks per CTA
    extern __shared__ double score[];  // [max(i, 1)], then the set bitmask [i / 32 + 1]
    __shared__ int is_last;
    uint32_t* bits = reinterpret_cast<uint32_t*>(score + (i > 0 ? i : 1));
    const size_t bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int words = (i >> 5) + 1;  // bits 0 .. i
    double* sg = score_g + bh * (size_t)nb;
    // scores of this CTA's completed blocks: warp per block, lane l owns columns
    // l, l + 32, ... (coalesced rows of the float64 pooled keys), U blocks' loads
    // in flight per warp, fixed butterfly sum
    {
        double qr[M];
#pragma unroll
        for (int m = 0; m < M; ++m) qr[m] = (double)to_f32(q[bh * D + lane + 32 * m]);
        const double* kb = kbar + bh * (size_t)nb * D;
        const int j0 = CHUNK * blockIdx.x + U * warp;
        if (j0 < i) {
            double a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const double* kr = kb + (size_t)min(j0 + u, i - 1) * D + lane;  // past the end: unused
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
                    if (j0 + u < i) sg[j0 + u] = a[u];
            }
        }
    }
    // the head's last CTA to finish takes the selection
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&counter[bh], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int j = threadIdx.x; j < i; j += kThreads) score[j] = __ldcg(sg + j);
    for (int w = threadIdx.x; w < words; w += kThreads) bits[w] = 0u;
    if (threadIdx.x == 0) counter[bh] = 0u;  // ready for the next step
    __syncthreads();
    if (warp != 0) return;
    // one warp: forced blocks, the free slots by warp-argmax rounds, then the
    // ascending index list (-1 padded) from the bitmask by popcount prefix
    const bool sink = force_sink && i > 0;
    const int want = topk < i + 1 ? topk : i + 1;  // fewer candidates than places: take all
    const int first = sink ? 1 : 0;                // candidates are first .. i-1
    const int r = want - (sink ? 2 : 1);           // free slots (>= 0: a sink needs topk >= 2)
    if (lane == 0) {
        bits[i >> 5] |= 1u << (i & 31);
        if (sink) bits[0] |= 1u;
    }
    __syncwarp();
    if (i - first <= r) {
        for (int j = first + lane; j < i; j += 32) atomicOr(&bits[j >> 5], 1u << (j & 31));
    } else {
        warp_topk_rounds(score, first, i, r, bits, lane);
    }
    __syncwarp();
    int32_t* srow = sel + bh * topk;
    int32_t* irow = idx_out ? idx_out + bh * topk : nullptr;
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        const uint32_t wv = w < words ? bits[w] : 0u;
        const int c = __popc(wv);
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        int pos = base + incl - c;
        for (uint32_t b = wv; b != 0u; b &= b - 1u, ++pos) {
            if (pos < topk) {  // NaN scores: stay in bounds
                const int v = w * 32 + __ffs(b) - 1;
                srow[pos] = v;
                if (irow) irow[pos] = v;
            }
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int p = base + lane; p < topk; p += 32) {
        srow[p] = -1;
        if (irow) irow[p] = -1;
    }
}

// E consecutive elements of a row, as float, in one vector load (E * sizeof(T)
// is 4, 8 or 16 bytes and the address a multiple of it)
template <typename T, int E>
__device__ __forceinline__ void load_row_piece(const T* p, float (&x)[E]) {
    constexpr int B = E * (int)sizeof(T);
    if constexpr (B == 16) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int z = 0; z < E; ++z) x[z] = to_f32(e[z]);
    } else if constexpr (B == 8) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int z = 0; z < E; ++z) x[z] = to_f32(e[z]);
    } else {
        static_assert(B == 4, "row piece of 4, 8 or 16 bytes");
        const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int z = 0; z < E; ++z) x[z] = to_f32(e[z]);
    }
}

// partial of one (head, selected block): m (max of x), l (sum e^{x-m}), o[D]
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_attend_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ sel, int Tcap, int block, int t, int topk,
                     float scale, float* __restrict__ part, unsigned int* __restrict__ counter,
                     T* __restrict__ h, float* __restrict__ lse) {
    constexpr int E = D / 32;            // columns per lane
    constexpr int NW = kThreads / 32;    // warps
    constexpr int KPW = 128 / NW;        // keys per warp (block <= 128)
    __shared__ float ps[128];            // scores, then e^{x - m}
    __shared__ float red[NW];
    __shared__ float og[kThreads];       // [key group][d] partial sums of P V
    const int slot = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* out = part + (bh * topk + slot) * (2 + D);
    const int j = sel[bh * topk + slot];
    const int s0 = j < 0 ? 0 : j * block;
    const int nks = j < 0 ? 0 : min((j + 1) * block, t + 1) - s0;  // keys of this block <= t
    // scores: warp w takes keys w, w + NW, ...; lane l reads columns
    // [E l, E l + E) of each key row (coalesced), all the warp's rows in flight
    float qv[E];
    load_row_piece<T, E>(q + bh * D + E * lane, qv);
    float acc[KPW];
#pragma unroll
    for (int kk = 0; kk < KPW; ++kk) {
        const int s = warp + NW * kk;
        acc[kk] = 0.f;
        if (s < nks) {
            float x[E];
            load_row_piece<T, E>(k + (bh * Tcap + s0 + s) * D + E * lane, x);
#pragma unroll
            for (int z = 0; z < E; ++z) acc[kk] = fmaf(qv[z], x[z], acc[kk]);
        }
    }
#pragma unroll
    for (int kk = 0; kk < KPW; ++kk) {
        const int s = warp + NW * kk;
        const float dot = warp_sum(acc[kk]);
        if (lane == 0 && s < nks) ps[s] = dot * scale;
    }
    __syncthreads();
    // m = max over the block's keys, then p = e^{x - m} and l = sum p
    const float x = threadIdx.x < nks ? ps[threadIdx.x] : -INFINITY;
    float mx = warp_max(x);
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float m = red[0];
    for (int w = 1; w < NW; ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    float p = 0.f;
    if (threadIdx.x < nks) {
        p = expf(x - m);
        ps[threadIdx.x] = p;
    }
    const float ls = warp_sum(p);
    if (lane == 0) red[warp] = ls;
    __syncthreads();
    float l = 0.f;
    for (int w = 0; w < NW; ++w) l += red[w];
    // o[d] = sum_s p_s v_s[d]: thread (g, d) over keys s = g, g + G, ... (coalesced in d)
    const int G = kThreads / D;
    const int d = threadIdx.x % D, g = threadIdx.x / D;
    // the value loads are independent: unrolled so that many are in flight
    const T* vcol = v + (bh * Tcap + s0) * D + d;
    float a4[4] = {0.f, 0.f, 0.f, 0.f};
    int s = g;
#pragma unroll 4
    for (; s + 3 * G < nks; s += 4 * G) {
        const float x0 = to_f32(vcol[(size_t)s * D]), x1 = to_f32(vcol[(size_t)(s + G) * D]);
        const float x2 = to_f32(vcol[(size_t)(s + 2 * G) * D]), x3 = to_f32(vcol[(size_t)(s + 3 * G) * D]);
        a4[0] = fmaf(ps[s], x0, a4[0]);
        a4[1] = fmaf(ps[s + G], x1, a4[1]);
        a4[2] = fmaf(ps[s + 2 * G], x2, a4[2]);
        a4[3] = fmaf(ps[s + 3 * G], x3, a4[3]);
    }
    for (; s < nks; s += G) a4[0] = fmaf(ps[s], to_f32(vcol[(size_t)s * D]), a4[0]);
    og[g * D + d] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    __syncthreads();
    if (threadIdx.x < D) {
        float o = 0.f;
        for (int gg = 0; gg < G; ++gg) o += og[gg * D + threadIdx.x];
        out[2 + threadIdx.x] = o;
    }
    if (threadIdx.x == 0) {
        out[0] = nks > 0 ? m : -INFINITY;
        out[1] = l;
    }
    // the head's last CTA to finish merges the partials: weights e^{m_a - M}
    __shared__ int is_last;
    __shared__ float wgt[kMaxTopk];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&counter[bh], 1u) == (unsigned)topk - 1u;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const float* pp = part + bh * topk * (2 + D);
    if (warp == 0) {
        float Mx = -INFINITY;
        for (int a = lane; a < topk; a += 32) Mx = fmaxf(Mx, __ldcg(pp + a * (2 + D)));
        Mx = warp_max(Mx);
        float L = 0.f;
        for (int a = lane; a < topk; a += 32) {
            const float ma = __ldcg(pp + a * (2 + D));
            const float w = ma > -INFINITY ? expf(ma - Mx) : 0.f;
            wgt[a] = w;
            L += w * __ldcg(pp + a * (2 + D) + 1);
        }
        L = warp_sum(L);
        if (lane == 0) {
            red[0] = L;
            lse[bh] = Mx + logf(L);
            counter[bh] = 0u;  // ready for the next step
        }
    }
    __syncthreads();
    const float inv_L = 1.f / red[0];
    for (int c = threadIdx.x; c < D; c += kThreads) {
        float acc = 0.f;
        for (int a = 0; a < topk; ++a) acc = fmaf(wgt[a], __ldcg(pp + a * (2 + D) + 2 + c), acc);
        h[bh * D + c] = from_f32<T>(acc * inv_L);
    }
}

}  // namespace

// selected indices [BH, topk] i32 | partials [BH, topk, 2 + D] f32 | scores
// [BH, n] f64 | two counters per head
size_t decode_workspace(const ssa_params_t& p) {
    const size_t bh = (size_t)p.B * p.H;
    return align_up(bh * p.topk * 4, 256) + align_up(bh * p.topk * (2 + p.D) * 4, 256) +
           align_up(bh * (size_t)num_blocks(p) * 8, 256) + align_up(bh * 2 * 4, 256);
}

int launch_decode_pool(const ssa_params_t& p, int j0, int j1, const void* k, double* kbar,
                       cudaStream_t s) {
    if (j1 <= j0) return SSA_OK;
    const dim3 grid((unsigned)(j1 - j0), (unsigned)(p.B * p.H));
    const int nb = num_blocks(p);
    if (p.dtype == SSA_BF16)
        decode_pool_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(k), p.T, p.D, p.block, j0, kbar, nb);
    else
        decode_pool_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(k), p.T, p.D,
                                                            p.block, j0, kbar, nb);
    return check_launch("decode_pool_kernel");
}

int launch_decode_step(const ssa_params_t& p, int t, const void* q, const void* k, const void* v,
                       const double* kbar, void* h, float* lse, int32_t* idx, void* ws,
                       cudaStream_t s) {
    const int BH = p.B * p.H;
    const int i = t / p.block;
    char* w = static_cast<char*>(ws);
    int32_t* sel = reinterpret_cast<int32_t*>(w);
    w += align_up((size_t)BH * p.topk * 4, 256);
    float* part = reinterpret_cast<float*>(w);
    w += align_up((size_t)BH * p.topk * (2 + p.D) * 4, 256);
    double* score_g = reinterpret_cast<double*>(w);
    w += align_up((size_t)BH * num_blocks(p) * 8, 256);
    unsigned int* counters = reinterpret_cast<unsigned int*>(w);  // [2][BH]
    cudaError_t me = cudaMemsetAsync(counters, 0, (size_t)BH * 2 * 4, s);
    if (me != cudaSuccess) return fail(SSA_ERR_CUDA, "decode: counters: %s", cudaGetErrorString(me));
    const size_t smem = (size_t)(i > 0 ? i : 1) * sizeof(double) + (size_t)((i >> 5) + 1) * 4;
    const bool sink = (p.flags & SSA_FLAG_FORCE_SINK) != 0;
    const int nb = num_blocks(p);
    auto run = [&](auto tag, auto dtag) -> int {
        using T = decltype(tag);
        constexpr int D = decltype(dtag)::value;
        auto sk = decode_select_kernel<T, D>;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "decode: smem attribute: %s", cudaGetErrorString(e));
        }
        constexpr int kChunk = (kThreads / 32) * 4;  // completed blocks per select CTA
        const unsigned chunks = (unsigned)(i > 0 ? (i + kChunk - 1) / kChunk : 1);
        sk<<<dim3(chunks, (unsigned)BH), kThreads, smem, s>>>(
            static_cast<const T*>(q), kbar, nb, i, p.topk, sink, score_g, counters, sel, idx);
        int st = check_launch("decode_select_kernel");
        if (st != SSA_OK) return st;
        decode_attend_kernel<T, D><<<dim3((unsigned)p.topk, (unsigned)BH), kThreads, 0, s>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), sel, p.T,
            p.block, t, p.topk, p.sm_scale, part, counters + BH, static_cast<T*>(h), lse);
        return check_launch("decode_attend_kernel");
    };
    using D64 = std::integral_constant<int, 64>;
    using D128 = std::integral_constant<int, 128>;
    if (p.dtype == SSA_BF16)
        return p.D == 64 ? run(__nv_bfloat16{}, D64{}) : run(__nv_bfloat16{}, D128{});
    return p.D == 64 ? run(float{}, D64{}) : run(float{}, D128{});
}

}  // namespace ssa

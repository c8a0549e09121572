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
// the key/value bytes it reads):
//   decode_pool_kernel     Kbar_j = mean of block j's keys (float64, exact)
//   decode_select_kernel   one CTA per head: scores (thread per block),
//                          top-k by rounds of a CTA-wide argmax
//   decode_attend_kernel   one CTA per (head, selected block): scores with a
//                          thread per key, softmax statistics CTA-wide, then
//                          P V with threads over (d, key group)
//   decode_combine_kernel  one warp per head merges the per-block partials
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

template <typename T>
__global__ void __launch_bounds__(kThreads)
decode_select_kernel(const T* __restrict__ q, const double* __restrict__ kbar, int nb, int D,
                     int i, int topk, bool force_sink, int32_t* __restrict__ sel,
                     int32_t* __restrict__ idx_out) {
    extern __shared__ double score[];  // [i]
    __shared__ double best_s[kThreads / 32];
    __shared__ int best_j[kThreads / 32];
    __shared__ int chosen[kMaxTopk];
    const size_t bh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* qh = q + bh * D;
    // scores of the completed blocks: thread per block, independent loads of its
    // float64 pooled key (one memory latency for the whole scan)
    for (int j = threadIdx.x; j < i; j += kThreads) {
        const double2* kb = reinterpret_cast<const double2*>(kbar + (bh * nb + j) * D);
        double acc = 0.0;
#pragma unroll 8
        for (int c = 0; c < D / 2; ++c) {
            const double2 x = kb[c];
            acc += (double)to_f32(qh[2 * c]) * x.x + (double)to_f32(qh[2 * c + 1]) * x.y;
        }
        score[j] = acc;
    }
    __syncthreads();
    int n = 0;
    if (threadIdx.x == 0) {
        chosen[n++] = i;
        if (force_sink && i > 0) {
            chosen[n++] = 0;
            score[0] = -INFINITY;  // taken
        }
    }
    __syncthreads();
    n = (force_sink && i > 0) ? 2 : 1;
    const int want = topk < i + 1 ? topk : i + 1;  // fewer candidates than places: take all
    for (; n < want; ++n) {
        // CTA-wide argmax by (score desc, index asc); taken blocks hold -inf
        double bs = -INFINITY;
        int bj = 1 << 30;
        for (int j = threadIdx.x; j < i; j += kThreads) {
            const double v = score[j];
            if (v > bs || (v == bs && j < bj)) {
                bs = v;
                bj = j;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double os = __shfl_xor_sync(0xffffffffu, bs, o);
            const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            if (os > bs || (os == bs && oj < bj)) {
                bs = os;
                bj = oj;
            }
        }
        if (lane == 0) {
            best_s[warp] = bs;
            best_j[warp] = bj;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double s = best_s[0];
            int jb = best_j[0];
            for (int w = 1; w < kThreads / 32; ++w)
                if (best_s[w] > s || (best_s[w] == s && best_j[w] < jb)) {
                    s = best_s[w];
                    jb = best_j[w];
                }
            chosen[n] = jb;
            score[jb] = -INFINITY;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {  // ascending, -1 padded
        for (int a = 1; a < want; ++a)
            for (int b = a; b > 0 && chosen[b - 1] > chosen[b]; --b) {
                const int x = chosen[b];
                chosen[b] = chosen[b - 1];
                chosen[b - 1] = x;
            }
        for (int a = 0; a < topk; ++a) {
            const int v = a < want ? chosen[a] : -1;
            sel[bh * topk + a] = v;
            if (idx_out) idx_out[bh * topk + a] = v;
        }
    }
}

// partial of one (head, selected block): m (max of x), l (sum e^{x-m}), o[D]
template <typename T>
__global__ void __launch_bounds__(kThreads)
decode_attend_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const int32_t* __restrict__ sel, int Tcap, int D, int block, int t, int topk,
                     float scale, float* __restrict__ part) {
    __shared__ float qs[128];
    __shared__ float ps[128];             // scores, then e^{x - m}
    __shared__ float red[kThreads / 32];
    __shared__ float og[kThreads];        // [key group][d] partial sums of P V
    const int slot = blockIdx.x;
    const size_t bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* out = part + (bh * topk + slot) * (2 + D);
    const int j = sel[bh * topk + slot];
    const int s0 = j < 0 ? 0 : j * block;
    const int nks = j < 0 ? 0 : min((j + 1) * block, t + 1) - s0;  // keys of this block <= t
    for (int c = threadIdx.x; c < D; c += kThreads) qs[c] = to_f32(q[bh * D + c]);
    __syncthreads();
    // scores: thread per key, its row read in 16-byte pieces (independent loads)
    float x = -INFINITY;
    if (threadIdx.x < nks) {
        const uint4* kr = reinterpret_cast<const uint4*>(k + (bh * Tcap + s0 + threadIdx.x) * D);
        constexpr int E = 16 / sizeof(T);  // elements per 16-byte piece
        float acc = 0.f;
        for (int c = 0; c < D / E; ++c) {
            const uint4 u = kr[c];
            const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
            for (int z = 0; z < E; ++z) acc = fmaf(qs[c * E + z], to_f32(e[z]), acc);
        }
        x = acc * scale;
        ps[threadIdx.x] = x;
    }
    // m = max over the block's keys, then p = e^{x - m} and l = sum p
    float mx = warp_max(x);
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float m = red[0];
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
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
    for (int w = 0; w < kThreads / 32; ++w) l += red[w];
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
}

template <typename T>
__global__ void __launch_bounds__(32)
decode_combine_kernel(const float* __restrict__ part, int D, int topk, T* __restrict__ h,
                      float* __restrict__ lse) {
    const size_t bh = blockIdx.x;
    const int lane = threadIdx.x;
    const float* p = part + bh * topk * (2 + D);
    float M = -INFINITY;
    for (int a = 0; a < topk; ++a) M = fmaxf(M, p[a * (2 + D)]);
    float L = 0.f;
    for (int a = 0; a < topk; ++a) {
        const float ma = p[a * (2 + D)];
        if (ma > -INFINITY) L += expf(ma - M) * p[a * (2 + D) + 1];
    }
    for (int c = lane; c < D; c += 32) {
        float acc = 0.f;
        for (int a = 0; a < topk; ++a) {
            const float ma = p[a * (2 + D)];
            if (ma > -INFINITY) acc += expf(ma - M) * p[a * (2 + D) + 2 + c];
        }
        h[bh * D + c] = from_f32<T>(acc / L);
    }
    if (lane == 0) lse[bh] = M + logf(L);
}

}  // namespace

size_t decode_workspace(const ssa_params_t& p) {
    const size_t bh = (size_t)p.B * p.H;
    return align_up(bh * p.topk * 4, 256) + align_up(bh * p.topk * (2 + p.D) * 4, 256);
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
    int32_t* sel = static_cast<int32_t*>(ws);
    float* part = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                           align_up((size_t)BH * p.topk * 4, 256));
    const size_t smem = (size_t)(i > 0 ? i : 1) * sizeof(double);
    const bool sink = (p.flags & SSA_FLAG_FORCE_SINK) != 0;
    const int nb = num_blocks(p);
    auto run = [&](auto tag) -> int {
        using T = decltype(tag);
        auto sk = decode_select_kernel<T>;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "decode: smem attribute: %s", cudaGetErrorString(e));
        }
        sk<<<BH, kThreads, smem, s>>>(static_cast<const T*>(q), kbar, nb, p.D, i, p.topk, sink, sel, idx);
        int st = check_launch("decode_select_kernel");
        if (st != SSA_OK) return st;
        decode_attend_kernel<T><<<dim3((unsigned)p.topk, (unsigned)BH), kThreads, 0, s>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), sel, p.T,
            p.D, p.block, t, p.topk, p.sm_scale, part);
        st = check_launch("decode_attend_kernel");
        if (st != SSA_OK) return st;
        decode_combine_kernel<T><<<BH, 32, 0, s>>>(part, p.D, p.topk, static_cast<T*>(h), lse);
        return check_launch("decode_combine_kernel");
    };
    return p.dtype == SSA_BF16 ? run(__nv_bfloat16{}) : run(float{});
}

}  // namespace ssa

// Backward through both SSA attention streams on CUDA cores (float32
// arithmetic).  Used for float32 inputs and under SSA_FLAG_FORCE_SIMT.
//
// Upstream reaching each output ("Sintesi Tecnica: SSA", section 2: the
// full stream gives gradient to every token; L_sparsity pulls h_full toward
// h_sparse, L_commit pulls h_sparse toward h_full, each with stop-gradient
// on the other stream):
//   G_f = dh_full   + w_s * 2/N * (h_full - h_sparse)
//   G_s = dh_sparse + w_c * 2/N * (h_sparse - h_full)
// For query t, key s <= t, x = sigma q_t.k_s:
//   P_f = exp(x - lse_full(t)),  P_s = exp(x - lse_sparse(t)) on selected s
//   dS  = P_f (G_f(t).v_s - D_f(t)) + [sel] P_s (G_s(t).v_s - D_s(t))
//   with D_f = G_f.h_full and D_s = G_s.h_sparse (row dots),
//   dq_t = sigma sum_s dS k_s,  dk_s = sigma sum_t dS q_t,
//   dv_s = sum_t P_f G_f(t) + [sel] P_s G_s(t).
// Two launches: a row preprocess (G_f, G_s, D_f, D_s into the workspace),
// then one grid whose CTAs take either a query tile (dq) or a key tile
// (dk/dv), the two kinds interleaved; no atomics, so results are bitwise
// repeatable.
#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kRowsB = 16;   // rows per CTA: queries (dq) or keys (dk/dv)
constexpr int kChunk = 32;   // keys (dq) or queries (dk/dv) per streamed chunk: lane j owns chunk row j
constexpr int kThreads = 512;  // a warp per row: the rows' dependency chains overlap
constexpr int kRowsPerWarp = kRowsB / (kThreads / 32);
constexpr int kPreThreads = 128;  // preprocess: a warp per row

struct BwdWs {
    float* gf;
    float* gs;
    float* df;
    float* ds;
};

BwdWs carve(const ssa_params_t& p, void* ws) {
    const size_t big = align_up(num_elems(p) * sizeof(float), 256);
    const size_t small = align_up(num_rows(p) * sizeof(float), 256);
    char* b = static_cast<char*>(ws);
    return {reinterpret_cast<float*>(b), reinterpret_cast<float*>(b + big),
            reinterpret_cast<float*>(b + 2 * big), reinterpret_cast<float*>(b + 2 * big + small)};
}

template <typename T>
__global__ void __launch_bounds__(kPreThreads)
bwd_pre_kernel(const T* __restrict__ hf, const T* __restrict__ hs, const T* __restrict__ dhf,
               const T* __restrict__ dhs, size_t rows, int D, float cf, float cs, BwdWs w) {
    const size_t row = (size_t)blockIdx.x * (kPreThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float sf = 0.f, ss = 0.f;
    for (int c = lane; c < D; c += 32) {
        const size_t e = row * D + c;
        const float f = to_f32(hf[e]), s = to_f32(hs[e]);
        const float gf = (dhf ? to_f32(dhf[e]) : 0.f) + cf * (f - s);
        const float gs = (dhs ? to_f32(dhs[e]) : 0.f) + cs * (s - f);
        w.gf[e] = gf;
        w.gs[e] = gs;
        sf = fmaf(gf, f, sf);
        ss = fmaf(gs, s, ss);
    }
    sf = warp_sum(sf);
    ss = warp_sum(ss);
    if (lane == 0) {
        w.df[row] = sf;
        w.ds[row] = ss;
    }
}

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
// two such sums side by side (independent chains, the same order in each)
template <int D>
__device__ __forceinline__ void dot2_seq(const float* x0, const float* y0, float& a0, const float* x1,
                                         const float* y1, float& a1) {
    const float4 *p4 = reinterpret_cast<const float4*>(x0), *q4 = reinterpret_cast<const float4*>(y0);
    const float4 *r4 = reinterpret_cast<const float4*>(x1), *s4 = reinterpret_cast<const float4*>(y1);
#pragma unroll 4
    for (int c = 0; c < D / 4; ++c) {
        const float4 p = p4[c], q = q4[c], r = r4[c], s = s4[c];
        a0 = fmaf(p.x, q.x, a0);
        a1 = fmaf(r.x, s.x, a1);
        a0 = fmaf(p.y, q.y, a0);
        a1 = fmaf(r.y, s.y, a1);
        a0 = fmaf(p.z, q.z, a0);
        a1 = fmaf(r.z, s.z, a1);
        a0 = fmaf(p.w, q.w, a0);
        a1 = fmaf(r.w, s.w, a1);
    }
}

template <int D>
struct DqSmem {
    float q[kRowsB][D], gf[kRowsB][D], gs[kRowsB][D];
    float k[kChunk][D + 4], v[kChunk][D + 4];  // +4: 16-byte rows, conflict-free per lane
    float lf[kRowsB], ls[kRowsB], df[kRowsB], ds[kRowsB];
    uint32_t mrow[256];
};

// dq of query tile L's 16 rows (tiles in longest-first order)
template <typename T, int D>
__device__ __forceinline__ void dq_tile(DqSmem<D>& sm, int L, const T* __restrict__ q,
                                        const T* __restrict__ k, const T* __restrict__ v,
                                        const uint32_t* __restrict__ mask,
                                        const float* __restrict__ lse_f,
                                        const float* __restrict__ lse_s, const BwdWs& w, int BH,
                                        int T_, int block, int words, float sm_scale,
                                        T* __restrict__ dq) {
    constexpr int DPL = D / 32;
    constexpr int kNE = kChunk * D / kThreads;  // elements per thread of a chunk operand
    static_assert(kNE * kThreads == kChunk * D, "whole chunks per CTA");
    const int ntiles = T_ / kRowsB;
    const int tile = ntiles - 1 - L / BH;
    const size_t bh = L % BH;
    const int t0 = tile * kRowsB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t base = bh * (size_t)T_ * D;
    const size_t rbase = bh * (size_t)T_ + t0;

    for (int e = tid; e < kRowsB * D; e += kThreads) {
        const size_t g = base + (size_t)t0 * D + e;
        sm.q[e / D][e % D] = to_f32(q[g]);
        sm.gf[e / D][e % D] = w.gf[g];
        sm.gs[e / D][e % D] = w.gs[g];
    }
    if (tid < kRowsB) {
        sm.lf[tid] = lse_f[rbase + tid];
        sm.ls[tid] = lse_s[rbase + tid];
        sm.df[tid] = w.df[rbase + tid];
        sm.ds[tid] = w.ds[rbase + tid];
    }
    const uint32_t* mrow = mask + (bh * (T_ / block) + t0 / block) * (size_t)words;
    for (int i = tid; i < words; i += kThreads) sm.mrow[i] = mrow[i];

    float acc[kRowsPerWarp][DPL];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int u = 0; u < DPL; ++u) acc[r][u] = 0.f;

    // chunks of 32 keys from 0 (a chunk lies inside one key block; keys past a
    // row are masked); chunk c + 1 is loaded into registers while chunk c is
    // computed
    T kn[kNE], vn[kNE];
    auto fetch = [&](int s0) {
#pragma unroll
        for (int x = 0; x < kNE; ++x) {
            const size_t g = base + (size_t)s0 * D + tid + x * kThreads;
            kn[x] = k[g];
            vn[x] = v[g];
        }
    };
    const int send = t0 + kRowsB;  // chunks starting below send end at or before T
    fetch(0);
    for (int s0 = 0; s0 < send; s0 += kChunk) {
        __syncthreads();
#pragma unroll
        for (int x = 0; x < kNE; ++x) {
            const int e = tid + x * kThreads;
            sm.k[e / D][e % D] = to_f32(kn[x]);
            sm.v[e / D][e % D] = to_f32(vn[x]);
        }
        __syncthreads();
        if (s0 + kChunk < send) fetch(s0 + kChunk);
        const bool sel = mask_bit(sm.mrow, s0 / block);
#pragma unroll 1
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int rr = warp * kRowsPerWarp + r;
            const int t = t0 + rr;
            const bool valid = s0 + lane <= t;
            float x = 0.f, dpf = 0.f, dps = 0.f;
            dot2_seq<D>(sm.q[rr], sm.k[lane], x, sm.gf[rr], sm.v[lane], dpf);
            x *= sm_scale;
            const float pf = valid ? expf(x - sm.lf[rr]) : 0.f;
            float dsv = pf * (dpf - sm.df[rr]);
            if (sel) {
                dps = dot_seq<D>(sm.gs[rr], sm.v[lane], dps);
                const float lsr = sm.ls[rr];
                const float ps = (valid && lsr > -INFINITY) ? expf(x - lsr) : 0.f;
                dsv += ps * (dps - sm.ds[rr]);
            }
#pragma unroll 8
            for (int j = 0; j < kChunk; ++j) {
                const float dj = __shfl_sync(0xffffffffu, dsv, j);
#pragma unroll
                for (int u = 0; u < DPL; ++u) acc[r][u] = fmaf(dj, sm.k[j][lane + 32 * u], acc[r][u]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const size_t row = rbase + warp * kRowsPerWarp + r;
#pragma unroll
        for (int u = 0; u < DPL; ++u) dq[row * D + lane + 32 * u] = from_f32<T>(sm_scale * acc[r][u]);
    }
}

template <int D>
struct DkvSmem {
    float k[kRowsB][D], v[kRowsB][D];
    float q[kChunk][D + 4], gf[kChunk][D + 4], gs[kChunk][D + 4];  // as above
    float lf[kChunk], ls[kChunk], df[kChunk], ds[kChunk];
};

// dk, dv of key tile L's 16 rows (key tile 0 sees every query: first)
template <typename T, int D>
__device__ __forceinline__ void dkdv_tile(DkvSmem<D>& sm, int L, const T* __restrict__ q,
                                          const T* __restrict__ k, const T* __restrict__ v,
                                          const uint32_t* __restrict__ mask,
                                          const float* __restrict__ lse_f,
                                          const float* __restrict__ lse_s, const BwdWs& w, int BH,
                                          int T_, int block, int words, float sm_scale,
                                          T* __restrict__ dk, T* __restrict__ dv) {
    constexpr int DPL = D / 32;
    constexpr int kNE = kChunk * D / kThreads;  // elements per thread of a chunk operand
    static_assert(kNE * kThreads == kChunk * D, "whole chunks per CTA");
    const int tile = L / BH;
    const size_t bh = L % BH;
    const int s_base = tile * kRowsB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t base = bh * (size_t)T_ * D;
    const int n = T_ / block;
    const int kblk = s_base / block;

    for (int e = tid; e < kRowsB * D; e += kThreads) {
        const size_t g = base + (size_t)s_base * D + e;
        sm.k[e / D][e % D] = to_f32(k[g]);
        sm.v[e / D][e % D] = to_f32(v[g]);
    }
    float adk[kRowsPerWarp][DPL], adv[kRowsPerWarp][DPL];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int u = 0; u < DPL; ++u) adk[r][u] = adv[r][u] = 0.f;

    // chunks of 32 queries from the 32-aligned chunk holding the first key (a
    // chunk lies inside one query block; queries before a key are masked);
    // chunk c + 1 is loaded into registers while chunk c is computed
    T qn[kNE];
    float gfn[kNE], gsn[kNE], lfn = 0.f, lsn = 0.f, dfn = 0.f, dsn = 0.f;
    auto fetch = [&](int t0) {
#pragma unroll
        for (int x = 0; x < kNE; ++x) {
            const size_t g = base + (size_t)t0 * D + tid + x * kThreads;
            qn[x] = q[g];
            gfn[x] = w.gf[g];
            gsn[x] = w.gs[g];
        }
        if (tid < kChunk) {
            const size_t rr = bh * (size_t)T_ + t0 + tid;
            lfn = lse_f[rr];
            lsn = lse_s[rr];
            dfn = w.df[rr];
            dsn = w.ds[rr];
        }
    };
    const int tbeg = s_base & ~(kChunk - 1);  // T is a multiple of 64: chunks end at or before T
    fetch(tbeg);
    for (int t0 = tbeg; t0 < T_; t0 += kChunk) {
        __syncthreads();
#pragma unroll
        for (int x = 0; x < kNE; ++x) {
            const int e = tid + x * kThreads;
            sm.q[e / D][e % D] = to_f32(qn[x]);
            sm.gf[e / D][e % D] = gfn[x];
            sm.gs[e / D][e % D] = gsn[x];
        }
        if (tid < kChunk) {
            sm.lf[tid] = lfn;
            sm.ls[tid] = lsn;
            sm.df[tid] = dfn;
            sm.ds[tid] = dsn;
        }
        __syncthreads();
        if (t0 + kChunk < T_) fetch(t0 + kChunk);
        const uint32_t* mrow = mask + (bh * n + t0 / block) * (size_t)words;
        const bool sel = mask_bit(mrow, kblk);
        const int t = t0 + lane;
#pragma unroll 1
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int rr = warp * kRowsPerWarp + r;
            const int s = s_base + rr;
            const bool valid = t >= s;
            float x = 0.f, dpf = 0.f, dps = 0.f;
            dot2_seq<D>(sm.q[lane], sm.k[rr], x, sm.gf[lane], sm.v[rr], dpf);
            x *= sm_scale;
            const float pf = valid ? expf(x - sm.lf[lane]) : 0.f;
            float dsv = pf * (dpf - sm.df[lane]);
            float ps = 0.f;
            if (sel) {
                dps = dot_seq<D>(sm.gs[lane], sm.v[rr], dps);
                const float lsr = sm.ls[lane];
                ps = (valid && lsr > -INFINITY) ? expf(x - lsr) : 0.f;
                dsv += ps * (dps - sm.ds[lane]);
            }
#pragma unroll 4
            for (int j = 0; j < kChunk; ++j) {
                const float pfj = __shfl_sync(0xffffffffu, pf, j);
                const float psj = __shfl_sync(0xffffffffu, ps, j);
                const float dj = __shfl_sync(0xffffffffu, dsv, j);
#pragma unroll
                for (int u = 0; u < DPL; ++u) {
                    const int c = lane + 32 * u;
                    adv[r][u] = fmaf(pfj, sm.gf[j][c], fmaf(psj, sm.gs[j][c], adv[r][u]));
                    adk[r][u] = fmaf(dj, sm.q[j][c], adk[r][u]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const size_t row = bh * (size_t)T_ + s_base + warp * kRowsPerWarp + r;
#pragma unroll
        for (int u = 0; u < DPL; ++u) {
            dk[row * D + lane + 32 * u] = from_f32<T>(sm_scale * adk[r][u]);
            dv[row * D + lane + 32 * u] = from_f32<T>(adv[r][u]);
        }
    }
}

// dq and dk/dv in one grid: even CTAs take dk/dv key tiles, odd ones dq query
// tiles, each role in its own longest-first order, so the two run side by
// side instead of one after the other.
template <int D>
union BwdSmem {
    DqSmem<D> dq;
    DkvSmem<D> kv;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const uint32_t* __restrict__ mask, const float* __restrict__ lse_f,
                const float* __restrict__ lse_s, BwdWs w, int BH, int T_, int block, int words,
                float sm_scale, T* __restrict__ dq, T* __restrict__ dk, T* __restrict__ dv) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(smem_raw);
    const int L = (int)(blockIdx.x >> 1);
    if (blockIdx.x & 1u)
        dq_tile<T, D>(sm.dq, L, q, k, v, mask, lse_f, lse_s, w, BH, T_, block, words, sm_scale, dq);
    else
        dkdv_tile<T, D>(sm.kv, L, q, k, v, mask, lse_f, lse_s, w, BH, T_, block, words, sm_scale, dk,
                        dv);
}

template <typename T, int D>
int launch_typed(const ssa_params_t& p, const void* q, const void* k, const void* v,
                 const uint32_t* mask, const void* hf, const void* hs, const float* lf,
                 const float* ls, const void* dhf, const void* dhs, float w_s, float w_c,
                 void* dq, void* dk, void* dv, void* ws, cudaStream_t s) {
    const BwdWs w = carve(p, ws);
    const size_t rows = num_rows(p);
    const double two_over_n = 2.0 / (double)num_elems(p);
    bwd_pre_kernel<T><<<(unsigned)((rows + kPreThreads / 32 - 1) / (kPreThreads / 32)), kPreThreads, 0, s>>>(
        static_cast<const T*>(hf), static_cast<const T*>(hs), static_cast<const T*>(dhf),
        static_cast<const T*>(dhs), rows, D, (float)(w_s * two_over_n), (float)(w_c * two_over_n), w);
    int st = check_launch("bwd_pre_kernel");
    if (st != SSA_OK) return st;

    const int BH = p.B * p.H;
    const unsigned grid = (unsigned)(2 * (size_t)BH * (p.T / kRowsB));  // dk/dv and dq tiles
    const size_t smem = sizeof(BwdSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(bwd_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "bwd_simt: smem attribute: %s", cudaGetErrorString(e));
    bwd_simt_kernel<T, D><<<grid, kThreads, smem, s>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), mask, lf, ls,
        w, BH, p.T, p.block, mask_words(p), p.sm_scale, static_cast<T*>(dq), static_cast<T*>(dk),
        static_cast<T*>(dv));
    return check_launch("bwd_simt_kernel");
}

}  // namespace

size_t bwd_simt_workspace(const ssa_params_t& p) {
    return 2 * align_up(num_elems(p) * sizeof(float), 256) +
           2 * align_up(num_rows(p) * sizeof(float), 256);
}

int launch_bwd_simt(const ssa_params_t& p, const void* q, const void* k, const void* v,
                    const uint32_t* mask, const void* hf, const void* hs, const float* lf,
                    const float* ls, const void* dhf, const void* dhs, float w_s, float w_c,
                    void* dq, void* dk, void* dv, void* ws, cudaStream_t s) {
    if (mask_words(p) > 256) return fail(SSA_ERR_UNSUPPORTED, "bwd_simt: more than 8192 blocks");
    if (2 * (size_t)p.B * p.H * (p.T / kRowsB) > 0x7fffffffull)
        return fail(SSA_ERR_UNSUPPORTED, "bwd_simt: grid too large");
    const bool bf = p.dtype == SSA_BF16;
#define SSA_BWD_ARGS p, q, k, v, mask, hf, hs, lf, ls, dhf, dhs, w_s, w_c, dq, dk, dv, ws, s
    if (p.D == 64)
        return bf ? launch_typed<__nv_bfloat16, 64>(SSA_BWD_ARGS) : launch_typed<float, 64>(SSA_BWD_ARGS);
    return bf ? launch_typed<__nv_bfloat16, 128>(SSA_BWD_ARGS) : launch_typed<float, 128>(SSA_BWD_ARGS);
#undef SSA_BWD_ARGS
}

}  // namespace ssa

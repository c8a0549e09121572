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
// the key/value bytes it reads and, at this size, by latency):
//   decode_pool_kernel   Kbar_j = mean of block j's keys (float64, exact)
//   decode_step_kernel   one cluster of 8 (or 4) CTAs per head; distributed shared
//                        memory carries every hand-off, so the step is one
//                        launch with no global round trips:
//     1. every CTA scores its share of the completed blocks (warp per block,
//        lanes over d, float64) into the leader CTA's score array;
//     2. the leader ranks the candidates (each thread counts, for its blocks,
//        the candidates ahead of it under (score desc, index asc)), keeps
//        those ranked below the free places, writes the ascending list and
//        hands it to every CTA;
//     3. every CTA attends over its selected blocks, two at a time (one per
//        half of its 16 warps): the block's keys and values are loaded
//        together (16-byte value loads), scores with a warp per group of
//        keys, softmax statistics over the half, P V with threads over
//        (8-column chunk, key group); the partial (max, sum, o) goes to the
//        leader;
//     4. the leader merges the partials into h and the log-sum-exp.
#include <cooperative_groups.h>
#include <type_traits>

#include "device_util.cuh"
#include "ssa_internal.h"

namespace cg = cooperative_groups;

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

constexpr int kStepThreads = 512; // two halves of 8 warps: two selected blocks at a time

// Shared memory of the step kernel (every CTA has the same layout; only the
// leader's score, list and partial areas are used): scores [nb] f64 | set
// bitmask [nb / 32 + 1] u32 | selected blocks [topk] i32 | partials
// [topk][2 + D] f32.
struct StepSmem {
    static size_t bytes(int nb, int topk, int D) {
        return (size_t)nb * 8 + ((size_t)nb / 32 + 1) * 4 + (size_t)topk * 4 +
               (size_t)topk * (2 + D) * 4 + 16;
    }
};

// kCluster: CTAs per head, 8 or 4 (chosen by the host from the head count)
template <typename T, int D, int kCluster>
__global__ void __launch_bounds__(kStepThreads, 1)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const double* __restrict__ kbar, int nb, int Tcap, int block, int t, int topk,
                   bool force_sink, float scale, T* __restrict__ h, float* __restrict__ lse,
                   int32_t* __restrict__ idx_out) {
    constexpr int M = D / 32;              // query columns per lane (scores)
    constexpr int U = 4;                   // key blocks in flight per warp
    constexpr int NWT = kStepThreads / 32; // warps of the CTA
    constexpr int HT = kStepThreads / 2;   // threads of a half
    constexpr int NW = HT / 32;            // warps of a half
    constexpr int E = D / 32;              // columns per lane (attention scores)
    constexpr int KPW = 128 / NW;          // keys per warp (block <= 128)
    constexpr int CH = D / 8;              // 8-column chunks of a value row
    constexpr int KG = HT / CH;            // key groups of a half
    constexpr int VPT = 128 / KG;          // value rows per thread
    extern __shared__ __align__(16) unsigned char sm[];
    __shared__ float ps[2][128];           // per half: scores, then e^{x - m}
    __shared__ float red[2][NW];
    __shared__ float og[2][KG * D];        // per half: [key group][d] partial sums of P V
    __shared__ float wgt[kMaxTopk];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = t / block;
    const int words = (i >> 5) + 1;  // bits 0 .. i
    double* score = reinterpret_cast<double*>(sm);
    uint32_t* bits = reinterpret_cast<uint32_t*>(score + nb);
    int32_t* sel = reinterpret_cast<int32_t*>(bits + nb / 32 + 1);
    float* part = reinterpret_cast<float*>(sel + topk);
    // the leader's arrays, as every CTA of the cluster addresses them
    double* score_l = cluster.map_shared_rank(score, 0);
    int32_t* sel_l = cluster.map_shared_rank(sel, 0);
    float* part_l = cluster.map_shared_rank(part, 0);

    // 1. scores of the completed blocks j < i: block j goes to CTA j % kCluster,
    // warp (j / kCluster) % 16; lane l owns columns l, l + 32, ... (coalesced rows of the
    // float64 pooled keys), U blocks' loads in flight per warp
    {
        double qr[M];
#pragma unroll
        for (int m = 0; m < M; ++m) qr[m] = (double)to_f32(q[bh * D + lane + 32 * m]);
        const double* kb = kbar + bh * (size_t)nb * D;
        for (int c0 = rank + kCluster * warp; c0 < i; c0 += kCluster * NWT * U) {
            double a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = c0 + kCluster * NWT * u;
                const double* kr = kb + (size_t)min(j, i - 1) * D + lane;  // past the end: unused
                double acc = 0.0;
#pragma unroll
                for (int m = 0; m < M; ++m) acc = fma(qr[m], kr[32 * m], acc);
                a[u] = acc;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) a[u] = warp_sum(a[u]);
            if (lane == 0) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = c0 + kCluster * NWT * u;
                    if (j < i) score_l[j] = a[u];
                }
            }
        }
    }
    cluster.sync();

    // 2. the leader selects: forced blocks, then candidate j (first <= j < i) is
    // kept iff fewer than r candidates come before it in (score desc, index asc)
    if (rank == 0) {
        const bool sink = force_sink && i > 0;
        const int want = topk < i + 1 ? topk : i + 1;  // fewer candidates than places: take all
        const int first = sink ? 1 : 0;                // candidates are first .. i-1
        const int r = want - (sink ? 2 : 1);           // free slots (>= 0: a sink needs topk >= 2)
        for (int w = tid; w < words; w += kStepThreads) bits[w] = 0u;
        __syncthreads();
        if (tid == 0) {
            bits[i >> 5] |= 1u << (i & 31);
            if (sink) bits[0] |= 1u;
        }
        for (int j = first + tid; j < i; j += kStepThreads) {
            const double sj = score[j];
            int ahead = 0;
            int j2 = first;
            for (; j2 + 4 <= i; j2 += 4) {  // four independent loads per iteration
                const double a0 = score[j2], a1 = score[j2 + 1], a2 = score[j2 + 2], a3 = score[j2 + 3];
                ahead += (a0 > sj || (a0 == sj && j2 < j)) ? 1 : 0;
                ahead += (a1 > sj || (a1 == sj && j2 + 1 < j)) ? 1 : 0;
                ahead += (a2 > sj || (a2 == sj && j2 + 2 < j)) ? 1 : 0;
                ahead += (a3 > sj || (a3 == sj && j2 + 3 < j)) ? 1 : 0;
            }
            for (; j2 < i; ++j2) {
                const double a0 = score[j2];
                ahead += (a0 > sj || (a0 == sj && j2 < j)) ? 1 : 0;
            }
            if (ahead < r) atomicOr(&bits[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
        if (warp == 0) {  // the ascending list (-1 padded) by popcount prefix
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
                        const int vv = w * 32 + __ffs(b) - 1;
                        sel[pos] = vv;
                        if (irow) irow[pos] = vv;
                    }
                }
                base += __shfl_sync(0xffffffffu, incl, 31);
            }
            for (int pp = base + lane; pp < topk; pp += 32) {
                sel[pp] = -1;
                if (irow) irow[pp] = -1;
            }
        }
    }
    cluster.sync();

    // 3. slots rank, rank + kCluster, ... of the list: half hf (8 warps) of the CTA takes
    // every other one, so that two blocks' loads are in flight at once.  Per
    // block: keys and values loaded together (16-byte value loads; thread
    // (8-column chunk c8, key group g)), scores by a warp per group of keys,
    // softmax statistics over the half, partial (m, l, o[D]) to the leader.
    {
        const int hf = warp / NW, hw = warp % NW, ht = tid % HT;
        const uint32_t hbar = 1u + (uint32_t)hf;  // named barrier of the half
        auto hsync = [hbar] { asm volatile("bar.sync %0, %1;" ::"r"(hbar), "n"(HT) : "memory"); };
        float qv[E];
        load_row_piece<T, E>(q + bh * D + E * lane, qv);
        for (int slot = rank + kCluster * hf; slot < topk; slot += 2 * kCluster) {
            float* out = part_l + slot * (2 + D);
            const int j = sel_l[slot];
            const int s0 = j < 0 ? 0 : j * block;
            const int nks = j < 0 ? 0 : min((j + 1) * block, t + 1) - s0;  // keys of this block <= t
            const int c8 = ht % CH, g = ht / CH;
            uint4 vr[VPT];
#pragma unroll
            for (int m = 0; m < VPT; ++m) {
                const int s = g + KG * m;
                vr[m] = s < nks ? *reinterpret_cast<const uint4*>(
                                      reinterpret_cast<const char*>(v + (bh * Tcap + s0 + s) * D) +
                                      16 * c8 * (int)sizeof(T) / 2)
                                : make_uint4(0u, 0u, 0u, 0u);
            }
            float acc[KPW];
#pragma unroll
            for (int kk = 0; kk < KPW; ++kk) {
                const int s = hw + NW * kk;
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
                const int s = hw + NW * kk;
                const float dot = warp_sum(acc[kk]);
                if (lane == 0 && s < nks) ps[hf][s] = dot * scale;
            }
            hsync();
            // m = max over the block's keys, then p = e^{x - m} and l = sum p
            const float x = ht < nks ? ps[hf][ht] : -INFINITY;
            float mx = warp_max(x);
            if (lane == 0) red[hf][hw] = mx;
            hsync();
            float m = red[hf][0];
            for (int w = 1; w < NW; ++w) m = fmaxf(m, red[hf][w]);
            hsync();
            float p = 0.f;
            if (ht < nks) {
                p = expf(x - m);
                ps[hf][ht] = p;
            }
            const float ls = warp_sum(p);
            if (lane == 0) red[hf][hw] = ls;
            hsync();
            float l = 0.f;
            for (int w = 0; w < NW; ++w) l += red[hf][w];
            // o = sum_s p_s v_s over this thread's value rows and 8 columns, then
            // over the key groups through shared memory
            float o8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m2 = 0; m2 < VPT; ++m2) {
                const int s = g + KG * m2;
                if (s < nks) {
                    const float pw = ps[hf][s];
                    const T* e = reinterpret_cast<const T*>(&vr[m2]);
                    if constexpr (sizeof(T) == 2) {
#pragma unroll
                        for (int z = 0; z < 8; ++z) o8[z] = fmaf(pw, to_f32(e[z]), o8[z]);
                    } else {  // float: a 16-byte load holds 4 columns; the chunk's other 4 follow
                        const T* e2 = reinterpret_cast<const T*>(v + (bh * Tcap + s0 + s) * D) + 8 * c8 + 4;
#pragma unroll
                        for (int z = 0; z < 4; ++z) {
                            o8[z] = fmaf(pw, to_f32(e[z]), o8[z]);
                            o8[4 + z] = fmaf(pw, to_f32(e2[z]), o8[4 + z]);
                        }
                    }
                }
            }
#pragma unroll
            for (int z = 0; z < 8; ++z) og[hf][g * D + 8 * c8 + z] = o8[z];
            hsync();
            for (int c = ht; c < D; c += HT) {
                float o = 0.f;
                for (int gg = 0; gg < KG; ++gg) o += og[hf][gg * D + c];
                out[2 + c] = o;
            }
            if (ht == 0) {
                out[0] = nks > 0 ? m : -INFINITY;
                out[1] = l;
            }
            hsync();  // ps, red and og are reused by the half's next block
        }
    }
    cluster.sync();

    // 4. the leader merges the partials: weights e^{m_a - M}
    if (rank != 0) return;
    if (warp == 0) {
        float Mx = -INFINITY;
        for (int a = lane; a < topk; a += 32) Mx = fmaxf(Mx, part[a * (2 + D)]);
        Mx = warp_max(Mx);
        float L = 0.f;
        for (int a = lane; a < topk; a += 32) {
            const float ma = part[a * (2 + D)];
            const float w = ma > -INFINITY ? expf(ma - Mx) : 0.f;
            wgt[a] = w;
            L += w * part[a * (2 + D) + 1];
        }
        L = warp_sum(L);
        if (lane == 0) {
            red[0][0] = L;
            lse[bh] = Mx + logf(L);
        }
    }
    __syncthreads();
    const float inv_L = 1.f / red[0][0];
    for (int c = tid; c < D; c += kStepThreads) {
        float acc = 0.f;
        for (int a = 0; a < topk; ++a) acc = fmaf(wgt[a], part[a * (2 + D) + 2 + c], acc);
        h[bh * D + c] = from_f32<T>(acc * inv_L);
    }
}

}  // namespace

// the step keeps everything in the clusters' shared memory: no workspace
size_t decode_workspace(const ssa_params_t&) { return 0; }

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
                       const double* kbar, void* h, float* lse, int32_t* idx, void*,
                       cudaStream_t s) {
    const int BH = p.B * p.H;
    const int nb = num_blocks(p);
    const bool sink = (p.flags & SSA_FLAG_FORCE_SINK) != 0;
    const size_t smem = StepSmem::bytes(nb, p.topk, p.D);
    // 8 CTAs per head while every head's cluster fits in one wave (a cluster of
    // 8 CTAs of 512 threads takes 8 SMs of one GPC; measured: 8 clusters at a
    // time), else 4 (two selected blocks per half then run one after the other)
    const int cl = BH <= 8 ? 8 : 4;
    auto run = [&](auto tag, auto dtag, auto ctag) -> int {
        using T = decltype(tag);
        constexpr int D = decltype(dtag)::value;
        constexpr int kCluster = decltype(ctag)::value;
        auto kern = decode_step_kernel<T, D, kCluster>;
        size_t limit = 0;
        int st = opt_in_max_smem<decode_step_kernel<T, D, kCluster>>("decode_step_kernel", &limit);
        if (st != SSA_OK) return st;
        if (smem > limit)
            return fail(SSA_ERR_UNSUPPORTED, "decode: T/block = %d blocks need %zu bytes of shared memory (limit %zu)",
                        nb, smem, limit);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)kCluster, (unsigned)BH);
        cfg.blockDim = dim3(kStepThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(k),
                                           static_cast<const T*>(v), kbar, nb, p.T, p.block, t, p.topk,
                                           sink, p.sm_scale, static_cast<T*>(h), lse, idx);
        if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "decode_step_kernel: %s", cudaGetErrorString(e));
        return check_launch("decode_step_kernel");
    };
    using D64 = std::integral_constant<int, 64>;
    using D128 = std::integral_constant<int, 128>;
    using C4 = std::integral_constant<int, 4>;
    using C8 = std::integral_constant<int, 8>;
    auto with_cluster = [&](auto tag, auto dtag) -> int {
        return cl == 8 ? run(tag, dtag, C8{}) : run(tag, dtag, C4{});
    };
    if (p.dtype == SSA_BF16)
        return p.D == 64 ? with_cluster(__nv_bfloat16{}, D64{}) : with_cluster(__nv_bfloat16{}, D128{});
    return p.D == 64 ? with_cluster(float{}, D64{}) : with_cluster(float{}, D128{});
}

}  // namespace ssa

// Small device helpers shared by the CUDA-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssa {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Bit j of the selection mask row (query block) `row` of width `words`.
__device__ __forceinline__ bool mask_bit(const uint32_t* row, int j) {
    return (row[j >> 5] >> (j & 31)) & 1u;
}

// Top-k of a row of block scores by one warp (block selection, and the
// decode step): the r free slots among the candidates first .. i-1 are
// filled by r rounds of warp argmax under (score desc, index asc).  Lane
// l owns the candidates j = first + l (mod 32) and keeps its best one; after
// a round only the winning lane rescans, for its best candidate strictly
// below the one just taken in that order.  Winners are OR-ed into bits.
__device__ __forceinline__ void warp_topk_rounds(const double* sc, int first, int i, int r,
                                                 uint32_t* bits, int lane) {
    double bs = 0.0;
    int bj = -1;
    for (int j = first + lane; j < i; j += 32) {
        const double s = sc[j];
        if (bj < 0 || s > bs) { bs = s; bj = j; }  // ascending j: ties keep the lower index
    }
    for (int round = 0; round < r; ++round) {
        double ws = bs;
        int wj = bj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const double os = __shfl_xor_sync(0xffffffffu, ws, off);
            const int oj = __shfl_xor_sync(0xffffffffu, wj, off);
            if (oj >= 0 && (wj < 0 || os > ws || (os == ws && oj < wj))) { ws = os; wj = oj; }
        }
        wj = __shfl_sync(0xffffffffu, wj, 0);  // lane 0 decides (NaN scores need not agree)
        ws = __shfl_sync(0xffffffffu, ws, 0);
        if (wj < 0) break;
        if (lane == 0) atomicOr(&bits[wj >> 5], 1u << (wj & 31));
        if (bj == wj) {
            bj = -1;
            for (int j = first + lane; j < i; j += 32) {
                const double s = sc[j];
                if (!(s < ws || (s == ws && j > wj))) continue;  // taken already
                if (bj < 0 || s > bs) { bs = s; bj = j; }
            }
        }
    }
}

}  // namespace ssa

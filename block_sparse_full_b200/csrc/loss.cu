// Alignment losses L_sparsity and L_commit ("Sintesi Tecnica: SSA",
// section 2, "Allineamento Bidirezionale").  Both are the mean squared
// difference of the two outputs over all B*H*T*D elements; their values are
// equal and they differ only in which stream receives the gradient, so the
// forward reduces the per-row sums sqdiff_rows once and scales by each
// weight.  Two launches, fixed partition and fixed reduction order in
// float64: bitwise repeatable.
#include "device_util.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxParts = 1024;
constexpr size_t kRowsPerPart = 4096;

__device__ double block_sum(double x) {
    __shared__ double warp_part[kThreads / 32];
    x = warp_sum(x);
    if ((threadIdx.x & 31) == 0) warp_part[threadIdx.x >> 5] = x;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kThreads / 32; ++w) s += warp_part[w];
    return s;  // valid in thread 0
}

__global__ void __launch_bounds__(kThreads)
loss_partial_kernel(const float* __restrict__ r, size_t rows, size_t per_part,
                    double* __restrict__ part) {
    const size_t beg = blockIdx.x * per_part;
    const size_t end = beg + per_part < rows ? beg + per_part : rows;
    double acc = 0.0;
    for (size_t i = beg + threadIdx.x; i < end; i += kThreads) acc += (double)r[i];
    const double s = block_sum(acc);
    if (threadIdx.x == 0) part[blockIdx.x] = s;
}

__global__ void __launch_bounds__(kThreads)
loss_final_kernel(const double* __restrict__ part, int nparts, double inv_n, float w_s,
                  float w_c, float* __restrict__ out) {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nparts; i += kThreads) acc += part[i];
    const double s = block_sum(acc);
    if (threadIdx.x == 0) {
        const double L = s * inv_n;
        out[0] = (float)((double)w_s * L);
        out[1] = (float)((double)w_c * L);
    }
}

int parts_for(size_t rows) {
    size_t per = kRowsPerPart;
    size_t parts = (rows + per - 1) / per;
    return parts > (size_t)kMaxParts ? kMaxParts : (int)parts;
}

}  // namespace

size_t loss_workspace(const ssa_params_t& p) {
    return align_up((size_t)parts_for(num_rows(p)) * sizeof(double), 256);
}

int launch_loss(const ssa_params_t& p, const float* sqdiff, float w_s, float w_c,
                float* loss_out, void* ws, cudaStream_t s) {
    const size_t rows = num_rows(p);
    const int parts = parts_for(rows);
    const size_t per = (rows + parts - 1) / parts;
    double* part = static_cast<double*>(ws);
    loss_partial_kernel<<<parts, kThreads, 0, s>>>(sqdiff, rows, per, part);
    int st = check_launch("loss_partial_kernel");
    if (st != SSA_OK) return st;
    loss_final_kernel<<<1, kThreads, 0, s>>>(part, parts, 1.0 / (double)num_elems(p), w_s, w_c,
                                             loss_out);
    return check_launch("loss_final_kernel");
}

}  // namespace ssa

// Block selection for callers that cannot allocate device memory.
//
// ssa_select_blocks needs a caller-provided scratch buffer (the float64 block
// means of Q and K).  Some host programs cannot produce one at the point
// where they run selection: a plugin loaded into a serving process whose
// memory pool owns all device memory and exposes no allocator to plugins, or
// a latency-critical loop that must not call cudaMalloc after start-up
// (cudaMalloc can synchronise the device and stall every other stream).
// ssa_select_blocks_noalloc serves them with a scratch buffer that lives in
// this library's own device memory: a file-scope array that every GPU which
// loads the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a shadow variable), so the device address is looked up with
// cudaGetSymbolAddress while the device is current, on the first call made in
// each CUDA context, and cached against that context's unique ID: after a
// cudaDeviceReset the next call runs in a new primary context, where the
// module (and with it the array) has been loaded again, and looks the address
// up again instead of using the old one.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ssa_internal.h"

namespace {

// 16 MiB: enough for B*H*(T/block)*D <= 1,048,576, e.g. B=4 H=32 T=4096
// block=64 d=128 or B=1 H=8 T=65536 block=128 d=128.
constexpr size_t kScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
struct Cached {
    unsigned long long ctx_id;  // 0 = nothing cached
    void* addr;
};
Cached g_cache[kMaxDevices] = {};

// Unique ID of the calling thread's current CUDA context (0 if none or the
// driver entry points are unavailable), through the runtime's driver
// entry-point query so that the library needs no link against libcuda.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_select_scratch on the current device, valid in the
// current context.  Returns an SSA status.
int scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ssa::fail(SSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return ssa::fail(SSA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_mutex);
    const unsigned long long id = current_context_id();
    if (id == 0 || g_cache[dev].ctx_id != id) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || !p)
            return ssa::fail(SSA_ERR_CUDA, "cudaGetSymbolAddress(select scratch): %s",
                             cudaGetErrorString(e));
        // the lookup makes the primary context current if none was; cache under it
        g_cache[dev] = Cached{id ? id : current_context_id(), p};
    }
    *out = g_cache[dev].addr;
    return SSA_OK;
}

}  // namespace

extern "C" int ssa_select_blocks_noalloc(const ssa_params_t* p, const void* q, const void* k,
                                         int32_t* idx, int32_t* cnt, uint32_t* mask,
                                         void* stream) {
    const size_t need = ssa_workspace_size(p, SSA_WS_SELECT);
    if (need == (size_t)-1) return SSA_ERR_INVALID_ARG;  // detail already recorded
    if (need > kScratchBytes)
        return ssa::fail(SSA_ERR_UNSUPPORTED,
                         "ssa_select_blocks_noalloc: these shapes need %zu bytes of scratch but the "
                         "built-in scratch holds %zu (B*H*(T/block)*D must be <= %zu); call "
                         "ssa_select_blocks with a caller-allocated workspace instead",
                         need, kScratchBytes, kScratchBytes / (2 * sizeof(double)));
    void* scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != SSA_OK) return st;
    // The pooling kernel writes every block mean before the scoring kernel
    // reads it, so leftovers from an earlier call never need clearing.
    return ssa_select_blocks(p, q, k, idx, cnt, mask, scratch, kScratchBytes, stream);
}

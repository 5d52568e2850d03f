// route_noalloc.cu -- routing that never allocates device memory.
//
// moe_route() needs a handle, and creating a handle calls cudaMalloc for its
// scratch.  Some callers cannot do that: code that runs while a CUDA graph is
// being captured (an allocation there breaks or invalidates the capture),
// plug-ins that live inside another framework which owns all device memory
// through its own allocator, and latency-critical loops that cannot afford
// the device-wide synchronisation cudaMalloc may imply.  moe_route_noalloc()
// serves them: the caller passes the router weights, the activations and the
// output buffers, and every intermediate (per-expert row norms, fp32 logits,
// counters) lives in one fixed array of device memory declared below, which
// each GPU that loads this library holds until the process exits.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace {

// Capacity of the fixed scratch: logits of up to kMaxLogits (token, expert)
// pairs, norms of up to 1024 experts, and the small counter block.
constexpr int kMaxLogits = 65536;  // T * E
constexpr int kMaxExperts = 1024;
// Largest model width: the logits kernel stages four token rows of d fp32
// values in shared memory (16 * d bytes), within every sm_100 part's opt-in
// limit at d = 8192.
constexpr int kMaxWidth = 8192;
constexpr size_t kScratchFloats = kMaxLogits + kMaxExperts + 64;

// File-scope device array; the host side only ever sees its symbol, whose
// device address comes from cudaGetSymbolAddress on the device in use.
static __device__ __align__(256) float g_route_scratch[kScratchFloats];

// The array's device address, looked up on every call with the caller's
// device current.  The lookup is a host-side table read, cheap next to the
// three launches; caching it would go stale if the context holding the module
// were torn down and recreated (the module reloads, and the array may move),
// and a shared cache would need synchronising between host threads.
// Returns nullptr if the lookup fails.
float* scratch_for_current_device() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
    return static_cast<float*>(p);
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* x, int32_t T, int32_t d, int32_t n_experts, int32_t top_k,
                                        const void* router_w, const float* router_bias, int32_t* ids, float* w,
                                        void* stream) {
    if (T < 0 || d <= 0 || d % 128 || d > kMaxWidth || n_experts < 1 || n_experts > kMaxExperts || top_k < 1 || top_k > 32 ||
        top_k > n_experts)
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)T * n_experts > kMaxLogits) return MOE_ERR_INVALID_ARG;  // beyond the fixed scratch
    if (T == 0) return MOE_OK;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!x || !router_w || !ids || !w || !al16(x) || !al16(router_w) || !al16(ids) || !al16(w) ||
        (router_bias && (reinterpret_cast<uintptr_t>(router_bias) & 3u)))
        return MOE_ERR_INVALID_ARG;
    float* base = scratch_for_current_device();
    if (!base) return MOE_ERR_CUDA;
    float* logits = base;
    float* norms = base + kMaxLogits;
    moe::Meta* meta = reinterpret_cast<moe::Meta*>(base + kMaxLogits + kMaxExperts);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The counter block keeps the previous call's values: start it at zero.
    if (cudaMemsetAsync(meta, 0, sizeof(moe::Meta), s) != cudaSuccess) return MOE_ERR_CUDA;
    if (moe::launch_router_norms(router_w, n_experts, d, norms, s) != cudaSuccess) return MOE_ERR_CUDA;
    moe::RouteArgs ra;
    ra.x = x;
    ra.T = T;
    ra.d = d;
    ra.E = n_experts;
    ra.k = top_k;
    ra.wr = router_w;
    ra.bias = router_bias;
    ra.wnorm = norms;
    ra.logits = logits;
    ra.ids = ids;
    ra.w = w;
    ra.meta = meta;
    if (moe::launch_router_logits(ra, s) != cudaSuccess) return MOE_ERR_CUDA;
    return moe::launch_topk(ra, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// norm.cu -- root-mean-square normalisation of a bf16 residual stream.
//
// Not a step of the routed-MoE layer: a helper for callers that chain layers.
// The model family the pages describe normalises the residual stream before
// each MoE layer (pre-norm, tech.okbari.net guide, section "Strata, Qwen and
// GSQ-RCO are different components": a standard transformer stack of 48
// layers); without it x_{l+1} = x_l + y_l grows without bound, because the
// SwiGLU output is quadratic in its input.
//   out[t] = bf16( x[t] / sqrt(mean_i x[t,i]^2 + eps) )   (no learned gain)
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) rms_normalize_kernel(const __nv_bfloat16* __restrict__ x, int d,
                                                            __nv_bfloat16* __restrict__ out, float eps) {
    __shared__ float part[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const __nv_bfloat16* xr = x + (int64_t)t * d;
    float ss = 0.f;
    for (int i = tid * 8; i < d; i += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(u[q] << 16), b = __uint_as_float(u[q] & 0xFFFF0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) part[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += part[w];
    const float inv = rsqrtf(tot / (float)d + eps);
    for (int i = tid * 8; i < d; i += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t o4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 r = __floats2bfloat162_rn(__uint_as_float(u[q] << 16) * inv,
                                                           __uint_as_float(u[q] & 0xFFFF0000u) * inv);
            o4[q] = *reinterpret_cast<const uint32_t*>(&r);
        }
        *reinterpret_cast<uint4*>(out + (int64_t)t * d + i) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

cudaError_t launch_rms_normalize(const void* x, int T, int d, void* out, float eps, cudaStream_t s) {
    rms_normalize_kernel<<<T, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), d, static_cast<__nv_bfloat16*>(out),
                                           eps);
    return cudaGetLastError();
}

}  // namespace moe

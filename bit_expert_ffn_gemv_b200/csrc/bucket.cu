// bucket.cu -- group the T*k (token, slot) pairs by expert.
//
// Counting sort, stable in the token index: per-expert counts, an exclusive
// scan over experts, and a scatter that keeps ascending token order inside
// each expert's group (so the grouping, and everything computed from it, is
// deterministic).  One CTA of 32 warps; warp w owns a contiguous token range,
// which makes the per-warp counts a stable prefix.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBucketWarps = 32;

__global__ void __launch_bounds__(kBucketWarps * 32)
    bucket_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ pairs, int32_t* __restrict__ inv, int32_t* __restrict__ active,
                  Meta* __restrict__ meta, uint32_t* __restrict__ status) {
    extern __shared__ int32_t sm[];
    int32_t* cnt = sm;                          // [kBucketWarps][E]
    int32_t* total = sm + kBucketWarps * E;     // [E]
    int32_t* off_s = total + E;                 // [E + 1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tpw = (T + kBucketWarps - 1) / kBucketWarps;
    const int t_begin = min(T, warp * tpw), t_end = min(T, t_begin + tpw);

    for (int i = threadIdx.x; i < kBucketWarps * E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();

    // phase 1: per-warp counts
    for (int t = t_begin; t < t_end; ++t) {
        if (lane < k) {
            int e = ids[(int64_t)t * k + lane];
            if (e < 0 || e >= E) {
                flag_status(status, kStatusBounds);
            } else {
                atomicAdd(&cnt[warp * E + e], 1);
            }
        }
    }
    __syncthreads();

    // phase 2: per-expert prefix over warps, totals
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kBucketWarps; ++w) {
            int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
        total[e] = run;
    }
    __syncthreads();

    // exclusive scan over experts + active list (warp 0)
    if (warp == 0) {
        int base = 0, nact = 0, mx = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            int e = e0 + lane;
            int c = e < E ? total[e] : 0;
            int inc = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (e < E) off_s[e] = base + inc - c;
            unsigned b = __ballot_sync(0xffffffffu, c > 0);
            if (c > 0) active[nact + __popc(b & ((1u << lane) - 1u))] = e;
            nact += __popc(b);
            int m = c;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            mx = max(mx, m);
            base += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            off_s[E] = base;
            meta->n_active = nact;
            meta->max_count = mx;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = off_s[e];

    // phase 3: stable scatter (a token's k experts are distinct)
    for (int t = t_begin; t < t_end; ++t) {
        if (lane < k) {
            int e = ids[(int64_t)t * k + lane];
            if (e >= 0 && e < E) {
                int pos = off_s[e] + cnt[warp * E + e];
                cnt[warp * E + e] += 1;
                pairs[pos] = t * k + lane;
                inv[(int64_t)t * k + lane] = pos;
            } else {
                inv[(int64_t)t * k + lane] = -1;
            }
        }
        __syncwarp();
    }
}

cudaError_t launch_bucket(const BucketArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(int32_t) * ((size_t)kBucketWarps * a.E + 2 * (size_t)a.E + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    bucket_kernel<<<1, kBucketWarps * 32, smem, s>>>(a.ids, a.T, a.k, a.E, a.offsets, a.pairs, a.inv, a.active,
                                                     a.meta, a.status);
    return cudaGetLastError();
}

}  // namespace moe

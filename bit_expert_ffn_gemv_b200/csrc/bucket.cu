// bucket.cu -- group the T*k (token, slot) pairs by expert.
//
// Counting sort, stable in the token index: per-expert counts, an exclusive
// scan over experts, and a scatter that keeps ascending token order inside
// each expert's group (so the grouping, and everything computed from it, is
// deterministic).  One CTA of 32 warps; warp w owns a contiguous range of
// (token, rank) pairs, which makes the per-warp counts a stable prefix.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBucketWarps = 32;

// Warp w owns the contiguous range of pair indices p = t*k + r in
// [w*ppw, (w+1)*ppw); ascending p means ascending t, so per-warp counts and
// in-warp ranks (lanes with equal expert, by lane order) give a stable order.
__global__ void __launch_bounds__(kBucketWarps * 32)
    bucket_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ pairs, int32_t* __restrict__ inv, int32_t* __restrict__ active,
                  Meta* __restrict__ meta, uint32_t* __restrict__ status, const float* __restrict__ w,
                  float* __restrict__ wsorted) {
    extern __shared__ int32_t sm[];
    int32_t* cnt = sm;                          // [kBucketWarps][E]
    int32_t* total = sm + kBucketWarps * E;     // [E]
    int32_t* off_s = total + E;                 // [E + 1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_pairs = T * k;
    const int ppw = ((n_pairs + kBucketWarps - 1) / kBucketWarps + 31) & ~31;
    const int p_begin = min(n_pairs, warp * ppw), p_end = min(n_pairs, p_begin + ppw);
    const uint32_t lt = (1u << lane) - 1u;

    for (int i = threadIdx.x; i < kBucketWarps * E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();

    // phase 1: per-warp counts (one smem update per distinct expert per 32
    // pairs); ids are read 8 x 32 at a time so the loads overlap
    for (int p0 = p_begin; p0 < p_end; p0 += 256) {
        int ev[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int p = p0 + 32 * u + lane;
            ev[u] = p < p_end ? __ldg(&ids[p]) : -1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = ev[u];
            const bool live = p0 + 32 * u + lane < p_end;
            const bool valid = live && e >= 0 && e < E;
            if (live && !valid) flag_status(status, kStatusBounds);
            const uint32_t same = __match_any_sync(0xffffffffu, valid ? e : -1);
            if (valid && (same & lt) == 0) cnt[warp * E + e] += __popc(same);
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
            if (c > 0) active[nact + __popc(b & lt)] = e;
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

    // phase 3: stable scatter (and, if asked, the routing weights in group order)
    for (int p0 = p_begin; p0 < p_end; p0 += 256) {
        int ev[8];
        float wv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int p = p0 + 32 * u + lane;
            ev[u] = p < p_end ? __ldg(&ids[p]) : -1;
            wv[u] = (wsorted && p < p_end) ? __ldg(&w[p]) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = ev[u];
            const int p = p0 + 32 * u + lane;
            const bool live = p < p_end;
            const bool valid = live && e >= 0 && e < E;
            const uint32_t same = __match_any_sync(0xffffffffu, valid ? e : -1);
            const int leader = __ffs(same) - 1;
            int base = 0;
            if (valid && lane == leader) {
                base = off_s[e] + cnt[warp * E + e];
                cnt[warp * E + e] += __popc(same);
            }
            base = __shfl_sync(0xffffffffu, base, leader);
            if (valid) {
                const int pos = base + __popc(same & lt);
                pairs[pos] = p;
                inv[p] = pos;
                if (wsorted) wsorted[pos] = wv[u];
            } else if (live) {
                inv[p] = -1;
            }
        }
    }
}

cudaError_t launch_bucket(const BucketArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(int32_t) * ((size_t)kBucketWarps * a.E + 2 * (size_t)a.E + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    bucket_kernel<<<1, kBucketWarps * 32, smem, s>>>(a.ids, a.T, a.k, a.E, a.offsets, a.pairs, a.inv, a.active,
                                                     a.meta, a.status, a.w, a.wsorted);
    return cudaGetLastError();
}

}  // namespace moe

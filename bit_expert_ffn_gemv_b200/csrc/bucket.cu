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
#include "tiles.cuh"

namespace moe {

constexpr int kBucketWarps = 32;
static_assert(kBucketWarps * 32 == kTileListThreads, "the bucketing CTA can build the tile list");
int bucket_kernel_count(const BucketArgs& a);

// Warp w owns the contiguous range of pair indices p = t*k + r in
// [w*ppw, (w+1)*ppw); ascending p means ascending t, so per-warp counts and
// in-warp ranks (lanes with equal expert, by lane order) give a stable order.
__global__ void __launch_bounds__(kBucketWarps * 32)
    bucket_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ pairs, int32_t* __restrict__ inv, int32_t* __restrict__ active,
                  Meta* __restrict__ meta, uint32_t* __restrict__ status, const float* __restrict__ w,
                  float* __restrict__ wsorted, int R, int e0, int e1, int4* __restrict__ desc_gu,
                  int4* __restrict__ desc_dn, int32_t* __restrict__ tile_counts, int n_shared, int jt_gateup,
                  int jt_down) {
    extern __shared__ int32_t sm[];
    __shared__ int s_nact;
    int32_t* cnt = sm;                          // [kBucketWarps][E]
    int32_t* total = sm + kBucketWarps * E;     // [E]
    int32_t* off_s = total + E;                 // [E + 1]
    int32_t* best = off_s + E + 1;              // [E] lowest rank of each expert (route-tail skip, R > 0)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_pairs = T * k;
    const int ppw = ((n_pairs + kBucketWarps - 1) / kBucketWarps + 31) & ~31;
    const int p_begin = min(n_pairs, warp * ppw), p_end = min(n_pairs, p_begin + ppw);
    const uint32_t lt = (1u << lane) - 1u;

    for (int i = threadIdx.x; i < kBucketWarps * E; i += blockDim.x) cnt[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) best[e] = k;
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
            if (R > 0 && valid) atomicMin(&best[e], (p0 + 32 * u + lane) % k);
        }
    }
    __syncthreads();

    // phase 2: per-expert prefix over warps, totals; an expert that no token
    // ranks before R (route-tail skip) gets no group
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kBucketWarps; ++w) {
            int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
        total[e] = ((R > 0 && best[e] >= R) || e < e0 || e >= e1) ? 0 : run;
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
            s_nact = nact;
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
            const bool valid = live && e >= 0 && e < E && !(R > 0 && best[e] >= R) && e >= e0 && e < e1;
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

    // the expert GEMMs' tile list from the groups (active was written by warp 0
    // before the barrier above; the builder synchronises the CTA first)
    if (desc_gu) {
        __shared__ TileListSmem tl;
        build_tile_list(T, k, E, n_shared, s_nact, off_s, active, jt_gateup, jt_down, desc_gu, desc_dn, tile_counts,
                        tl);
    }
}

// ---------------------------------------------------------------- multi-CTA variant (large T)
// The single-CTA kernel issues every scattered store of `pairs` (and of the
// sorted weights) from one SM, which bounds it at large T.  Three kernels
// spread the work over kChunks CTAs while keeping the same stable order:
//   count:   CTA c counts the experts of its contiguous pair range -> cnt[c][e]
//   scan:    one CTA turns cnt into per-(chunk, expert) bases, the expert
//            offsets, the active list and the meta block
//   scatter: CTA c ranks its pairs (per-warp counts in shared memory, lanes by
//            match-any, as in the single-CTA kernel) and writes them at
//            base[c][e] + rank.
constexpr int kChunks = 128;
constexpr int kScanCols = 256;  // experts per shared-memory tile of the scan (kChunks x 256 x 4 B = 128 KB)
constexpr int kScanThreads = 1024;
constexpr int kScanLoads = kChunks * kScanCols / kScanThreads;
constexpr int kChunkWarps = 8;

__global__ void __launch_bounds__(kChunkWarps * 32)
    bucket_count_kernel(const int32_t* __restrict__ ids, int n_pairs, int k, int E, int chunk,
                        int32_t* __restrict__ cnt, int32_t* __restrict__ best, int R, uint32_t* __restrict__ status) {
    extern __shared__ int32_t h[];  // [E] counts | [E] lowest rank (R > 0)
    int32_t* hb = h + E;
    const int c = blockIdx.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        h[e] = 0;
        if (R > 0) hb[e] = k;
    }
    __syncthreads();
    const int p0 = c * chunk, p1 = min(n_pairs, p0 + chunk);
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int e = __ldg(&ids[p]);
        if (e >= 0 && e < E) {
            atomicAdd(&h[e], 1);
            if (R > 0) atomicMin(&hb[e], p % k);
        } else {
            flag_status(status, kStatusBounds);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        cnt[(int64_t)c * E + e] = h[e];
        if (R > 0) best[(int64_t)c * E + e] = hb[e];
    }
}

__global__ void __launch_bounds__(kScanThreads) bucket_scan_kernel(int32_t* __restrict__ cnt, int32_t* __restrict__ best,
                                                           int R, int e0, int e1, int nchunks, int E,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ active, Meta* __restrict__ meta) {
    extern __shared__ int32_t sm_scan[];
    int32_t* tot = sm_scan;                       // [E]
    int32_t* tile = sm_scan + ((E + 31) & ~31);   // [nchunks][kScanCols] column tile of cnt
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // per expert: exclusive prefix over the chunks (in place), total; with
    // R > 0, the lowest rank over the chunks goes to best[e] (row 0) and an
    // expert with none below R gets no group.  The counts are staged in
    // column tiles of kScanCols experts (coalesced row loads and stores), and
    // a thread scans one expert's column in shared memory.
    for (int c0 = 0; c0 < E; c0 += kScanCols) {
        const int ncol = min(kScanCols, E - c0);
        {
            // every load of the tile in flight at once (1024 threads x 32 values)
            int v[kScanLoads];
#pragma unroll
            for (int j = 0; j < kScanLoads; ++j) {
                const int idx = threadIdx.x + j * kScanThreads, c = idx / kScanCols, ee = idx - c * kScanCols;
                v[j] = (c < nchunks && ee < ncol) ? cnt[(int64_t)c * E + c0 + ee] : 0;
            }
#pragma unroll
            for (int j = 0; j < kScanLoads; ++j) tile[threadIdx.x + j * kScanThreads] = v[j];
        }
        __syncthreads();
        for (int ee = threadIdx.x; ee < ncol; ee += blockDim.x) {
            const int e = c0 + ee;
            int run = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int v = tile[c * kScanCols + ee];
                tile[c * kScanCols + ee] = run;
                run += v;
            }
            if (R > 0) {
                int b = best[e];
                for (int c = 1; c < nchunks; ++c) b = min(b, best[(int64_t)c * E + e]);
                best[e] = b;
                if (b >= R) run = 0;
            }
            if (e < e0 || e >= e1) run = 0;
            tot[e] = run;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < nchunks * kScanCols; idx += blockDim.x) {
            const int c = idx / kScanCols, ee = idx - c * kScanCols;
            if (ee < ncol) cnt[(int64_t)c * E + c0 + ee] = tile[idx];
        }
        __syncthreads();  // the tile is refilled next
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0, nact = 0, mx = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int cv = e < E ? tot[e] : 0;
            int inc = cv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (e < E) offsets[e] = base + inc - cv;
            const unsigned b = __ballot_sync(0xffffffffu, cv > 0);
            if (cv > 0) active[nact + __popc(b & ((1u << lane) - 1u))] = e;
            nact += __popc(b);
            int m = cv;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            mx = max(mx, m);
            base += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            offsets[E] = base;
            meta->n_active = nact;
            meta->max_count = mx;
        }
    }
}

__global__ void __launch_bounds__(kChunkWarps * 32)
    bucket_scatter_kernel(const int32_t* __restrict__ ids, int n_pairs, int E, int chunk,
                          const int32_t* __restrict__ cbase, const int32_t* __restrict__ offsets,
                          int32_t* __restrict__ pairs, int32_t* __restrict__ inv, const float* __restrict__ w,
                          float* __restrict__ wsorted, const int32_t* __restrict__ best, int R, int e0, int e1) {
    extern __shared__ int32_t wc[];  // [kChunkWarps][E] per-warp running position
    const int c = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const int p0 = c * chunk, p1 = min(n_pairs, p0 + chunk);
    const int wchunk = ((chunk + kChunkWarps - 1) / kChunkWarps + 31) & ~31;
    const int q0 = min(p1, p0 + warp * wchunk), q1 = min(p1, q0 + wchunk);
    for (int i = threadIdx.x; i < kChunkWarps * E; i += blockDim.x) wc[i] = 0;
    __syncthreads();
    // per-warp counts of this warp's sub-range
    for (int p = q0; p < q1; p += 32) {
        const int e = p + lane < q1 ? __ldg(&ids[p + lane]) : -1;
        const bool valid = e >= e0 && e < e1 && e < E && !(R > 0 && best[e] >= R);
        const uint32_t same = __match_any_sync(0xffffffffu, valid ? e : -1);
        if (valid && (same & lt) == 0) wc[warp * E + e] += __popc(same);
    }
    __syncthreads();
    // exclusive prefix over the warps, plus this chunk's base and the expert offset
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = offsets[e] + cbase[(int64_t)c * E + e];
#pragma unroll
        for (int wv = 0; wv < kChunkWarps; ++wv) {
            const int v = wc[wv * E + e];
            wc[wv * E + e] = run;
            run += v;
        }
    }
    __syncthreads();
    for (int p = q0; p < q1; p += 32) {
        const bool live = p + lane < q1;
        const int e = live ? __ldg(&ids[p + lane]) : -1;
        const bool valid = e >= e0 && e < e1 && e < E && !(R > 0 && best[e] >= R);
        const uint32_t same = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int leader = __ffs(same) - 1;
        int base = 0;
        if (valid && lane == leader) {
            base = wc[warp * E + e];
            wc[warp * E + e] += __popc(same);
        }
        base = __shfl_sync(0xffffffffu, base, leader);
        if (valid) {
            const int pos = base + __popc(same & lt);
            pairs[pos] = p + lane;
            inv[p + lane] = pos;
            if (wsorted) wsorted[pos] = __ldg(&w[p + lane]);
        } else if (live) {
            inv[p + lane] = -1;
        }
    }
}

cudaError_t launch_bucket(const BucketArgs& a, cudaStream_t s) {
    const int n_pairs = a.T * a.k;
    const int R = a.skip_rank > 0 && a.skip_rank < a.k ? a.skip_rank : 0;
    const int e0 = max(0, a.e_begin), e1 = min(a.E, a.e_end);
    if (bucket_kernel_count(a) == 3) {
        const int chunk = (n_pairs + kChunks - 1) / kChunks;
        int32_t* best = a.cnt + (size_t)kChunks * a.E;
        bucket_count_kernel<<<kChunks, kChunkWarps * 32, 2 * sizeof(int32_t) * a.E, s>>>(a.ids, n_pairs, a.k, a.E,
                                                                                         chunk, a.cnt, best, R,
                                                                                         a.status);
        const size_t scan_smem = sizeof(int32_t) * (((size_t)a.E + 31) / 32 * 32 + (size_t)kChunks * kScanCols);
        cudaError_t es = cudaFuncSetAttribute(bucket_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)scan_smem);
        if (es != cudaSuccess) return es;
        bucket_scan_kernel<<<1, kScanThreads, scan_smem, s>>>(a.cnt, best, R, e0, e1, kChunks, a.E, a.offsets, a.active,
                                                       a.meta);
        const size_t smem = sizeof(int32_t) * (size_t)kChunkWarps * a.E;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(bucket_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
        }
        bucket_scatter_kernel<<<kChunks, kChunkWarps * 32, smem, s>>>(a.ids, n_pairs, a.E, chunk, a.cnt, a.offsets,
                                                                      a.pairs, a.inv, a.w, a.wsorted, best, R, e0, e1);
        return cudaGetLastError();
    }
    const size_t smem = sizeof(int32_t) * ((size_t)kBucketWarps * a.E + 3 * (size_t)a.E + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    if (a.desc_gu && a.n_shared + a.E > kTileMaxSlots) return cudaErrorInvalidValue;
    bucket_kernel<<<1, kBucketWarps * 32, smem, s>>>(a.ids, a.T, a.k, a.E, a.offsets, a.pairs, a.inv, a.active,
                                                     a.meta, a.status, a.w, a.wsorted, R, e0, e1, a.desc_gu,
                                                     a.desc_dn, a.tile_counts, a.n_shared, a.jt_gateup, a.jt_down);
    return cudaGetLastError();
}

}  // namespace moe

namespace moe {
size_t bucket_scratch_words(int E) { return 2 * (size_t)kChunks * E; }
int bucket_kernel_count(const BucketArgs& a) { return (a.cnt && a.T * a.k >= 8192) ? 3 : 1; }
bool bucket_builds_tiles(const BucketArgs& a) { return bucket_kernel_count(a) == 1; }
}  // namespace moe

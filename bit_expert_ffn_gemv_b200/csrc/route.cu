// route.cu -- router logits, certified top-k selection and renormalisation.
//
// The router the Strata pages place on the GPU (discuss.pytorch.kr post,
// section "Strata's operating principle": the GPU runs the router and writes
// the numbers of the 10 selected experts), with the formulas of the tiny-layer
// workload definition: logits l = W_r x + bias, softmax over the E experts,
// top-k with ties to the lower index, weights renormalised over the k chosen.
//
// Exact selection.  Logits are accumulated in fp32 from exact bf16 x bf16
// products; every logit carries the bound |l32 - l| <= delta_e with
//   delta_e = 2 * D * 2^-24 * (||W_r,e||_2 ||x||_2 + |bias_e|)
// (D = longest chain of fp32 roundings in the logits kernel).  When the fp32
// order of the top k+1 is not certified by these intervals, the token's
// candidate experts (those whose interval reaches the k-th one's) are re-ranked
// from fp64 logits, whose sums of bf16 products are exact in practice, so the
// result is the exact ranking.
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------- logits (CUDA cores)
// One warp per expert row, tokens in chunks of 4 held in shared memory as
// fp32.  Each lane accumulates d/32 products serially, then a 5-level shuffle
// tree, then the bias: D = d/32 + 6.
constexpr int kLogitTok = 4;

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ x, int T, int d,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const float* __restrict__ bias, int E,
                                                            float* __restrict__ logits) {
    extern __shared__ float xs[];  // [kLogitTok][d]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int t0 = 0; t0 < T; t0 += kLogitTok) {
        const int nt = min(kLogitTok, T - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < kLogitTok * d; i += blockDim.x) {
            int tt = i / d;
            xs[i] = tt < nt ? __bfloat162float(x[(int64_t)(t0 + tt) * d + (i - tt * d)]) : 0.0f;
        }
        __syncthreads();
        for (int e = blockIdx.x * nwarps + warp; e < E; e += gridDim.x * nwarps) {
            const __nv_bfloat16* row = wr + (int64_t)e * d;
            float acc[kLogitTok] = {0.f, 0.f, 0.f, 0.f};
            for (int i = lane * 8; i < d; i += 256) {
                uint4 v = __ldg(reinterpret_cast<const uint4*>(row + i));
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float w0 = __uint_as_float(wv[q] << 16), w1 = __uint_as_float(wv[q] & 0xFFFF0000u);
#pragma unroll
                    for (int tt = 0; tt < kLogitTok; ++tt) {
                        acc[tt] = fmaf(w0, xs[tt * d + i + 2 * q], acc[tt]);
                        acc[tt] = fmaf(w1, xs[tt * d + i + 2 * q + 1], acc[tt]);
                    }
                }
            }
#pragma unroll
            for (int tt = 0; tt < kLogitTok; ++tt) {
                float v = acc[tt];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && tt < nt) logits[(int64_t)(t0 + tt) * E + e] = v + (bias ? bias[e] : 0.0f);
            }
        }
    }
}

// ---------------------------------------------------------------- row norms
__global__ void router_norms_kernel(const __nv_bfloat16* __restrict__ wr, int E, int d, float* __restrict__ out) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= E) return;
    double acc = 0.0;
    for (int i = lane; i < d; i += 32) {
        double v = (double)__bfloat162float(wr[(int64_t)warp * d + i]);
        acc += v * v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    // round up so the bound stays a bound
    if (lane == 0) out[warp] = __double2float_ru(sqrt(acc) * (1.0 + 1e-12));
}

// ---------------------------------------------------------------- top-k
// (value desc, index asc) with NaN ranked as -inf
MOE_DEV bool better(float va, int ia, float vb, int ib) {
    va = isnan(va) ? -INFINITY : va;
    vb = isnan(vb) ? -INFINITY : vb;
    return va > vb || (va == vb && ia < ib);
}
MOE_DEV bool better64(double va, int ia, double vb, int ib) {
    va = isnan(va) ? -INFINITY : va;
    vb = isnan(vb) ? -INFINITY : vb;
    return va > vb || (va == vb && ia < ib);
}

constexpr int kTopkWarps = 4;
// Batches of up to this many tokens take a CTA of kTopkWideWarps warps per
// token (the GPU is otherwise mostly idle there): every warp selects the same
// k redundantly, and the fp64 candidate logits are split over the warps.
constexpr int kTopkWideWarps = 8;
constexpr int kTopkWideMaxT = 256;

// order-preserving image of an fp32 logit (NaN as -inf): a larger key is a
// larger value; 0 is below every key
MOE_DEV uint32_t fkey(float v) {
    v = isnan(v) ? -INFINITY : v;
    v = v + 0.0f;  // -0 -> +0
    const uint32_t b = __float_as_uint(v);
    return (b >> 31) ? ~b : (b | 0x80000000u);
}

// One warp per token (WIDE: one CTA per token, see kTopkWideWarps).  Shared
// memory per warp: E doubles (fp64 logits of the candidates), E floats (fp32
// logits), E floats (their error bounds, later the candidate list).
//
// Every fp32 logit l_e lies within d_e of the exact one.  k rounds of a warp
// max-reduction over the logits' keys select S, the k largest fp32 logits (in
// descending order; equal values in any order).  Every expert of S is then
// at least L = min over S of (l_s - d_s) exactly, so an expert whose interval
// ends below L has k experts above it: the exact top k lies within the
// candidates {e : l_e + d_e >= L}.  When the candidates are S itself and the
// intervals of consecutive ranks are disjoint, S in its fp32 order is the
// exact selection; otherwise the candidates' logits are recomputed in fp64
// (sums of exact bf16 products) and ranked exactly by (value desc, index asc).
template <int KPL, bool WIDE>
__global__ void __launch_bounds__((WIDE ? kTopkWideWarps : kTopkWarps) * 32)
    topk_kernel(const float* __restrict__ logits, const __nv_bfloat16* __restrict__ x, int T, int d, int E, int k,
                const __nv_bfloat16* __restrict__ wr, const float* __restrict__ bias,
                const float* __restrict__ wnorm, float depth, int32_t* __restrict__ ids_out,
                float* __restrict__ w_out, Meta* __restrict__ meta) {
    constexpr int NW = WIDE ? kTopkWideWarps : kTopkWarps;
    extern __shared__ unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = WIDE ? (int)blockIdx.x : (int)blockIdx.x * kTopkWarps + warp;
    double* lg64 = reinterpret_cast<double*>(smem_raw) + (size_t)warp * E;
    double* lg64_out = WIDE ? reinterpret_cast<double*>(smem_raw) : lg64;  // WIDE: warp 0's, shared by all
    float* lv = reinterpret_cast<float*>(smem_raw + sizeof(double) * (size_t)NW * E) + (size_t)warp * 2 * E;
    float* dv = lv + E;
    if (t >= T) return;  // WIDE: never (one CTA per token)

    // ||x_t||_2 (fp32, inflated to stay an upper bound); 8 values per lane per 256
    const __nv_bfloat16* xt = x + (int64_t)t * d;
    float ss = 0.f;
#pragma unroll 4
    for (int i = lane * 8; i < d; i += 256) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xt + i));
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
    const float xn = sqrtf(ss) * (1.0f + 1e-5f);
    const float c = 2.0f * depth * 5.9604645e-8f * (1.0f + 1e-5f);

    // logits, bounds and keys; lane holds experts lane + 32 j
    uint32_t key[KPL];
    uint32_t lmax = 0u;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const int e = lane + 32 * j;
        key[j] = 0u;
        if (e < E) {
            const float v = __ldg(&logits[(int64_t)t * E + e]);
            const float wn = __ldg(&wnorm[e]), b = bias ? fabsf(__ldg(&bias[e])) : 0.0f;
            lv[e] = v;
            dv[e] = c * (wn * xn + b);
            key[j] = fkey(v);
        }
        lmax = max(lmax, key[j]);
    }
    __syncwarp();

    // S: k rounds, each taking the largest remaining key (the lowest lane that
    // holds it, its first copy) -- lane r keeps rank r
    int my_sel = -1;
    float my_l = 0.f, my_d = 0.f, lo_min = INFINITY;
    bool nan_seen = false;
    for (int r = 0; r < k; ++r) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, lmax);
        const int owner = __ffs(__ballot_sync(0xffffffffu, lmax == m)) - 1;
        int er = 0;
        if (lane == owner) {
            bool done = false;
#pragma unroll
            for (int j = 0; j < KPL; ++j) {
                if (!done && key[j] == m) {
                    er = lane + 32 * j;
                    key[j] = 0u;
                    done = true;
                }
            }
            lmax = 0u;
#pragma unroll
            for (int j = 0; j < KPL; ++j) lmax = max(lmax, key[j]);
        }
        er = __shfl_sync(0xffffffffu, er, owner);
        const float lr = lv[er], dr = dv[er];
        if (lane == r) {
            my_sel = er;
            my_l = lr;
            my_d = dr;
        }
        nan_seen |= isnan(lr);
        lo_min = fminf(lo_min, lr - dr);
    }

    // certification: consecutive ranks' intervals disjoint and no other candidate
    const float nl = __shfl_down_sync(0xffffffffu, my_l, 1), nd = __shfl_down_sync(0xffffffffu, my_d, 1);
    const bool pair_ok = lane + 1 >= k || (my_l - my_d > nl + nd);
    bool ok = __all_sync(0xffffffffu, pair_ok) && !nan_seen && !isnan(lo_min);
    int* cand = reinterpret_cast<int*>(dv);  // the bounds are no longer needed after this pass
    int n_cand = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const bool is_c = e < E && (nan_seen || isnan(lv[e]) || lv[e] + dv[e] >= lo_min);
        const uint32_t bm = __ballot_sync(0xffffffffu, is_c);
        __syncwarp();  // every lane has read dv[e0 .. e0+31] before it is overwritten
        if (is_c) cand[n_cand + __popc(bm & ((1u << lane) - 1u))] = e;
        n_cand += __popc(bm);
    }
    __syncwarp();
    if (n_cand != k) ok = false;

    float my_w = 0.f;  // lane r < k: logit of rank r
    if (ok) {
        if (lane < k) my_w = my_l;
    } else {
        // fp64 logits of the candidates (sums of exact bf16 products), 8 products
        // per lane per 256-wide chunk, four candidates per pass (more loads in
        // flight); WIDE: the passes are dealt over the CTA's warps, which hold
        // the same candidate list
        for (int ci = WIDE ? 4 * warp : 0; ci < n_cand; ci += WIDE ? 4 * kTopkWideWarps : 4) {
            int ec[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) ec[u] = cand[min(ci + u, n_cand - 1)];
            double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 2
            for (int i = lane * 8; i < d; i += 256) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xt + i));
                uint4 wv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) wv[u] = __ldg(reinterpret_cast<const uint4*>(wr + (int64_t)ec[u] * d + i));
                const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const double xl = (double)__uint_as_float(xu[q] << 16);
                    const double xh = (double)__uint_as_float(xu[q] & 0xFFFF0000u);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t wq = q == 0 ? wv[u].x : q == 1 ? wv[u].y : q == 2 ? wv[u].z : wv[u].w;
                        acc[u] = fma((double)__uint_as_float(wq << 16), xl, acc[u]);
                        acc[u] = fma((double)__uint_as_float(wq & 0xFFFF0000u), xh, acc[u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
            if (lane == 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (ci + u < n_cand) lg64_out[ci + u] = acc[u] + (bias ? (double)bias[ec[u]] : 0.0);
            }
        }
        if (WIDE) {
            __syncthreads();  // every warp took the same branch: the certificate is computed alike
            if (warp != 0) return;
        }
        __syncwarp();
        if (n_cand <= 32) {
            // exact rank of each candidate (lane c): how many candidates beat it
            double v = -INFINITY;
            int e = 0x7fffffff;
            if (lane < n_cand) {
                v = lg64[lane];
                e = cand[lane];
            }
            int rank = 0;
            for (int j = 0; j < n_cand; ++j) {
                const double vj = __shfl_sync(0xffffffffu, v, j);
                const int ej = __shfl_sync(0xffffffffu, e, j);
                if (j != lane && better64(vj, ej, v, e)) ++rank;
            }
            for (int r = 0; r < k; ++r) {
                const int src = __ffs(__ballot_sync(0xffffffffu, lane < n_cand && rank == r)) - 1;
                const double vr = __shfl_sync(0xffffffffu, v, src);
                const int er = __shfl_sync(0xffffffffu, e, src);
                if (lane == r) {
                    my_sel = er;
                    my_w = (float)vr;
                }
            }
        } else {
            // many candidates (ties or NaN): k rounds of warp argmax on (fp64 logit, index)
            uint32_t tk = 0;  // bit j <-> candidate lane + 32 j (n_cand <= E <= 1024, so j < 32)
            for (int r = 0; r < k; ++r) {
                double bv = -INFINITY;
                int bi = 0x7fffffff, bc = -1;
                for (int j = 0, ci = lane; ci < n_cand; ++j, ci += 32) {
                    if (!((tk >> j) & 1u) && (bi == 0x7fffffff || better64(lg64[ci], cand[ci], bv, bi))) {
                        bv = lg64[ci];
                        bi = cand[ci];
                        bc = ci;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    double ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    int oc = __shfl_xor_sync(0xffffffffu, bc, o);
                    if (oi != 0x7fffffff && (bi == 0x7fffffff || better64(ov, oi, bv, bi))) {
                        bv = ov;
                        bi = oi;
                        bc = oc;
                    }
                }
                if (lane == r) {
                    my_sel = bi;
                    my_w = (float)bv;
                }
                if (bc >= 0 && (bc & 31) == lane) tk |= 1u << (bc >> 5);
            }
        }
        if (lane == 0) atomicAdd(&meta->n_fixup, 1);
    }

    if (WIDE && warp != 0) return;  // warp 0 writes the token's result
    // renormalised weights = softmax over the k selected logits (lane r: rank r)
    const float m = __shfl_sync(0xffffffffu, my_w, 0);
    const float ex = lane < k ? expf(my_w - m) : 0.0f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane < k) {
        ids_out[(int64_t)t * k + lane] = my_sel;
        w_out[(int64_t)t * k + lane] = ex * (1.0f / z);
    }
}

// ---------------------------------------------------------------- launchers
cudaError_t launch_router_norms(const void* wr, int E, int d, float* out, cudaStream_t s) {
    router_norms_kernel<<<(E * 32 + 255) / 256, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(wr), E, d, out);
    return cudaGetLastError();
}

cudaError_t launch_router_logits(const RouteArgs& a, cudaStream_t s) {
    const size_t smem_l = sizeof(float) * kLogitTok * a.d;
    if (smem_l > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_l);
        if (e != cudaSuccess) return e;
    }
    int grid = (a.E + 7) / 8;
    router_logits_kernel<<<grid, 256, smem_l, s>>>(static_cast<const __nv_bfloat16*>(a.x), a.T, a.d,
                                                  static_cast<const __nv_bfloat16*>(a.wr), a.bias, a.E, a.logits);
    return cudaGetLastError();
}

cudaError_t launch_topk(const RouteArgs& a, cudaStream_t s) {
    if (a.E > 1024 || a.logit_parts != 1) return cudaErrorInvalidValue;  // reads reduced logits
    const bool wide = a.T <= kTopkWideMaxT;
    const int nw = wide ? kTopkWideWarps : kTopkWarps;
    const size_t smem_t = (size_t)nw * a.E * (sizeof(double) + 2 * sizeof(float));
    auto kern = wide ? (a.E <= 512 ? topk_kernel<16, true> : topk_kernel<32, true>)
                     : (a.E <= 512 ? topk_kernel<16, false> : topk_kernel<32, false>);
    if (smem_t > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_t);
        if (e != cudaSuccess) return e;
    }
    const float depth = a.depth > 0.f ? a.depth : (float)(a.d / 32 + 6);
    const int grid = wide ? a.T : (a.T + kTopkWarps - 1) / kTopkWarps;
    kern<<<grid, nw * 32, smem_t, s>>>(a.logits, static_cast<const __nv_bfloat16*>(a.x), a.T, a.d, a.E, a.k,
                                      static_cast<const __nv_bfloat16*>(a.wr), a.bias, a.wnorm, depth, a.ids, a.w,
                                      a.meta);
    return cudaGetLastError();
}

}  // namespace moe

// gemv.cu -- grouped expert GEMV for small token counts (decode / MTP verify).
//
// The expert FFN of the layer (expert = W_d (silu(W_g x) * W_u x) on block-
// quantised weights, What = q * s, s one fp16 scale per 32 weights along the
// input dimension) for each expert's group of tokens.  Work item = (expert
// slot, 16-row tile); the 8 warps of a CTA split the input dimension into
// 128-wide super-tiles.  Each lane loads exactly the code words and scales of
// its A-fragment registers (the packed layout is built for that), turns codes
// into exact 16-bit integers q with one OR and one subtract per pair, and a
// 16x8x16 warp MMA accumulates q * x for one 32-weight block in fp32; the
// block's scale is applied to that partial afterwards (fp32 FMA).  Gate/up
// use bf16 operands (x is bf16, q is exact in bf16); down uses fp16 (h is
// held in fp16).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kGemvWarps = 8;

struct SlotInfo {
    int expert;   // expert index (E = shared)
    int count;    // tokens in the group
    int hbase;    // first row of the group in h / obuf
    bool shared;
    int pair0;    // first index into `pairs` (routed groups)
};

MOE_DEV bool slot_info(const ExpertArgs& a, int slot, SlotInfo& s) {
    if (slot < a.n_shared) {
        s.expert = a.E;
        s.count = a.T;
        s.hbase = a.T * a.k;
        s.shared = true;
        s.pair0 = 0;
        return true;
    }
    const int idx = slot - a.n_shared;
    if (idx >= a.meta->n_active) return false;
    const int e = a.active[idx];
    s.expert = e;
    s.pair0 = a.offsets[e];
    s.count = a.offsets[e + 1] - s.pair0;
    s.hbase = s.pair0;
    s.shared = false;
    return true;
}

MOE_DEV int slot_token(const ExpertArgs& a, const SlotInfo& s, int i) {
    return s.shared ? i : a.pairs[s.pair0 + i] / a.k;
}

MOE_DEV float half_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
MOE_DEV float half_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

// acc += s * tmp with the C-fragment row split (rows g: [0],[1]; rows g+8: [2],[3])
MOE_DEV void scale_acc(float (&acc)[4], const float (&tmp)[4], uint32_t sc) {
    const float slo = half_lo(sc), shi = half_hi(sc);
    acc[0] = fmaf(slo, tmp[0], acc[0]);
    acc[1] = fmaf(slo, tmp[1], acc[1]);
    acc[2] = fmaf(shi, tmp[2], acc[2]);
    acc[3] = fmaf(shi, tmp[3], acc[3]);
}

// ---------------------------------------------------------------- gate/up + SwiGLU
template <int BITS, int NT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_gateup_kernel(const ExpertArgs a) {
    extern __shared__ float red[];  // [kGemvWarps][2][NT][4][32]
    SlotInfo s;
    if (!slot_info(a, blockIdx.x, s)) return;
    const int jt = blockIdx.y;  // 16-row tile of f
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KT = a.d / 128;
    const int64_t mat_codes = (int64_t)a.f * a.d * BITS / 8, mat_scales = (int64_t)a.f * a.d / 32;
    const int64_t stride = a.code_stride ? a.code_stride : 3 * mat_codes;
    const uint8_t* cg = a.codes + (int64_t)s.expert * stride;
    const uint8_t* cu = cg + mat_codes;
    const __half* sg = reinterpret_cast<const __half*>(a.scales) + (int64_t)s.expert * 3 * mat_scales;
    const __half* su = sg + mat_scales;
    const uint16_t* x = static_cast<const uint16_t*>(a.x);
    __half* h = static_cast<__half*>(a.h);

    for (int p0 = 0; p0 < s.count; p0 += 8 * NT) {
        const int nrem = min(8 * NT, s.count - p0);
        int tok[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int i = p0 + nt * 8 + g;
            tok[nt] = (nt * 8 + g < nrem) ? slot_token(a, s, i) : -1;
        }
        float accg[NT][4], accu[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) accg[nt][i] = accu[nt][i] = 0.f;

        for (int kt = warp; kt < KT; kt += kGemvWarps) {
            const int64_t st = (int64_t)jt * KT + kt;
            TileRegs<BITS> tg, tu;
            load_tile<BITS>(cg, sg, st, lane, tg);
            load_tile<BITS>(cu, su, st, lane, tu);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                uint32_t ag[8], au[8];
                decode_block<false, BITS>(tg.lo[kb], tg.hi[kb], ag);
                decode_block<false, BITS>(tu.lo[kb], tu.hi[kb], au);
                const int k0 = kt * 128 + kb * 32 + 2 * c;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    uint32_t b[4] = {0u, 0u, 0u, 0u};
                    if (tok[nt] >= 0) {
                        const uint16_t* xr = x + (int64_t)tok[nt] * a.d + k0;
                        b[0] = __ldg(reinterpret_cast<const uint32_t*>(xr));
                        b[1] = __ldg(reinterpret_cast<const uint32_t*>(xr + 8));
                        b[2] = __ldg(reinterpret_cast<const uint32_t*>(xr + 16));
                        b[3] = __ldg(reinterpret_cast<const uint32_t*>(xr + 24));
                    }
                    const uint32_t ag0[4] = {ag[0], ag[1], ag[2], ag[3]}, ag1[4] = {ag[4], ag[5], ag[6], ag[7]};
                    const uint32_t au0[4] = {au[0], au[1], au[2], au[3]}, au1[4] = {au[4], au[5], au[6], au[7]};
                    float tg4[4] = {0.f, 0.f, 0.f, 0.f}, tu4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_bf16(tg4, ag0, b[0], b[1], tg4);
                    mma_bf16(tg4, ag1, b[2], b[3], tg4);
                    mma_bf16(tu4, au0, b[0], b[1], tu4);
                    mma_bf16(tu4, au1, b[2], b[3], tu4);
                    scale_acc(accg[nt], tg4, tg.sc[kb]);
                    scale_acc(accu[nt], tu4, tu.sc[kb]);
                }
            }
        }
        // cross-warp reduction in a fixed order, then SwiGLU
        __syncthreads();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                red[(((warp * 2 + 0) * NT + nt) * 4 + i) * 32 + lane] = accg[nt][i];
                red[(((warp * 2 + 1) * NT + nt) * 4 + i) * 32 + lane] = accu[nt][i];
            }
        __syncthreads();
        for (int id = threadIdx.x; id < NT * 4 * 32; id += blockDim.x) {
            const int ln = id & 31, i = (id >> 5) & 3, nt = id >> 7;
            const int m = (ln >> 2) + 8 * (i >> 1);
            const int n = nt * 8 + 2 * (ln & 3) + (i & 1);
            if (n >= nrem) continue;
            float gs = 0.f, us = 0.f;
            for (int w = 0; w < kGemvWarps; ++w) {
                gs += red[(((w * 2 + 0) * NT + nt) * 4 + i) * 32 + ln];
                us += red[(((w * 2 + 1) * NT + nt) * 4 + i) * 32 + ln];
            }
            const float hv = silu(gs) * us;
            h[(int64_t)(s.hbase + p0 + n) * a.f + jt * 16 + m] = __float2half_rn(hv);
        }
    }
}

// ---------------------------------------------------------------- down projection
template <int BITS, int NT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_down_kernel(const ExpertArgs a) {
    extern __shared__ float red[];  // [kGemvWarps][NT][4][32]
    SlotInfo s;
    if (!slot_info(a, blockIdx.x, s)) return;
    const int nt16 = blockIdx.y;  // 16-row tile of d
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int KT = a.f / 128;
    // BITS is the down matrices' width; gate and up (at a.bits) come first in each expert's block
    const int64_t mat_codes = (int64_t)a.f * a.d * BITS / 8, mat_scales = (int64_t)a.f * a.d / 32;
    const int64_t gu_codes = (int64_t)a.f * a.d * a.bits / 8;
    const int64_t stride = a.code_stride ? a.code_stride : 2 * gu_codes + mat_codes;
    const uint8_t* cd = a.codes + (int64_t)s.expert * stride + 2 * gu_codes;
    const __half* sd = reinterpret_cast<const __half*>(a.scales) + (int64_t)s.expert * 3 * mat_scales + 2 * mat_scales;
    const uint16_t* h = static_cast<const uint16_t*>(a.h);

    for (int p0 = 0; p0 < s.count; p0 += 8 * NT) {
        const int nrem = min(8 * NT, s.count - p0);
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
        for (int kt = warp; kt < KT; kt += kGemvWarps) {
            const int64_t st = (int64_t)nt16 * KT + kt;
            TileRegs<BITS> td;
            load_tile<BITS>(cd, sd, st, lane, td);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                uint32_t ad[8];
                decode_block<true, BITS>(td.lo[kb], td.hi[kb], ad);
                const int k0 = kt * 128 + kb * 32 + 2 * c;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    uint32_t b[4] = {0u, 0u, 0u, 0u};
                    if (nt * 8 + g < nrem) {
                        const uint16_t* hr = h + (int64_t)(s.hbase + p0 + nt * 8 + g) * a.f + k0;
                        b[0] = *reinterpret_cast<const uint32_t*>(hr);
                        b[1] = *reinterpret_cast<const uint32_t*>(hr + 8);
                        b[2] = *reinterpret_cast<const uint32_t*>(hr + 16);
                        b[3] = *reinterpret_cast<const uint32_t*>(hr + 24);
                    }
                    const uint32_t a0[4] = {ad[0], ad[1], ad[2], ad[3]}, a1[4] = {ad[4], ad[5], ad[6], ad[7]};
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(t4, a0, b[0], b[1], t4);
                    mma_f16(t4, a1, b[2], b[3], t4);
                    scale_acc(acc[nt], t4, td.sc[kb]);
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) red[((warp * NT + nt) * 4 + i) * 32 + lane] = acc[nt][i];
        __syncthreads();
        for (int id = threadIdx.x; id < NT * 4 * 32; id += blockDim.x) {
            const int ln = id & 31, i = (id >> 5) & 3, nt = id >> 7;
            const int m = (ln >> 2) + 8 * (i >> 1);
            const int n = nt * 8 + 2 * (ln & 3) + (i & 1);
            if (n >= nrem) continue;
            float o = 0.f;
            for (int w = 0; w < kGemvWarps; ++w) o += red[((w * NT + nt) * 4 + i) * 32 + ln];
            a.obuf[(int64_t)(s.hbase + p0 + n) * a.d + nt16 * 16 + m] = o;
        }
    }
}

// ---------------------------------------------------------------- launchers
template <int BITS, int NT>
static cudaError_t gateup_bits_nt(const ExpertArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * kGemvWarps * 2 * NT * 4 * 32;
    auto kern = gemv_gateup_kernel<BITS, NT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(a.n_shared + min(a.T * a.k, a.E), a.f / 16);
    kern<<<grid, kGemvWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int BITS, int NT>
static cudaError_t down_bits_nt(const ExpertArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * kGemvWarps * NT * 4 * 32;
    auto kern = gemv_down_kernel<BITS, NT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(a.n_shared + min(a.T * a.k, a.E), a.d / 16);
    kern<<<grid, kGemvWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}

template <int BITS>
static cudaError_t gateup_bits(const ExpertArgs& a, cudaStream_t s) {
    if (a.T <= 8) return gateup_bits_nt<BITS, 1>(a, s);
    if (a.T <= 16) return gateup_bits_nt<BITS, 2>(a, s);
    if (a.T <= 32) return gateup_bits_nt<BITS, 4>(a, s);
    return gateup_bits_nt<BITS, 8>(a, s);
}

template <int BITS>
static cudaError_t down_bits(const ExpertArgs& a, cudaStream_t s) {
    if (a.T <= 8) return down_bits_nt<BITS, 1>(a, s);
    if (a.T <= 16) return down_bits_nt<BITS, 2>(a, s);
    if (a.T <= 32) return down_bits_nt<BITS, 4>(a, s);
    return down_bits_nt<BITS, 8>(a, s);
}

cudaError_t launch_gemv_gateup(const ExpertArgs& a, cudaStream_t s) {
    switch (a.bits) {
        case 2: return gateup_bits<2>(a, s);
        case 3: return gateup_bits<3>(a, s);
        case 4: return gateup_bits<4>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemv_down(const ExpertArgs& a, cudaStream_t s) {
    switch (a.bits_down ? a.bits_down : a.bits) {
        case 2: return down_bits<2>(a, s);
        case 3: return down_bits<3>(a, s);
        case 4: return down_bits<4>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------- combine
// y[t] = o_shared[t] + sum_r w[t,r] o[t,r]  (then optionally + y_in), fixed order
__global__ void combine_kernel(const CombineArgs a) {
    const int t = blockIdx.y;
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (n >= a.d) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.n_shared) acc = *reinterpret_cast<const float4*>(a.obuf + ((int64_t)a.T * a.k + t) * a.d + n);
    for (int r = 0; r < a.k; ++r) {
        const int pos = a.inv[(int64_t)t * a.k + r];
        if (pos < 0) continue;
        const float w = a.w[(int64_t)t * a.k + r];
        const float4 o = *reinterpret_cast<const float4*>(a.obuf + (int64_t)pos * a.d + n);
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
    }
    if (a.out_fp32) {
        float4* y = reinterpret_cast<float4*>(static_cast<float*>(a.y) + (int64_t)t * a.d + n);
        if (a.accumulate) {
            float4 v = *y;
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        *y = acc;
    } else {
        __nv_bfloat162* y = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.y) + (int64_t)t * a.d + n);
        if (a.accumulate) {
            float2 v0 = __bfloat1622float2(y[0]), v1 = __bfloat1622float2(y[1]);
            acc.x += v0.x;
            acc.y += v0.y;
            acc.z += v1.x;
            acc.w += v1.y;
        }
        y[0] = __floats2bfloat162_rn(acc.x, acc.y);
        y[1] = __floats2bfloat162_rn(acc.z, acc.w);
    }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    dim3 grid((a.d / 4 + 127) / 128, a.T);
    combine_kernel<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- debug dequant
template <int BITS>
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const __half* __restrict__ scales, int N, int K,
                               float* __restrict__ out) {
    const int KT = K / 128;
    const int64_t n_st = (int64_t)(N / 16) * KT;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= n_st) return;
    const int R = (int)(gw / KT), C = (int)(gw % KT);
    const int g = lane >> 2, c = lane & 3;
    TileRegs<BITS> t;
    load_tile<BITS>(codes, scales, gw, lane, t);
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
        uint32_t q[8];
        decode_block<true, BITS>(t.lo[kb], t.hi[kb], q);
        const float slo = half_lo(t.sc[kb]), shi = half_hi(t.sc[kb]);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int ks = p >> 2, reg = p & 3, half = reg & 1, hi8 = reg >> 1;
            const int row = 16 * R + g + 8 * half;
            const int col = 128 * C + 32 * kb + 16 * ks + 8 * hi8 + 2 * c;
            const float sv = half ? shi : slo;
            const float q0 = __half2float(__ushort_as_half((unsigned short)(q[p] & 0xFFFFu)));
            const float q1 = __half2float(__ushort_as_half((unsigned short)(q[p] >> 16)));
            out[(int64_t)row * K + col] = q0 * sv;
            out[(int64_t)row * K + col + 1] = q1 * sv;
        }
    }
}

cudaError_t launch_dequant(const uint8_t* codes, const uint16_t* scales, int N, int K, int bits, float* out,
                           cudaStream_t s) {
    const int64_t warps = (int64_t)(N / 16) * (K / 128);
    const int64_t blocks = (warps * 32 + 255) / 256;
    const __half* sc = reinterpret_cast<const __half*>(scales);
    switch (bits) {
        case 2: dequant_kernel<2><<<(unsigned)blocks, 256, 0, s>>>(codes, sc, N, K, out); break;
        case 3: dequant_kernel<3><<<(unsigned)blocks, 256, 0, s>>>(codes, sc, N, K, out); break;
        case 4: dequant_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(codes, sc, N, K, out); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace moe

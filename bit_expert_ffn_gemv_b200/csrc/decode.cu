// decode.cu -- the whole routed-MoE layer for up to 64 tokens in ONE persistent kernel.
//
// Decode and draft-verify batches (1 token plus up to 3 drafts; the layer the
// Strata pages run per generated token: the router picks the experts, they
// run, "the GPU combines each result, then moves to the next layer" --
// discuss.pytorch.kr post, section "Strata's operating principle") move ~18 MB
// of weights per token-layer, a few microseconds of HBM time, so separate
// launches per step would dominate.  Here one launch does everything.  CTAs
// pull tasks from a global queue in dependency order:
//   1. router rows (8 experts per CTA, fp32 logits with a rounding bound)
//   2. shared-expert gate/up tiles (no routing dependency: overlap the router)
//   3. certified top-k (8 tokens per CTA; the last one also buckets the pairs)
//   4. shared-expert down tiles
//   5. routed gate/up tiles, expert-major (expert s, 16-row tile of f)
//   6. routed down tiles (expert s, 8 x 16-row tiles of d)
// Dependencies are counters in global memory: router rows done, tokens
// ranked, bucketing published, per-expert gate/up tiles done, per
// (token, 16-row output tile) experts done.  The task that completes an output
// tile's last expert sums it in a fixed order (shared expert, then rank order),
// so the result is deterministic without atomics on data.  A task only waits
// on tasks claimed before it, so any grid size makes progress; every wait is
// bounded and, if one gives up, sets the status word and an abort flag that
// ends all other waits.  The last CTA to leave resets the counters.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kSpinLimit = 1u << 21;  // x >= 100 ns per spin: >= 0.2 s

// sync block (int32 words)
enum { SY_HEAD = 0, SY_ROUTER = 1, SY_TOPK = 2, SY_BUCKET = 3, SY_EXIT = 4, SY_ABORT = 5, SY_FIXUP = 6,
       SY_SLOTS = 16 };

MOE_DEV int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
MOE_DEV int atom_add_acqrel(int* p, int v) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
MOE_DEV void red_add_release(int* p, int v) {
    asm volatile("red.add.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
MOE_DEV void st_release(int* p, int v) { asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory"); }

// Wait until *p >= target.  False if the wait gave up (timeout or abort).
MOE_DEV bool wait_geq(const int* p, int target, int* sync, uint32_t* status) {
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire(p) >= target) return true;
        if (ld_acquire(sync + SY_ABORT)) return false;
        if (it > kSpinLimit) {
            flag_status(status, kStatusTimeout);
            st_release(sync + SY_ABORT, 1);
            return false;
        }
        __nanosleep(128);
    }
}

struct DecodeArgs {
    int T, d, f, E, k, n_shared;
    const uint16_t* x;  // bf16 [T x d]
    void* y;
    int out_fp32, accumulate;
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* wr;  // bf16 [E x d]
    const float* bias;
    const float* wnorm;
    float* logits;    // [T x E]
    double* logits64; // [T x E]
    int32_t* ids;
    float* w;
    int32_t* offsets;
    int32_t* pairs;
    int32_t* inv;
    int32_t* active;
    Meta* meta;
    uint32_t* status;
    __half* h;
    float* obuf;
    int* sync;
};

struct TaskMap {
    int nRt, nSG, nTK, nSD, nRG, nRD, RT16, nRTG, maxR, FT;
    int b1, b2, b3, b4, b5, total;
};

MOE_DEV TaskMap task_map(const DecodeArgs& a) {
    TaskMap m;
    m.nRt = (a.E + kDecWarps - 1) / kDecWarps;
    m.FT = a.f / 16;
    m.nSG = a.n_shared ? m.FT : 0;
    m.nTK = (a.T + kDecWarps - 1) / kDecWarps;
    m.RT16 = a.d / 16;
    m.nRTG = (m.RT16 + kDecWarps - 1) / kDecWarps;
    m.nSD = a.n_shared ? m.nRTG : 0;
    m.maxR = min(a.T * a.k, a.E);
    m.nRG = m.maxR * m.FT;
    m.nRD = m.maxR * m.nRTG;
    m.b1 = m.nRt;
    m.b2 = m.b1 + m.nSG;
    m.b3 = m.b2 + m.nTK;
    m.b4 = m.b3 + m.nSD;
    m.b5 = m.b4 + m.nRG;
    m.total = m.b5 + m.nRD;
    return m;
}

// slot 0 = shared expert (if any); slot n_shared + s = s-th active routed expert
struct Slot {
    int expert, count, hbase, pair0;
    bool shared;
};

MOE_DEV Slot make_slot(const DecodeArgs& a, int slot) {
    Slot s;
    if (slot < a.n_shared) {
        s.expert = a.E;
        s.count = a.T;
        s.hbase = a.T * a.k;
        s.pair0 = 0;
        s.shared = true;
    } else {
        const int e = a.active[slot - a.n_shared];
        s.expert = e;
        s.pair0 = a.offsets[e];
        s.count = a.offsets[e + 1] - s.pair0;
        s.hbase = s.pair0;
        s.shared = false;
    }
    return s;
}

MOE_DEV int slot_tok(const DecodeArgs& a, const Slot& s, int i) { return s.shared ? i : a.pairs[s.pair0 + i] / a.k; }

MOE_DEV float h_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
MOE_DEV float h_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

MOE_DEV void acc_scaled(float (&acc)[4], const float (&t)[4], uint32_t sc) {
    const float slo = h_lo(sc), shi = h_hi(sc);
    acc[0] = fmaf(slo, t[0], acc[0]);
    acc[1] = fmaf(slo, t[1], acc[1]);
    acc[2] = fmaf(shi, t[2], acc[2]);
    acc[3] = fmaf(shi, t[3], acc[3]);
}

MOE_DEV bool better32(float va, int ia, float vb, int ib) {
    va = isnan(va) ? -INFINITY : va;
    vb = isnan(vb) ? -INFINITY : vb;
    return va > vb || (va == vb && ia < ib);
}
MOE_DEV bool better64d(double va, int ia, double vb, int ib) {
    va = isnan(va) ? -INFINITY : va;
    vb = isnan(vb) ? -INFINITY : vb;
    return va > vb || (va == vb && ia < ib);
}

// ---------------------------------------------------------------- 1. router row
// logits[t][e] for all T tokens; lane covers columns lane*4 + 128 j.  Each
// lane's sum is a serial FMA chain of d/32 terms, then 5 shuffle levels, then
// the bias: at most d/32 + 6 roundings.
MOE_DEV void router_row(const DecodeArgs& a, int e, int lane) {
    const uint16_t* row = a.wr + (int64_t)e * a.d;
    const float b = a.bias ? a.bias[e] : 0.0f;
    for (int t0 = 0; t0 < a.T; t0 += 8) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int p = lane * 4; p < a.d; p += 128) {
            const uint2 wv = *reinterpret_cast<const uint2*>(row + p);
            const float w0 = __uint_as_float(wv.x << 16), w1 = __uint_as_float(wv.x & 0xFFFF0000u);
            const float w2 = __uint_as_float(wv.y << 16), w3 = __uint_as_float(wv.y & 0xFFFF0000u);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (t0 + q < a.T) {
                    const uint2 xv = *reinterpret_cast<const uint2*>(a.x + (int64_t)(t0 + q) * a.d + p);
                    acc[q] = fmaf(w0, __uint_as_float(xv.x << 16), acc[q]);
                    acc[q] = fmaf(w1, __uint_as_float(xv.x & 0xFFFF0000u), acc[q]);
                    acc[q] = fmaf(w2, __uint_as_float(xv.y << 16), acc[q]);
                    acc[q] = fmaf(w3, __uint_as_float(xv.y & 0xFFFF0000u), acc[q]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float v = acc[q];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && t0 + q < a.T) a.logits[(int64_t)(t0 + q) * a.E + e] = v + b;
        }
    }
}

// ---------------------------------------------------------------- 3. certified top-k of one token
MOE_DEV void topk_token(const DecodeArgs& a, int t, int lane, float* v) {
    const int E = a.E, k = a.k, d = a.d;
    const uint16_t* xt = a.x + (int64_t)t * d;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) {
        const float xv = __uint_as_float((uint32_t)xt[i] << 16);
        ss = fmaf(xv, xv, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float xn = sqrtf(ss) * (1.0f + 1e-5f);
    const float c = 2.0f * (float)(d / 32 + 6) * 5.9604645e-8f * (1.0f + 1e-5f);
    const float* lg = a.logits + (int64_t)t * E;
    auto bound = [&](int e) { return c * (a.wnorm[e] * xn + (a.bias ? fabsf(a.bias[e]) : 0.0f)); };
    for (int e = lane; e < E; e += 32) v[e] = lg[e];  // this warp's shared-memory copy
    __syncwarp();

    int sel[33];
    uint32_t taken = 0;
    const int kk = min(k + 1, E);
    for (int r = 0; r < kk; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int j = 0, e = lane; e < E; ++j, e += 32) {
            const float ve = v[e];
            if (!((taken >> j) & 1u) && (bi == 0x7fffffff || better32(ve, e, bv, bi))) {
                bv = ve;
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != 0x7fffffff && (bi == 0x7fffffff || better32(ov, oi, bv, bi))) {
                bv = ov;
                bi = oi;
            }
        }
        sel[r] = bi;
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    }
    bool ok = true;
    for (int r = 0; r + 1 < k; ++r) {
        const int p = sel[r], q = sel[r + 1];
        if (!(lg[p] - bound(p) > lg[q] + bound(q))) ok = false;
    }
    const float lower_k = lg[sel[k - 1]] - bound(sel[k - 1]);
    int ncand = 0;
    for (int e = lane; e < E; e += 32)
        if (!isnan(v[e]) && v[e] + bound(e) >= lower_k) ++ncand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ncand += __shfl_xor_sync(0xffffffffu, ncand, o);
    if (ncand != k || isnan(lower_k)) ok = false;

    float wsel[32];
    if (ok) {
        for (int r = 0; r < k; ++r) wsel[r] = lg[sel[r]];
    } else {
        // fp64 logits of the candidates (exact sums of bf16 products), then exact ranking
        double* l64 = a.logits64 + (int64_t)t * E;
        const uint16_t* wr = a.wr;
        for (int e = 0; e < E; ++e) {
            const float ve = lg[e];
            const bool cand = isnan(lower_k) || isnan(ve) || (ve + bound(e) >= lower_k);
            double acc = 0.0;
            if (cand) {
                for (int i = lane; i < d; i += 32)
                    acc = fma((double)__uint_as_float((uint32_t)wr[(int64_t)e * d + i] << 16),
                              (double)__uint_as_float((uint32_t)xt[i] << 16), acc);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                acc += a.bias ? (double)a.bias[e] : 0.0;
            }
            if (lane == 0) l64[e] = cand ? acc : -INFINITY;
        }
        __syncwarp();
        uint32_t tk = 0;
        for (int r = 0; r < k; ++r) {
            double bv = -INFINITY;
            int bi = 0x7fffffff;
            for (int j = 0, e = lane; e < E; ++j, e += 32) {
                const double ve = l64[e];
                if (!((tk >> j) & 1u) && (bi == 0x7fffffff || better64d(ve, e, bv, bi))) {
                    bv = ve;
                    bi = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (oi != 0x7fffffff && (bi == 0x7fffffff || better64d(ov, oi, bv, bi))) {
                    bv = ov;
                    bi = oi;
                }
            }
            sel[r] = bi;
            wsel[r] = (float)bv;
            if ((bi & 31) == lane) tk |= 1u << (bi >> 5);
        }
        if (lane == 0) atomicAdd(a.sync + SY_FIXUP, 1);
    }
    if (lane == 0) {
        const float m = wsel[0];
        float z = 0.f;
        for (int r = 0; r < k; ++r) {
            wsel[r] = expf(wsel[r] - m);
            z += wsel[r];
        }
        const float inv = 1.0f / z;
        for (int r = 0; r < k; ++r) {
            a.ids[(int64_t)t * k + r] = sel[r];
            a.w[(int64_t)t * k + r] = wsel[r] * inv;
        }
    }
}

// ---------------------------------------------------------------- bucketing (one warp)
// Counting sort of the T*k pairs by expert, stable in token order.
MOE_DEV void bucket_warp(const DecodeArgs& a, int lane, int* sm) {
    const int E = a.E, k = a.k, n = a.T * a.k;
    int* cnt = sm;          // [E]
    int* off = sm + E;      // [E + 1]
    for (int e = lane; e < E; e += 32) cnt[e] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int e = a.ids[i];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else flag_status(a.status, kStatusBounds);
    }
    __syncwarp();
    int base = 0, nact = 0, mx = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int cv = e < E ? cnt[e] : 0;
        int inc = cv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += u;
        }
        if (e < E) {
            off[e] = base + inc - cv;
            a.offsets[e] = base + inc - cv;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, cv > 0);
        if (cv > 0) a.active[nact + __popc(bal & ((1u << lane) - 1u))] = e;
        nact += __popc(bal);
        int m = cv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        mx = max(mx, m);
        base += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
        a.offsets[E] = base;
        a.meta->n_active = nact;
        a.meta->max_count = mx;
        a.meta->n_fixup = ld_acquire(a.sync + SY_FIXUP);
    }
    __syncwarp();
    for (int t = 0; t < a.T; ++t) {
        if (lane < k) {
            const int e = a.ids[(int64_t)t * k + lane];
            if (e >= 0 && e < E) {
                const int pos = off[e]++;
                a.pairs[pos] = t * k + lane;
                a.inv[(int64_t)t * k + lane] = pos;
            } else {
                a.inv[(int64_t)t * k + lane] = -1;
            }
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------- gate/up tile (CTA)
// h[hbase + i][jt*16 .. +15] = silu(g) * u for the slot's tokens i; the 8
// warps split the input dimension into 128-wide super-tiles.
template <int BITS, int NT>
MOE_DEV void gateup_tile(const DecodeArgs& a, const Slot& s, int jt, float* red, int warp, int lane) {
    const int g = lane >> 2, c = lane & 3;
    const int KT = a.d / 128;
    const int64_t mc = (int64_t)a.f * a.d * BITS / 8, ms = (int64_t)a.f * a.d / 32;
    const uint8_t* cg = a.codes + (int64_t)s.expert * 3 * mc;
    const uint8_t* cu = cg + mc;
    const __half* sg = reinterpret_cast<const __half*>(a.scales) + (int64_t)s.expert * 3 * ms;
    const __half* su = sg + ms;
    const int nrem = s.count;
    int tok[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) tok[nt] = (nt * 8 + g < nrem) ? slot_tok(a, s, nt * 8 + g) : -1;
    float accg[NT][4], accu[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) accg[nt][i] = accu[nt][i] = 0.f;

    auto process = [&](const TileRegs<BITS>& tg, const TileRegs<BITS>& tu, int kt) {
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            const int k0 = kt * 128 + kb * 32 + 2 * c;
            uint32_t b[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                b[nt][0] = b[nt][1] = b[nt][2] = b[nt][3] = 0u;
                if (tok[nt] >= 0) {
                    const uint16_t* xr = a.x + (int64_t)tok[nt] * a.d + k0;
                    b[nt][0] = *reinterpret_cast<const uint32_t*>(xr);
                    b[nt][1] = *reinterpret_cast<const uint32_t*>(xr + 8);
                    b[nt][2] = *reinterpret_cast<const uint32_t*>(xr + 16);
                    b[nt][3] = *reinterpret_cast<const uint32_t*>(xr + 24);
                }
            }
            {
                uint32_t ag[8];
                decode_block<false, BITS>(tg.lo[kb], tg.hi[kb], ag);
                const uint32_t g0[4] = {ag[0], ag[1], ag[2], ag[3]}, g1[4] = {ag[4], ag[5], ag[6], ag[7]};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_bf16(t4, g0, b[nt][0], b[nt][1], t4);
                    mma_bf16(t4, g1, b[nt][2], b[nt][3], t4);
                    acc_scaled(accg[nt], t4, tg.sc[kb]);
                }
            }
            {
                uint32_t au[8];
                decode_block<false, BITS>(tu.lo[kb], tu.hi[kb], au);
                const uint32_t u0[4] = {au[0], au[1], au[2], au[3]}, u1[4] = {au[4], au[5], au[6], au[7]};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_bf16(t4, u0, b[nt][0], b[nt][1], t4);
                    mma_bf16(t4, u1, b[nt][2], b[nt][3], t4);
                    acc_scaled(accu[nt], t4, tu.sc[kb]);
                }
            }
        }
    };
    for (int kt0 = warp; kt0 < KT; kt0 += 2 * kDecWarps) {
        const int kt1 = kt0 + kDecWarps;
        TileRegs<BITS> g0, u0, g1, u1;
        load_tile<BITS>(cg, sg, (int64_t)jt * KT + kt0, lane, g0);
        load_tile<BITS>(cu, su, (int64_t)jt * KT + kt0, lane, u0);
        if (kt1 < KT) {
            load_tile<BITS>(cg, sg, (int64_t)jt * KT + kt1, lane, g1);
            load_tile<BITS>(cu, su, (int64_t)jt * KT + kt1, lane, u1);
        }
        process(g0, u0, kt0);
        if (kt1 < KT) process(g1, u1, kt1);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            red[(((warp * 2 + 0) * NT + nt) * 4 + i) * 32 + lane] = accg[nt][i];
            red[(((warp * 2 + 1) * NT + nt) * 4 + i) * 32 + lane] = accu[nt][i];
        }
    __syncthreads();
    for (int id = threadIdx.x; id < NT * 4 * 32; id += kDecThreads) {
        const int ln = id & 31, i = (id >> 5) & 3, nt = id >> 7;
        const int m = (ln >> 2) + 8 * (i >> 1);
        const int n = nt * 8 + 2 * (ln & 3) + (i & 1);
        if (n >= nrem) continue;
        float gs = 0.f, us = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            gs += red[(((w * 2 + 0) * NT + nt) * 4 + i) * 32 + ln];
            us += red[(((w * 2 + 1) * NT + nt) * 4 + i) * 32 + ln];
        }
        a.h[(int64_t)(s.hbase + n) * a.f + jt * 16 + m] = __float2half_rn(silu(gs) * us);
    }
}

// ---------------------------------------------------------------- combine of one (token, 16-row tile)
MOE_DEV void combine_tile(const DecodeArgs& a, int t, int rt, int lane) {
    if (lane >= 16) return;
    const int n = rt * 16 + lane;
    float acc = a.n_shared ? a.obuf[((int64_t)a.T * a.k + t) * a.d + n] : 0.0f;
    for (int r = 0; r < a.k; ++r) {
        const int pos = a.inv[(int64_t)t * a.k + r];
        if (pos < 0) continue;
        acc = fmaf(a.w[(int64_t)t * a.k + r], a.obuf[(int64_t)pos * a.d + n], acc);
    }
    if (a.out_fp32) {
        float* y = static_cast<float*>(a.y) + (int64_t)t * a.d + n;
        *y = a.accumulate ? *y + acc : acc;
    } else {
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y) + (int64_t)t * a.d + n;
        *y = __float2bfloat16_rn(a.accumulate ? __bfloat162float(*y) + acc : acc);
    }
}

// ---------------------------------------------------------------- down tile (warp)
// o for the slot's tokens on output rows rt*16 .. +15, then per-token
// completion counting; the warp that completes a (token, tile) combines it.
template <int BITS, int NT>
MOE_DEV void down_tile(const DecodeArgs& a, const Slot& s, int rt, int lane) {
    const int g = lane >> 2, c = lane & 3;
    const int KT = a.f / 128;
    const int64_t mc = (int64_t)a.f * a.d * BITS / 8, ms = (int64_t)a.f * a.d / 32;
    const uint8_t* cd = a.codes + (int64_t)s.expert * 3 * mc + 2 * mc;
    const __half* sd = reinterpret_cast<const __half*>(a.scales) + (int64_t)s.expert * 3 * ms + 2 * ms;
    const int nrem = s.count;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    constexpr int G = 3;  // super-tiles in flight per warp
    for (int kt0 = 0; kt0 < KT; kt0 += G) {
        TileRegs<BITS> td[G];
#pragma unroll
        for (int q = 0; q < G; ++q)
            if (kt0 + q < KT) load_tile<BITS>(cd, sd, (int64_t)rt * KT + kt0 + q, lane, td[q]);
#pragma unroll
        for (int q = 0; q < G; ++q) {
            if (kt0 + q >= KT) break;
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                uint32_t ad[8];
                decode_block<true, BITS>(td[q].lo[kb], td[q].hi[kb], ad);
                const int k0 = (kt0 + q) * 128 + kb * 32 + 2 * c;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    uint32_t b[4] = {0u, 0u, 0u, 0u};
                    if (nt * 8 + g < nrem) {
                        const __half* hr = a.h + (int64_t)(s.hbase + nt * 8 + g) * a.f + k0;
                        b[0] = *reinterpret_cast<const uint32_t*>(hr);
                        b[1] = *reinterpret_cast<const uint32_t*>(hr + 8);
                        b[2] = *reinterpret_cast<const uint32_t*>(hr + 16);
                        b[3] = *reinterpret_cast<const uint32_t*>(hr + 24);
                    }
                    const uint32_t a0[4] = {ad[0], ad[1], ad[2], ad[3]}, a1[4] = {ad[4], ad[5], ad[6], ad[7]};
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(t4, a0, b[0], b[1], t4);
                    mma_f16(t4, a1, b[2], b[3], t4);
                    acc_scaled(acc[nt], t4, td[q].sc[kb]);
                }
            }
        }
    }
    // o -> obuf (rows g, g+8 of the tile; tokens 2c, 2c+1 of each n-tile)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = nt * 8 + 2 * c + (i & 1);
            if (n < nrem) a.obuf[(int64_t)(s.hbase + n) * a.d + rt * 16 + g + 8 * (i >> 1)] = acc[nt][i];
        }
    __threadfence();
    __syncwarp();
    const int target = a.k + a.n_shared;
    for (int i0 = 0; i0 < nrem; i0 += 32) {
        const int i = i0 + lane;
        int t = -1;
        bool last = false;
        if (i < nrem) {
            t = slot_tok(a, s, i);
            last = atom_add_acqrel(a.sync + SY_SLOTS + (1 + a.E) + t * (a.d / 16) + rt, 1) == target - 1;
        }
        unsigned jobs = __ballot_sync(0xffffffffu, last);
        while (jobs) {
            const int src = __ffs(jobs) - 1;
            jobs &= jobs - 1;
            const int tt = __shfl_sync(0xffffffffu, t, src);
            __threadfence();
            combine_tile(a, tt, rt, lane);
        }
    }
}

// ---------------------------------------------------------------- the kernel
template <int BITS, int NT>
__global__ void __launch_bounds__(kDecThreads, NT <= 2 ? 2 : 1) decode_kernel(const DecodeArgs a) {
    extern __shared__ float smem[];
    __shared__ int s_task, s_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TaskMap m = task_map(a);
    int* sync = a.sync;
    int* slot_done = sync + SY_SLOTS;  // [1 + E] (slot index)

    for (;;) {
        if (threadIdx.x == 0) s_task = atomicAdd(sync + SY_HEAD, 1);
        __syncthreads();
        const int task = s_task;
        __syncthreads();
        if (task >= m.total) break;

        if (task < m.b1) {  // router rows
            const int e = task * kDecWarps + warp;
            if (e < a.E) router_row(a, e, lane);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) red_add_release(sync + SY_ROUTER, 1);
        } else if (task < m.b2) {  // shared gate/up
            const int jt = task - m.b1;
            const Slot s = make_slot(a, 0);
            gateup_tile<BITS, NT>(a, s, jt, smem, warp, lane);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) red_add_release(slot_done + 0, 1);
        } else if (task < m.b3) {  // top-k (+ bucketing by the last)
            if (threadIdx.x == 0) s_flag = wait_geq(sync + SY_ROUTER, m.nRt, sync, a.status) ? 1 : 0;
            __syncthreads();
            const int t = (task - m.b2) * kDecWarps + warp;
            if (s_flag && t < a.T) topk_token(a, t, lane, smem + warp * a.E);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) {
                const int ntok = min(kDecWarps, a.T - (task - m.b2) * kDecWarps);
                s_flag = (atom_add_acqrel(sync + SY_TOPK, ntok) + ntok == a.T) ? 1 : 0;
            }
            __syncthreads();
            if (s_flag) {
                if (warp == 0) bucket_warp(a, lane, reinterpret_cast<int*>(smem));
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) st_release(sync + SY_BUCKET, 1);
            }
        } else if (task < m.b4) {  // shared down
            if (threadIdx.x == 0) s_flag = wait_geq(slot_done + 0, m.FT, sync, a.status) ? 1 : 0;
            __syncthreads();
            const int rt = (task - m.b3) * kDecWarps + warp;
            if (threadIdx.x == 0 && s_flag) s_flag = wait_geq(sync + SY_BUCKET, 1, sync, a.status) ? 1 : 0;
            __syncthreads();
            if (s_flag && rt < m.RT16) down_tile<BITS, NT>(a, make_slot(a, 0), rt, lane);
        } else if (task < m.b5) {  // routed gate/up
            const int sidx = (task - m.b4) / m.FT, jt = (task - m.b4) % m.FT;
            if (threadIdx.x == 0) s_flag = wait_geq(sync + SY_BUCKET, 1, sync, a.status) ? 1 : 0;
            __syncthreads();
            if (s_flag && sidx < a.meta->n_active) {
                const Slot s = make_slot(a, a.n_shared + sidx);
                gateup_tile<BITS, NT>(a, s, jt, smem, warp, lane);
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) red_add_release(slot_done + a.n_shared + sidx, 1);
            }
        } else {  // routed down
            const int sidx = (task - m.b5) / m.nRTG, rtg = (task - m.b5) % m.nRTG;
            if (threadIdx.x == 0) s_flag = wait_geq(sync + SY_BUCKET, 1, sync, a.status) ? 1 : 0;
            __syncthreads();
            if (s_flag && sidx < a.meta->n_active) {
                if (threadIdx.x == 0) s_flag = wait_geq(slot_done + a.n_shared + sidx, m.FT, sync, a.status) ? 1 : 0;
                __syncthreads();
                const int rt = rtg * kDecWarps + warp;
                if (s_flag && rt < m.RT16) down_tile<BITS, NT>(a, make_slot(a, a.n_shared + sidx), rt, lane);
            }
        }
        __syncthreads();
    }

    // leave; the last CTA resets the counters for the next launch
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_flag = (atom_add_acqrel(sync + SY_EXIT, 1) == (int)gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (s_flag) {
        __threadfence();
        const int n = SY_SLOTS + (1 + a.E) + a.T * (a.d / 16);
        for (int i = threadIdx.x; i < n; i += kDecThreads) sync[i] = 0;
    }
}

// ---------------------------------------------------------------- launcher
template <int BITS, int NT>
static cudaError_t decode_bits_nt(const DecodeLaunch& L, cudaStream_t st) {
    auto kern = decode_kernel<BITS, NT>;
    const int E = L.E;
    // union: gate/up partials | per-warp top-k logits | bucket counters
    const size_t smem = (size_t)max(max(NT * kDecWarps * 2 * 4 * 32, kDecWarps * E), 2 * E + 1) * sizeof(float);
    static int blocks_per_sm[64] = {};  // per device, looked up once
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    if (blocks_per_sm[dev] == 0) {
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kDecThreads, smem);
        if (e != cudaSuccess) return e;
        blocks_per_sm[dev] = nb > 0 ? nb : 1;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    DecodeArgs a;
    a.T = L.T;
    a.d = L.d;
    a.f = L.f;
    a.E = L.E;
    a.k = L.k;
    a.n_shared = L.n_shared;
    a.x = static_cast<const uint16_t*>(L.x);
    a.y = L.y;
    a.out_fp32 = L.out_fp32;
    a.accumulate = L.accumulate;
    a.codes = L.codes;
    a.scales = L.scales;
    a.wr = static_cast<const uint16_t*>(L.wr);
    a.bias = L.bias;
    a.wnorm = L.wnorm;
    a.logits = L.logits;
    a.logits64 = L.logits64;
    a.ids = L.ids;
    a.w = L.w;
    a.offsets = L.offsets;
    a.pairs = L.pairs;
    a.inv = L.inv;
    a.active = L.active;
    a.meta = L.meta;
    a.status = L.status;
    a.h = static_cast<__half*>(L.h);
    a.obuf = L.obuf;
    a.sync = L.sync;
    const int grid = blocks_per_sm[dev] * sms;
    kern<<<grid, kDecThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int BITS>
static cudaError_t decode_bits(const DecodeLaunch& L, cudaStream_t s) {
    if (L.T <= 8) return decode_bits_nt<BITS, 1>(L, s);
    if (L.T <= 16) return decode_bits_nt<BITS, 2>(L, s);
    if (L.T <= 32) return decode_bits_nt<BITS, 4>(L, s);
    return decode_bits_nt<BITS, 8>(L, s);
}

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t s) {
    if (L.T < 1 || L.T > kDecodeMaxTokens || L.E > 1024 || L.k > 32) return cudaErrorInvalidValue;
    switch (L.bits) {
        case 2: return decode_bits<2>(L, s);
        case 3: return decode_bits<3>(L, s);
        case 4: return decode_bits<4>(L, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t decode_sync_words(int max_tokens, int E, int d) {
    return (size_t)SY_SLOTS + (1 + (size_t)E) + (size_t)max_tokens * (d / 16);
}

}  // namespace moe

// decode.cu -- the whole routed-MoE layer for up to 64 tokens in ONE persistent kernel.
//
// Decode and draft-verify batches (1 token plus up to 3 drafts; the layer the
// Strata pages run per generated token: the router picks the experts, they
// run, "the GPU combines each result, then moves to the next layer" --
// discuss.pytorch.kr post, section "Strata's operating principle") move ~18 MB
// of weights per token-layer, a few microseconds of HBM time, so separate
// launches per step would dominate.  Here one launch does everything.  CTAs
// pull tasks from a global queue in dependency order:
//   1. router rows (8 experts per CTA, exact fp64 logits)
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
//
// Every task that multiplies weights stages them in shared memory with 1-D
// bulk copies (TMA, one elected thread, completion on an mbarrier): a gate/up
// tile is 2 x 16 contiguous super-tiles, a down task 8 row-tiles x f/128
// contiguous super-tiles, a router task 8 contiguous W_r rows.  The activation
// rows (or h rows) it multiplies are staged the same way into padded rows, so
// warps read their MMA operands from shared memory without bank conflicts and
// hold no weights in registers.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kSpinLimit = 1u << 21;  // spins of >= 32 ns (mostly 256 ns): >= 0.5 s
constexpr int kPad = 8;                    // 16-bit elements of padding per staged row
constexpr int kRouterRows = 4;             // router rows per task (two warps per row)

// sync block (int32 words); each scalar counter has a 128-byte line of its own
enum { SY_HEAD = 0, SY_ROUTER = 32, SY_TOPK = 64, SY_BUCKET = 96, SY_EXIT = 128, SY_ABORT = 160, SY_FIXUP = 192,
       SY_SLOTS = 224 };

MOE_DEV int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
MOE_DEV int ld_relaxed(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
MOE_DEV void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
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
// Polls with relaxed loads and a growing sleep (hundreds of CTAs may wait on
// one flag), then fences once so later reads see what the release published.
MOE_DEV bool wait_geq(const int* p, int target, int* sync, uint32_t* status) {
    uint32_t ns = 32;
    for (uint32_t it = 0;; ++it) {
        if (ld_relaxed(p) >= target) {
            fence_acq_rel_gpu();
            return true;
        }
        if ((it & 7) == 7 && ld_relaxed(sync + SY_ABORT)) return false;
        if (it > kSpinLimit) {
            flag_status(status, kStatusTimeout);
            st_release(sync + SY_ABORT, 1);
            return false;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
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
    int skip_rank;  // route-tail skip: drop experts whose best rank is >= this (0: off)
    int e_begin, e_end;  // experts outside [e_begin, e_end) are dropped (expert parallelism)
    int red_bytes;  // shared memory: [red_bytes] reductions | 2 x [buf_bytes] staging buffers
    int buf_bytes;  //   each buffer: [w_bytes] weights | activations
    int w_bytes;
};

struct TaskMap {
    int nRt, nSG, nTK, nSD, nRG, nRD, RT16, nRTG, maxR, FT;
    int b1, b2, b3, b4, b5, total;
};

MOE_DEV TaskMap task_map(const DecodeArgs& a) {
    TaskMap m;
    m.nRt = (a.E + kRouterRows - 1) / kRouterRows;
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
    const int* tok;  // routed slot with the CTA's slot table: token of each of its pairs (shared memory)
};

// The CTA's copy of the bucketing, loaded once after it is published:
// tbl[0] = n_active, tbl[1] = pairs, then expert[maxR], pair0[maxR],
// count[maxR], token[T*k] (token of each pair position).
__host__ __device__ inline size_t slot_table_words(int maxR, int npairs) { return 2 + 3 * (size_t)maxR + (size_t)npairs; }

MOE_DEV Slot make_slot(const DecodeArgs& a, int slot, const int* tbl, int maxR) {
    Slot s;
    s.tok = nullptr;
    if (slot < a.n_shared) {
        s.expert = a.E;
        s.count = a.T;
        s.hbase = a.T * a.k;
        s.pair0 = 0;
        s.shared = true;
    } else if (tbl) {
        const int i = slot - a.n_shared;
        s.expert = tbl[2 + i];
        s.pair0 = tbl[2 + maxR + i];
        s.count = tbl[2 + 2 * maxR + i];
        s.hbase = s.pair0;
        s.shared = false;
        s.tok = tbl + 2 + 3 * maxR + s.pair0;
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
MOE_DEV Slot make_slot(const DecodeArgs& a, int slot) { return make_slot(a, slot, nullptr, 0); }

MOE_DEV int slot_tok(const DecodeArgs& a, const Slot& s, int i) {
    return s.shared ? i : (s.tok ? s.tok[i] : a.pairs[s.pair0 + i] / a.k);
}

MOE_DEV float h_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu))); }
MOE_DEV float h_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }
MOE_DEV float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEV float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

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

// ---------------------------------------------------------------- 1. router rows (CTA)
// logits64[t][e] = sum_i double(W_r[e,i]) * double(x[t,i]) + double(bias_e).
// A task covers kRouterRows experts; warp w takes expert w/2 and half w%2 of
// the columns (lane: columns half*d/2 + lane*8 + 256 j, j while < d/2).  A bf16 x bf16
// product is exact in fp32, and it and every partial sum are exact in fp64
// (their bits span far less than 53), so the logits are the exact fp64 values
// of the plain definition in any summation order: ranking them is the exact
// ranking.  part: [kRouterRows][2][8] doubles of shared memory.
MOE_DEV void router_compute(const DecodeArgs& a, int e0, int nrow, int t0, int nt, const uint16_t* W,
                            const uint16_t* xs, double* part, int warp, int lane) {
    const int d = a.d, stride = d + kPad;
    const int r = warp >> 1, half = warp & 1;
    if (r < nrow) {
        const uint16_t* wrow = W + r * d + half * (d / 2);
        const uint16_t* xh = xs + half * (d / 2);
        double acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0;
        for (int c0 = lane * 8; c0 < d / 2; c0 += 256) {
            const uint4 wv = *reinterpret_cast<const uint4*>(wrow + c0);
            const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (q >= nt) break;
                const uint4 xv = *reinterpret_cast<const uint4*>(xh + q * stride + c0);
                const uint32_t x4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc[q] += (double)(bf_lo(w4[u]) * bf_lo(x4[u]));  // exact product, exact sum
                    acc[q] += (double)(bf_hi(w4[u]) * bf_hi(x4[u]));
                }
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q >= nt) break;
            double v = acc[q];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) part[(r * 2 + half) * 8 + q] = v;
        }
    }
    __syncthreads();
    if (threadIdx.x < nrow * 8) {
        const int rr = threadIdx.x >> 3, q = threadIdx.x & 7;
        if (q < nt) {
            const int e = e0 + rr;
            const double b = a.bias ? (double)a.bias[e] : 0.0;
            a.logits64[(int64_t)(t0 + q) * a.E + e] = part[(rr * 2) * 8 + q] + part[(rr * 2 + 1) * 8 + q] + b;
        }
    }
}

// ---------------------------------------------------------------- 3. exact top-k of one token (warp)
// Order (l desc, e asc), NaN ranked as -inf: a 64-bit key that orders like the
// double (with -0 == +0), compared together with the expert index.
MOE_DEV uint64_t order_key(double v) {
    if (isnan(v)) v = -INFINITY;
    v = v + 0.0;  // -0 -> +0
    const uint64_t b = (uint64_t)__double_as_longlong(v);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
MOE_DEV bool key_better(uint64_t ka, int ia, uint64_t kb, int ib) { return ka > kb || (ka == kb && ia < ib); }

// v: this warp's E-double shared-memory buffer.
// Fast path (E <= 512, k <= 15): 32-bit keys = an order-preserving image of
// fp32(l) with the low 10 bits replaced by (1023 - e).  A strictly larger key
// prefix means a strictly larger logit, so the exact top-k lies among the
// elements whose prefix is >= the k-th key's prefix.  Each lane sorts its 16
// keys (bitonic, min/max), a 5-level butterfly merges the sorted lists so every
// lane holds the global top 16, and those candidates are ranked exactly by
// (fp64 logit desc, index asc) with pairwise comparisons.  If the candidates do
// not fit in 16 (ties in the key prefix) or E, k are larger, a slow exact scan
// runs instead.  ids_s: the token's k ids are also left here for bucketing.
constexpr int kTopkLane = 16;

MOE_DEV uint32_t key32(double v, int e) {
    float f = (float)(isnan(v) ? -INFINITY : v);
    f = f + 0.0f;  // -0 -> +0
    const uint32_t b = __float_as_uint(f);
    const uint32_t o = (b >> 31) ? ~b : (b | 0x80000000u);
    return (o & 0xFFFFFC00u) | (uint32_t)(1023 - e);
}

MOE_DEV void topk_exact_scan(const double* v, int E, int k, int lane, int& sel, double& lsel, double& top) {
    uint32_t taken = 0;
    auto local_best = [&](uint64_t& bk, int& bi) {
        bk = 0;
        bi = 0x7fffffff;
        for (int j = 0, e = lane; e < E; ++j, e += 32) {
            if ((taken >> j) & 1u) continue;
            const uint64_t ke = order_key(v[e]);
            if (bi == 0x7fffffff || key_better(ke, e, bk, bi)) {
                bk = ke;
                bi = e;
            }
        }
    };
    uint64_t mk;
    int mi;
    local_best(mk, mi);
    for (int r = 0; r < k; ++r) {
        uint64_t bk = mk;
        int bi = mi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != 0x7fffffff && (bi == 0x7fffffff || key_better(ok, oi, bk, bi))) {
                bk = ok;
                bi = oi;
            }
        }
        const double lv = v[bi];
        if (lane == r) {
            sel = bi;
            lsel = lv;
        }
        if (r == 0) top = lv;
        if ((bi & 31) == lane) {
            taken |= 1u << (bi >> 5);
            local_best(mk, mi);
        }
    }
}

// v: the token's E fp64 logits, already copied to this warp's shared buffer.
MOE_DEV void topk_token(const DecodeArgs& a, int t, int lane, double* v, int* ids_s) {
    const int E = a.E, k = a.k;
    int sel = -1;     // lane r < k keeps ids[r]
    double lsel = 0;  //   and its logit
    double top = 0;
    bool done = false;
    if (E <= 32 * kTopkLane && k < kTopkLane) {
        uint32_t kk[kTopkLane];
#pragma unroll
        for (int j = 0; j < kTopkLane; ++j) {
            const int e = lane + 32 * j;
            kk[j] = e < E ? key32(v[e], e) : 0u;
        }
        // sort descending (bitonic network on registers)
#pragma unroll
        for (int size = 2; size <= kTopkLane; size <<= 1)
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
                for (int i = 0; i < kTopkLane; ++i) {
                    const int jx = i ^ stride;
                    if (jx > i) {
                        const uint32_t lo = min(kk[i], kk[jx]), hi = max(kk[i], kk[jx]);
                        const bool desc = (i & size) == 0;
                        kk[i] = desc ? hi : lo;
                        kk[jx] = desc ? lo : hi;
                    }
                }
        // butterfly: merge with the partner's sorted list, keep the top 16, re-sort
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
            for (int j = 0; j < kTopkLane; ++j) {
                const uint32_t other = __shfl_xor_sync(0xffffffffu, kk[kTopkLane - 1 - j], o);
                kk[j] = max(kk[j], other);  // bitonic: top 16 of the two lists
            }
#pragma unroll
            for (int stride = kTopkLane >> 1; stride > 0; stride >>= 1)
#pragma unroll
                for (int i = 0; i < kTopkLane; ++i) {
                    const int jx = i ^ stride;
                    if (jx > i) {
                        const uint32_t lo = min(kk[i], kk[jx]), hi = max(kk[i], kk[jx]);
                        kk[i] = hi;
                        kk[jx] = lo;
                    }
                }
        }
        // candidates: key prefix >= the k-th key's prefix (a sorted prefix of kk)
        uint32_t kth = 0xFFFFFFFFu;
#pragma unroll
        for (int j = 0; j < kTopkLane; ++j)
            if (j < k) kth = min(kth, kk[j]);
        const uint32_t pk = kth & 0xFFFFFC00u;
        if ((kk[kTopkLane - 1] & 0xFFFFFC00u) < pk) {
            int m = 0;
            uint32_t mine = 0;
#pragma unroll
            for (int j = 0; j < kTopkLane; ++j) {
                if ((kk[j] & 0xFFFFFC00u) >= pk) ++m;
                if (j == lane) mine = kk[j];
            }
            const int my_e = 1023 - (int)(mine & 0x3FFu);
            const double my_v = lane < m ? v[my_e] : 0.0;
            const uint64_t my_k = order_key(my_v);
            int rank = 0;
            for (int j = 0; j < m; ++j) {
                const uint64_t ok = __shfl_sync(0xffffffffu, my_k, j);
                const int oe = __shfl_sync(0xffffffffu, my_e, j);
                if (j != lane && key_better(ok, oe, my_k, my_e)) ++rank;
            }
            // lane r < k fetches the candidate of rank r
            for (int j = 0; j < m; ++j) {
                const int rj = __shfl_sync(0xffffffffu, rank, j);
                const int ej = __shfl_sync(0xffffffffu, my_e, j);
                const double vj = __shfl_sync(0xffffffffu, my_v, j);
                if (rj == lane) {
                    sel = ej;
                    lsel = vj;
                }
                if (rj == 0) top = vj;
            }
            done = true;
        }
    }
    if (!done) topk_exact_scan(v, E, k, lane, sel, lsel, top);
    // renormalised weights: softmax over the k selected logits (fp32)
    const float ex = lane < k ? expf((float)(lsel - top)) : 0.0f;
    float z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane < k) {
        a.ids[(int64_t)t * k + lane] = sel;
        a.w[(int64_t)t * k + lane] = ex / z;
        ids_s[lane] = sel;
    }
}

// ---------------------------------------------------------------- bucketing (CTA)
// Counting sort of the T*k pairs by expert, stable in token order.
// sm: cnt[E] | off[E + 1] | ids[T*k] | wtot[3 * kDecWarps]
MOE_DEV void bucket_cta(const DecodeArgs& a, int* sm, const int* ids_local) {
    const int E = a.E, k = a.k, n = a.T * a.k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* cnt = sm;
    int* off = sm + E;
    int* ids = off + E + 1;
    int* wtot = ids + n;
    const int R = a.skip_rank;  // > 0: route-tail skip from this rank on
    const int e0 = a.e_begin, e1 = a.e_end;  // kept expert range
    for (int e = threadIdx.x; e < E; e += kDecThreads) {
        cnt[e] = 0;
        off[e] = k;  // best (lowest) rank of expert e in the batch, until the scan
    }
    for (int i = threadIdx.x; i < n; i += kDecThreads) ids[i] = ids_local ? ids_local[i] : a.ids[i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kDecThreads) {
        const int e = ids[i];
        if (e >= 0 && e < E) {
            atomicAdd(&cnt[e], 1);
            if (R > 0) atomicMin(&off[e], i % k);
        } else {
            flag_status(a.status, kStatusBounds);
        }
    }
    __syncthreads();
    if (R > 0 || e0 > 0 || e1 < E) {
        // dropped experts (no rank below R in the batch, or outside the kept
        // range): no count, their pairs get inv = -1
        auto dropped = [&](int e) { return (R > 0 && off[e] >= R) || e < e0 || e >= e1; };
        for (int e = threadIdx.x; e < E; e += kDecThreads)
            if (dropped(e)) cnt[e] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kDecThreads) {
            const int e = ids[i];
            if (e >= 0 && e < E && dropped(e)) ids[i] = -1;
        }
        __syncthreads();
        // A dropped pair never reports to its token's combine counters (one per
        // 16-row output tile, complete at k + n_shared): count it in advance.
        // Nothing touches these counters before the bucketing is published.
        const int RT = a.d / 16;
        for (int j = threadIdx.x; j < a.T * RT; j += kDecThreads) {
            const int t = j / RT;
            int nd = 0;
            for (int r = 0; r < k; ++r) {
                const int e = ids[t * k + r];
                nd += (e < 0 || e >= E) ? 1 : 0;
            }
            if (nd == k && a.n_shared == 0) {
                // nothing reaches this token's combine: its output is 0 here
                const int n0 = (j - t * RT) * 16;
                if (a.out_fp32) {
                    float* y = static_cast<float*>(a.y) + (int64_t)t * a.d + n0;
                    if (!a.accumulate)
                        for (int q = 0; q < 16; ++q) y[q] = 0.0f;
                } else if (!a.accumulate) {
                    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y) + (int64_t)t * a.d + n0;
                    for (int q = 0; q < 16; ++q) y[q] = __float2bfloat16_rn(0.0f);
                }
            } else if (nd) {
                atomicAdd(a.sync + SY_SLOTS + (1 + E) + j, nd);
            }
        }
    }
    // block-wide exclusive scan of cnt and of the active flags: warp w owns a
    // contiguous chunk of experts, 32 per step
    const int chunk = ((E + kDecWarps - 1) / kDecWarps + 31) & ~31;
    const int e_begin = warp * chunk, e_end = min(E, e_begin + chunk);
    int run = 0, runa = 0, mx = 0;
    for (int e0 = e_begin; e0 < e_end; e0 += 32) {
        const int e = e0 + lane;
        const int cv = e < e_end ? cnt[e] : 0;
        int inc = cv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += u;
        }
        if (e < e_end) off[e] = run + inc - cv;  // chunk-local for now
        run += __shfl_sync(0xffffffffu, inc, 31);
        runa += __popc(__ballot_sync(0xffffffffu, cv > 0));
        mx = max(mx, cv);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) {
        wtot[warp] = run;
        wtot[kDecWarps + warp] = runa;
        wtot[2 * kDecWarps + warp] = mx;
    }
    __syncthreads();
    int base = 0, abase = 0;
    for (int w = 0; w < warp; ++w) {
        base += wtot[w];
        abase += wtot[kDecWarps + w];
    }
    for (int e0 = e_begin; e0 < e_end; e0 += 32) {
        const int e = e0 + lane;
        const int cv = e < e_end ? cnt[e] : 0;
        if (e < e_end) {
            off[e] += base;
            a.offsets[e] = off[e];
        }
        const unsigned bal = __ballot_sync(0xffffffffu, cv > 0);
        if (cv > 0) a.active[abase + __popc(bal & ((1u << lane) - 1u))] = e;
        abase += __popc(bal);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int tot = 0, nact = 0, big = 0;
        for (int w = 0; w < kDecWarps; ++w) {
            tot += wtot[w];
            nact += wtot[kDecWarps + w];
            big = max(big, wtot[2 * kDecWarps + w]);
        }
        a.offsets[E] = tot;
        a.meta->n_active = nact;
        a.meta->max_count = big;
        a.meta->n_fixup = 0;  // the fp64 logits need no re-ranking
    }
    __syncthreads();
    // stable scatter by warp 0, token by token (a token's k experts are distinct)
    if (warp == 0) {
        for (int t = 0; t < a.T; ++t) {
            if (lane < k) {
                const int e = ids[t * k + lane];
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
}

// ---------------------------------------------------------------- gate/up tile (CTA)
// h[hbase + i][jt*16 .. +15] = silu(g) * u for the slot's tokens i.  W holds
// the 16-row tile's gate codes (KT super-tiles), gate scales, up codes, up
// scales; with STAGE, xs holds the slot's activation rows (padded).  The 8
// warps split the KT super-tiles of the input dimension.
template <int BITS, int NT, bool STAGE>
MOE_DEV void gateup_compute(const DecodeArgs& a, const Slot& s, int jt, float* red, const uint8_t* W,
                            const uint16_t* xs, int warp, int lane) {
    constexpr int TB = 256 * BITS;
    const int g = lane >> 2, c = lane & 3;
    const int KT = a.d / 128;
    const int xstride = a.d + kPad;
    const uint8_t* gc = W;
    const uint8_t* gs = gc + KT * TB;
    const uint8_t* uc = gs + KT * 128;
    const uint8_t* us = uc + KT * TB;
    const int nrem = s.count;
    int tok[NT];
    if (!STAGE) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tok[nt] = (nt * 8 + g < nrem) ? slot_tok(a, s, nt * 8 + g) : -1;
    }
    float accg[NT][4], accu[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) accg[nt][i] = accu[nt][i] = 0.f;

    for (int kt = warp; kt < KT; kt += kDecWarps) {
        TileRegs<BITS> tg, tu;
        load_tile_smem<BITS>(gc + kt * TB, gs + kt * 128, lane, tg);
        load_tile_smem<BITS>(uc + kt * TB, us + kt * 128, lane, tu);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            const int k0 = kt * 128 + kb * 32 + 2 * c;
            uint32_t b[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                b[nt][0] = b[nt][1] = b[nt][2] = b[nt][3] = 0u;
                const int i = nt * 8 + g;
                const uint16_t* xr = nullptr;
                if (STAGE) {
                    if (i < nrem) xr = xs + i * xstride + k0;
                } else if (tok[nt] >= 0) {
                    xr = a.x + (int64_t)tok[nt] * a.d + k0;
                }
                if (xr) {
                    b[nt][0] = *reinterpret_cast<const uint32_t*>(xr);
                    b[nt][1] = *reinterpret_cast<const uint32_t*>(xr + 8);
                    b[nt][2] = *reinterpret_cast<const uint32_t*>(xr + 16);
                    b[nt][3] = *reinterpret_cast<const uint32_t*>(xr + 24);
                }
            }
            {
                uint32_t q[8];
                decode_block<false, BITS>(tg.lo[kb], tg.hi[kb], q);
                const uint32_t q0[4] = {q[0], q[1], q[2], q[3]}, q1[4] = {q[4], q[5], q[6], q[7]};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_bf16(t4, q0, b[nt][0], b[nt][1], t4);
                    mma_bf16(t4, q1, b[nt][2], b[nt][3], t4);
                    acc_scaled(accg[nt], t4, tg.sc[kb]);
                }
            }
            {
                uint32_t q[8];
                decode_block<false, BITS>(tu.lo[kb], tu.hi[kb], q);
                const uint32_t q0[4] = {q[0], q[1], q[2], q[3]}, q1[4] = {q[4], q[5], q[6], q[7]};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt * 8 >= nrem) break;
                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_bf16(t4, q0, b[nt][0], b[nt][1], t4);
                    mma_bf16(t4, q1, b[nt][2], b[nt][3], t4);
                    acc_scaled(accu[nt], t4, tu.sc[kb]);
                }
            }
        }
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
        float gsum = 0.f, usum = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            gsum += red[(((w * 2 + 0) * NT + nt) * 4 + i) * 32 + ln];
            usum += red[(((w * 2 + 1) * NT + nt) * 4 + i) * 32 + ln];
        }
        a.h[(int64_t)(s.hbase + n) * a.f + jt * 16 + m] = __float2half_rn(silu(gsum) * usum);
    }
}

// Thread 0: issue the bulk copies of one gate/up task (weights of tile jt of
// the slot's expert; with STAGE its activation rows too).  Returns the bytes.
template <int BITS, bool STAGE>
MOE_DEV uint32_t gateup_issue(const DecodeArgs& a, const Slot& s, int jt, uint8_t* W, uint16_t* xs, uint64_t* bar) {
    constexpr int TB = 256 * BITS;
    const int KT = a.d / 128;
    const int64_t mc = (int64_t)a.f * a.d * BITS / 8, msb = (int64_t)a.f * a.d / 16;  // bytes per matrix
    const uint8_t* cbase = a.codes + (int64_t)s.expert * 3 * mc;
    const uint8_t* sbase = reinterpret_cast<const uint8_t*>(a.scales) + (int64_t)s.expert * 3 * msb;
    const uint32_t cb = KT * TB, sb = KT * 128;
    const uint32_t xb = STAGE ? (uint32_t)s.count * a.d * 2 : 0;
    mbar_arrive_expect_tx(bar, 2 * (cb + sb) + xb);
    bulk_g2s(W, cbase + (int64_t)jt * cb, cb, bar);
    bulk_g2s(W + cb, sbase + (int64_t)jt * sb, sb, bar);
    bulk_g2s(W + cb + sb, cbase + mc + (int64_t)jt * cb, cb, bar);
    bulk_g2s(W + 2 * cb + sb, sbase + msb + (int64_t)jt * sb, sb, bar);
    if (STAGE)
        for (int i = 0; i < s.count; ++i)
            bulk_g2s(xs + i * (a.d + kPad), a.x + (int64_t)slot_tok(a, s, i) * a.d, a.d * 2, bar);
    return 2 * (cb + sb) + xb;
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

// ---------------------------------------------------------------- down tiles (CTA: one 16-row tile per warp)
// o for the slot's tokens on output rows rt*16 .. +15 (rt = 8 rtg + warp),
// then per-token completion counting; the warp that completes a (token, tile)
// combines it.  W holds the CTA's 8 row-tiles x KTd super-tiles of codes, then
// their scales; with STAGE, hs holds the slot's h rows (padded).
template <int BITS, int NT, bool STAGE>
MOE_DEV void down_compute(const DecodeArgs& a, const Slot& s, int rtg, int RT16, const uint8_t* W,
                          const uint16_t* hs, int warp, int lane) {
    constexpr int TB = 256 * BITS;
    const int g = lane >> 2, c = lane & 3;
    const int KTd = a.f / 128;
    const int rt = rtg * kDecWarps + warp;
    if (rt >= RT16) return;
    const int hstride = a.f + kPad;
    const uint8_t* wc = W + warp * KTd * TB;
    const uint8_t* ws = W + kDecWarps * KTd * TB + warp * KTd * 128;
    const int nrem = s.count;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    for (int kt = 0; kt < KTd; ++kt) {
        TileRegs<BITS> td;
        load_tile_smem<BITS>(wc + kt * TB, ws + kt * 128, lane, td);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            uint32_t q[8];
            decode_block<true, BITS>(td.lo[kb], td.hi[kb], q);
            const int k0 = kt * 128 + kb * 32 + 2 * c;
            const uint32_t a0[4] = {q[0], q[1], q[2], q[3]}, a1[4] = {q[4], q[5], q[6], q[7]};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (nt * 8 >= nrem) break;
                uint32_t b[4] = {0u, 0u, 0u, 0u};
                if (nt * 8 + g < nrem) {
                    const uint16_t* hr = STAGE ? hs + (nt * 8 + g) * hstride + k0
                                               : reinterpret_cast<const uint16_t*>(a.h) +
                                                     (int64_t)(s.hbase + nt * 8 + g) * a.f + k0;
                    b[0] = *reinterpret_cast<const uint32_t*>(hr);
                    b[1] = *reinterpret_cast<const uint32_t*>(hr + 8);
                    b[2] = *reinterpret_cast<const uint32_t*>(hr + 16);
                    b[3] = *reinterpret_cast<const uint32_t*>(hr + 24);
                }
                float t4[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16(t4, a0, b[0], b[1], t4);
                mma_f16(t4, a1, b[2], b[3], t4);
                acc_scaled(acc[nt], t4, td.sc[kb]);
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

// Thread 0: announce and issue the weight copies of a down task.
template <int BITS>
MOE_DEV uint32_t down_weight_bytes(const DecodeArgs& a, int rtg, int RT16) {
    const int nrt = min(kDecWarps, RT16 - rtg * kDecWarps);
    return (uint32_t)nrt * (a.f / 128) * (256 * BITS + 128);
}
template <int BITS>
MOE_DEV void down_issue_weights(const DecodeArgs& a, const Slot& s, int rtg, int RT16, uint8_t* W, uint64_t* bar) {
    constexpr int TB = 256 * BITS;
    const int KTd = a.f / 128;
    const int nrt = min(kDecWarps, RT16 - rtg * kDecWarps);
    const int64_t mc = (int64_t)a.f * a.d * BITS / 8, msb = (int64_t)a.f * a.d / 16;
    const uint8_t* cbase = a.codes + (int64_t)s.expert * 3 * mc + 2 * mc;
    const uint8_t* sbase = reinterpret_cast<const uint8_t*>(a.scales) + (int64_t)s.expert * 3 * msb + 2 * msb;
    const int64_t st0 = (int64_t)rtg * kDecWarps * KTd;
    bulk_g2s(W, cbase + st0 * TB, (uint32_t)nrt * KTd * TB, bar);
    bulk_g2s(W + kDecWarps * KTd * TB, sbase + st0 * 128, (uint32_t)nrt * KTd * 128, bar);
}
// All threads: copy the slot's h rows (written by other CTAs, published by the
// release the caller acquired) into shared memory with padded rows.
MOE_DEV void stage_h_rows(const DecodeArgs& a, const Slot& s, uint16_t* hs) {
    const int vpr = a.f / 8, stride = a.f + kPad;
    const uint16_t* h = reinterpret_cast<const uint16_t*>(a.h);
    for (int v = threadIdx.x; v < s.count * vpr; v += kDecThreads) {
        const int r = v / vpr, c = v - r * vpr;
        *reinterpret_cast<uint4*>(hs + r * stride + 8 * c) =
            *reinterpret_cast<const uint4*>(h + (int64_t)(s.hbase + r) * a.f + 8 * c);
    }
}

// ---------------------------------------------------------------- the kernel
// Wait for a buffer's staged copies (all threads).  On a timeout: flag it,
// stop every other wait, give the copies in flight a second bounded wait, and
// report failure.
MOE_DEV bool stage_wait(uint64_t* bar, uint32_t& phase, const DecodeArgs& a) {
    for (uint32_t it = 0; it <= kSpinLimit; ++it)
        if (mbar_try_wait(bar, phase)) {
            phase ^= 1u;
            return true;
        }
    if (threadIdx.x == 0) {
        flag_status(a.status, kStatusTimeout);
        st_release(a.sync + SY_ABORT, 1);
    }
    for (uint32_t it = 0; it <= kSpinLimit; ++it)
        if (mbar_try_wait(bar, phase)) {
            phase ^= 1u;
            break;
        }
    return false;
}

enum { K_ROUTER, K_SGU, K_TOPK, K_SDN, K_RGU, K_RDN };

struct Task {
    int kind, slot, sidx, idx;  // idx: jt (gate/up), rtg (down), router task or top-k task index
};

MOE_DEV Task decode_task(const TaskMap& m, int task) {
    Task t;
    t.slot = 0;
    t.sidx = 0;
    if (task < m.b1) {
        t.kind = K_ROUTER;
        t.idx = task;
    } else if (task < m.b2) {
        t.kind = K_SGU;
        t.idx = task - m.b1;
    } else if (task < m.b3) {
        t.kind = K_TOPK;
        t.idx = task - m.b2;
    } else if (task < m.b4) {
        t.kind = K_SDN;
        t.idx = task - m.b3;
    } else if (task < m.b5) {
        t.kind = K_RGU;
        t.sidx = (task - m.b4) / m.FT;
        t.idx = (task - m.b4) % m.FT;
    } else {
        t.kind = K_RDN;
        t.sidx = (task - m.b5) / m.nRTG;
        t.idx = (task - m.b5) % m.nRTG;
    }
    return t;
}

// Per-CTA pipeline: buffer b holds the running task's staged operands while
// the next task's weights land in buffer 1 - b.
struct Pipe {
    uint8_t* R[2];     // staging regions: [weights W | activations A]
    int w_bytes;       // size of the W part
    uint64_t* bar;     // [2]
    uint32_t phase[2];
};

// Thread 0: issue the copies a task can start now (routed tasks need the
// bucketing, which the caller has checked).  Returns 1 if copies were issued.
template <int BITS, bool STAGE>
MOE_DEV int issue_task(const DecodeArgs& a, const TaskMap& m, const Task& t, Pipe& p, int buf, const int* tbl) {
    uint8_t* W = p.R[buf];
    uint16_t* A = reinterpret_cast<uint16_t*>(p.R[buf] + p.w_bytes);
    uint64_t* bar = p.bar + buf;
    fence_proxy_async_smem();  // earlier generic use of this buffer happens before the copies
    switch (t.kind) {
        case K_ROUTER: {
            const int e0 = t.idx * kRouterRows, nrow = min(kRouterRows, a.E - e0), nt = min(8, a.T);
            mbar_arrive_expect_tx(bar, (uint32_t)(nrow + nt) * a.d * 2);
            bulk_g2s(W, a.wr + (int64_t)e0 * a.d, (uint32_t)nrow * a.d * 2, bar);
            for (int q = 0; q < nt; ++q) bulk_g2s(A + q * (a.d + kPad), a.x + (int64_t)q * a.d, a.d * 2, bar);
            return 1;
        }
        case K_SGU:
            gateup_issue<BITS, STAGE>(a, make_slot(a, 0), t.idx, W, A, bar);
            return 1;
        case K_SDN:
            mbar_arrive_expect_tx(bar, down_weight_bytes<BITS>(a, t.idx, m.RT16));
            down_issue_weights<BITS>(a, make_slot(a, 0), t.idx, m.RT16, W, bar);
            return 1;
        case K_RGU:
            if (!tbl || t.sidx >= tbl[0]) return 0;
            gateup_issue<BITS, STAGE>(a, make_slot(a, a.n_shared + t.sidx, tbl, m.maxR), t.idx, W, A, bar);
            return 1;
        case K_RDN:
            if (!tbl || t.sidx >= tbl[0]) return 0;
            mbar_arrive_expect_tx(bar, down_weight_bytes<BITS>(a, t.idx, m.RT16));
            down_issue_weights<BITS>(a, make_slot(a, a.n_shared + t.sidx, tbl, m.maxR), t.idx, m.RT16, W, bar);
            return 1;
        default:
            return 0;
    }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int s_claim, s_flag, s_issued[2], s_nact;
    constexpr bool STAGE = NT <= 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TaskMap m = task_map(a);
    int* sync = a.sync;
    int* slot_done = sync + SY_SLOTS;  // [1 + E] (slot index)
    float* red = reinterpret_cast<float*>(smem_raw);  // gate/up partial sums, router partials
    Pipe p;
    p.R[0] = smem_raw + a.red_bytes;
    p.R[1] = p.R[0] + a.buf_bytes;
    p.w_bytes = a.w_bytes;
    p.bar = bars;
    p.phase[0] = p.phase[1] = 0;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_proxy_async_smem();
        s_nact = -1;
    }
    __syncthreads();

    // Claim the next task.  Routed tasks exist for min(T*k, E) expert slots,
    // but only n_active of them have an expert: once the bucketing is
    // published, a claim that lands past the last active slot moves the head
    // to the next phase (or the end), so empty tasks are never run.
    auto claim = [&]() {
        if (threadIdx.x == 0) {
            int v;
            for (;;) {
                v = ld_relaxed(sync + SY_ABORT) ? m.total : atomicAdd(sync + SY_HEAD, 1);
                if (v < m.b4 || v >= m.total) break;
                if (s_nact < 0) {
                    if (ld_relaxed(sync + SY_BUCKET) < 1) break;  // not known yet: run it (it checks)
                    fence_acq_rel_gpu();
                    s_nact = a.meta->n_active;
                }
                if (v < m.b5) {
                    if ((v - m.b4) / m.FT < s_nact) break;
                    atomicMax(sync + SY_HEAD, m.b5);  // no gate/up work left: go to the down tasks
                    continue;
                }
                if ((v - m.b5) / m.nRTG < s_nact) break;
                atomicMax(sync + SY_HEAD, m.total);  // no down work left
                v = m.total;
                break;
            }
            s_claim = v;
        }
        __syncthreads();
        const int v = s_claim;
        __syncthreads();
        return v;
    };
    // Stage a task's operands into buffer `buf`.  Routed tasks need the
    // bucketing: the first one a CTA meets waits for it (blocking) or gives up
    // (returns false) when it is not published yet; then all threads copy the
    // slot table into shared memory once, and every later routed task reads it
    // there instead of chasing active -> offsets -> pairs in global memory.
    int* tbl = reinterpret_cast<int*>(p.R[1] + a.buf_bytes);
    bool tbl_ready = false;
    auto prepare = [&](int task, int buf, bool blocking) {
        const Task t = decode_task(m, task);
        if ((t.kind == K_RGU || t.kind == K_RDN) && !tbl_ready) {
            if (threadIdx.x == 0) {
                int ok = 1;
                if (blocking) ok = wait_geq(sync + SY_BUCKET, 1, sync, a.status) ? 1 : 0;
                else if (ld_relaxed(sync + SY_BUCKET) >= 1) fence_acq_rel_gpu();
                else ok = -1;
                s_flag = ok;
            }
            __syncthreads();
            const int f = s_flag;
            __syncthreads();
            if (f == -1) return false;
            if (f == 1) {
                const int nact = a.meta->n_active, npairs = a.offsets[a.E];
                for (int i = threadIdx.x; i < nact; i += kDecThreads) {
                    const int e = a.active[i], p0 = a.offsets[e];
                    tbl[2 + i] = e;
                    tbl[2 + m.maxR + i] = p0;
                    tbl[2 + 2 * m.maxR + i] = a.offsets[e + 1] - p0;
                }
                for (int q = threadIdx.x; q < npairs; q += kDecThreads) tbl[2 + 3 * m.maxR + q] = a.pairs[q] / a.k;
                if (threadIdx.x == 0) {
                    tbl[0] = nact;
                    tbl[1] = npairs;
                }
                __syncthreads();
                tbl_ready = true;
            }
        }
        if (threadIdx.x == 0) s_issued[buf] = issue_task<BITS, STAGE>(a, m, t, p, buf, tbl_ready ? tbl : nullptr);
        __syncthreads();
        return true;
    };
    auto run = [&](int task, int buf) {
        const Task t = decode_task(m, task);
        uint8_t* W = p.R[buf];
        uint16_t* A = reinterpret_cast<uint16_t*>(p.R[buf] + p.w_bytes);
        const bool staged = s_issued[buf] != 0;
        bool ok = true;
        if (staged) ok = stage_wait(&p.bar[buf], p.phase[buf], a);
        switch (t.kind) {
            case K_ROUTER: {
                const int e0 = t.idx * kRouterRows, nrow = min(kRouterRows, a.E - e0);
                double* part = reinterpret_cast<double*>(red);
                for (int t0 = 0; t0 < a.T; t0 += 8) {
                    const int nt = min(8, a.T - t0);
                    if (t0 > 0) {  // next chunk of activation rows
                        __syncthreads();
                        if (threadIdx.x == 0) {
                            fence_proxy_async_smem();
                            mbar_arrive_expect_tx(&p.bar[buf], (uint32_t)nt * a.d * 2);
                            for (int q = 0; q < nt; ++q)
                                bulk_g2s(A + q * (a.d + kPad), a.x + (int64_t)(t0 + q) * a.d, a.d * 2, &p.bar[buf]);
                        }
                        ok = stage_wait(&p.bar[buf], p.phase[buf], a) && ok;
                    }
                    if (ok) router_compute(a, e0, nrow, t0, nt, reinterpret_cast<const uint16_t*>(W), A, part, warp,
                                           lane);
                    __syncthreads();
                }
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) red_add_release(sync + SY_ROUTER, 1);
                break;
            }
            case K_SGU:
            case K_RGU: {
                if (!staged) break;  // an expert slot beyond the active ones
                const int slot = t.kind == K_SGU ? 0 : a.n_shared + t.sidx;
                const Slot sl = make_slot(a, slot, tbl_ready ? tbl : nullptr, m.maxR);
                if (ok) gateup_compute<BITS, NT, STAGE>(a, sl, t.idx, red, W, A, warp, lane);
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) red_add_release(slot_done + slot, 1);
                break;
            }
            case K_TOPK: {
                if (threadIdx.x == 0) s_flag = wait_geq(sync + SY_ROUTER, m.nRt, sync, a.status) ? 1 : 0;
                __syncthreads();
                const int tk = t.idx * kDecWarps + warp;
                int* ids_s = reinterpret_cast<int*>(red);  // [8 x k] ids of this CTA's tokens
                // all warps copy the logits of the CTA's tokens (one load round trip),
                // then warp w ranks token t.idx * 8 + w
                const int ntk = min(kDecWarps, a.T - t.idx * kDecWarps);
                double* vb = reinterpret_cast<double*>(p.R[buf]);
                if (s_flag) {
                    const double* lg = a.logits64 + (int64_t)t.idx * kDecWarps * a.E;
#pragma unroll 4
                    for (int i = threadIdx.x; i < ntk * a.E; i += kDecThreads) vb[i] = lg[i];
                }
                __syncthreads();
                if (s_flag && tk < a.T) topk_token(a, tk, lane, vb + warp * a.E, ids_s + warp * a.k);
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0) {
                    const int ntok = min(kDecWarps, a.T - t.idx * kDecWarps);
                    s_flag = (atom_add_acqrel(sync + SY_TOPK, ntok) + ntok == a.T) ? 1 : 0;
                }
                __syncthreads();
                if (s_flag) {
                    bucket_cta(a, reinterpret_cast<int*>(p.R[buf]), a.T <= kDecWarps ? ids_s : nullptr);
                    __threadfence();
                    __syncthreads();
                    if (threadIdx.x == 0) st_release(sync + SY_BUCKET, 1);
                }
                break;
            }
            default: {  // K_SDN, K_RDN
                if (!staged) break;
                const int slot = t.kind == K_SDN ? 0 : a.n_shared + t.sidx;
                if (threadIdx.x == 0) {
                    s_flag = wait_geq(slot_done + slot, m.FT, sync, a.status) ? 1 : 0;
                    if (s_flag && t.kind == K_SDN) s_flag = wait_geq(sync + SY_BUCKET, 1, sync, a.status) ? 1 : 0;
                }
                __syncthreads();
                const Slot sl = make_slot(a, slot, (t.kind == K_RDN && tbl_ready) ? tbl : nullptr, m.maxR);
                if (STAGE && s_flag) {
                    stage_h_rows(a, sl, A);
                    __syncthreads();
                }
                if (ok && s_flag) down_compute<BITS, NT, STAGE>(a, sl, t.idx, m.RT16, W, A, warp, lane);
                break;
            }
        }
        __syncthreads();
    };

    int b = 0;
    int cur = claim();
    if (cur < m.total) prepare(cur, b, true);
    while (cur < m.total) {
        const int nxt = claim();
        bool ready = false;
        if (nxt < m.total) ready = prepare(nxt, b ^ 1, false);
        run(cur, b);
        if (nxt < m.total && !ready) prepare(nxt, b ^ 1, true);
        cur = nxt;
        b ^= 1;
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
// Shared memory: [gate/up reduction] 2 x [staged weights: max of router rows,
// gate/up tile, down task | activations: max of router x chunk, gate/up x rows,
// down h rows, top-k buffers (8 warps x 2E floats), bucket (2E + 1 + T*k ints)]
// [slot table].
static size_t round128(size_t n) { return (n + 127) & ~size_t(127); }

static size_t decode_smem(int BITS, int NT, int d, int f, int E, int T, int k, int* red_b, int* buf_b, int* w_b) {
    const bool stage = NT <= 2;
    const size_t tb = 256 * (size_t)BITS + 128;
    const size_t red = round128(std::max((size_t)NT * kDecWarps * 2 * 4 * 32 * 4, (size_t)kRouterRows * 2 * 8 * 8));
    size_t w = (size_t)kRouterRows * d * 2;
    w = std::max(w, 2 * (size_t)(d / 128) * tb);
    w = std::max(w, (size_t)kDecWarps * (f / 128) * tb);
    w = round128(w);
    const size_t rows = (size_t)std::min(T, 8 * NT);
    size_t act = (size_t)std::min(T, 8) * (d + kPad) * 2;  // router chunk
    if (stage) {
        act = std::max(act, rows * (d + kPad) * 2);
        act = std::max(act, rows * (f + kPad) * 2);
    }
    size_t buf = w + round128(act);
    buf = std::max(buf, (size_t)kDecWarps * E * 8);                          // top-k
    buf = std::max(buf, (size_t)(2 * E + 1 + T * k + 3 * kDecWarps) * 4);    // bucket
    buf = round128(buf);
    *red_b = (int)red;
    *buf_b = (int)buf;
    *w_b = (int)w;
    const size_t tbl = round128(4 * slot_table_words(std::min(T * k, E), T * k));  // the CTA's slot table
    return red + 2 * buf + tbl;
}

template <int BITS, int NT>
static cudaError_t decode_bits_nt(const DecodeLaunch& L, cudaStream_t st) {
    auto kern = decode_kernel<BITS, NT>;
    int red_b = 0, buf_b = 0, w_b = 0;
    const size_t smem = decode_smem(BITS, NT, L.d, L.f, L.E, L.T, L.k, &red_b, &buf_b, &w_b);
    static int blocks_per_sm[64] = {};  // per device, looked up once per shared-memory size
    static size_t smem_seen[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (smem != smem_seen[dev]) {
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kDecThreads, smem);
        if (e != cudaSuccess) return e;
        blocks_per_sm[dev] = nb > 0 ? nb : 1;
        smem_seen[dev] = smem;
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
    a.skip_rank = L.skip_rank;
    a.e_begin = max(0, L.e_begin);
    a.e_end = min(L.E, L.e_end);
    a.red_bytes = red_b;
    a.buf_bytes = buf_b;
    a.w_bytes = w_b;
    const int grid = blocks_per_sm[dev] * sms;
    kern<<<grid, kDecThreads, smem, st>>>(a);
    return cudaGetLastError();
}

static int max_smem_optin() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 227 * 1024;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 227 * 1024;
    return v;
}

static bool fits(int BITS, int NT, const DecodeLaunch& L) {
    int r, b, w;
    return decode_smem(BITS, NT, L.d, L.f, L.E, L.T, L.k, &r, &b, &w) <= (size_t)max_smem_optin();
}

// Tokens per task: the smallest of 1, 2, 4, 8 that covers T in 8 slots and
// whose shared memory fits; a batch that fits no variant runs as 32-token
// slices (each slice a full layer pass over its own tokens).
template <int BITS>
static cudaError_t decode_bits(const DecodeLaunch& L, cudaStream_t s) {
    if (L.T <= 8 && fits(BITS, 1, L)) return decode_bits_nt<BITS, 1>(L, s);
    if (L.T <= 16 && fits(BITS, 2, L)) return decode_bits_nt<BITS, 2>(L, s);
    if (L.T <= 32 && fits(BITS, 4, L)) return decode_bits_nt<BITS, 4>(L, s);
    if (fits(BITS, 8, L)) return decode_bits_nt<BITS, 8>(L, s);
    const size_t ysz = L.out_fp32 ? 4 : 2;
    for (int t0 = 0; t0 < L.T; t0 += 32) {
        DecodeLaunch S = L;
        S.T = std::min(32, L.T - t0);
        S.x = static_cast<const uint16_t*>(L.x) + (size_t)t0 * L.d;
        S.y = static_cast<char*>(L.y) + (size_t)t0 * L.d * ysz;
        S.ids = L.ids + (size_t)t0 * L.k;
        S.w = L.w + (size_t)t0 * L.k;
        if (!fits(BITS, 4, S)) return cudaErrorInvalidConfiguration;
        cudaError_t e = decode_bits_nt<BITS, 4>(S, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
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

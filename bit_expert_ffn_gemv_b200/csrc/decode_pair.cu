// decode_pair.cu -- the whole routed-MoE layer for up to 16 tokens in ONE launch
// of 148 CTAs (74 clusters of two, one CTA per SM).
//
// A decode or draft-verify batch (one token plus up to three drafts; the layer
// the Strata pages run per generated token: the router picks the experts, the
// GPU combines their results, then moves to the next layer -- discuss.pytorch.kr
// post, section "Strata's operating principle") touches ~18 MB of packed
// expert weights per token, a few microseconds of HBM time.  The launch is
// shaped so that those bytes stream at full bandwidth behind a short chain of
// hand-offs:
//
//   1. Router.  CTA b computes the exact logits of experts [bE/G, (b+1)E/G)
//      for all T tokens (bf16 x bf16 products are exact in fp64, summed by
//      fp64 FMAs; a warp task is one row, four tokens, half the input
//      dimension), writes them to global memory and announces them on a
//      64-bit arrival counter.  Clusters whose first work units belong to the
//      shared expert run those units' gate/up meanwhile (no routing needed).
//   2. Top-k and schedule, redundantly in every CTA, once all CTAs arrived:
//      each warp ranks one token's E logits (k + 1 warp max-reductions over
//      unique 32-bit keys; fp64 ranking only where keys share a prefix; ties
//      to the lower index, exact rank order), then the CTA lists the active
//      experts ("slots": the shared expert, then the selected routed experts
//      in ascending order) and the work units.  No second grid-wide hand-off
//      is needed before the experts.  This code runs once per launch, so it is
//      kept short: cold instructions stream from L2.
//   3. Work units, pipelined (gate/up of unit i, then down of unit i - 1; one
//      loop for the shared-expert units, the routing step and the routed
//      units).  Unit u = (slot u / (f/128), chunk j = u % (f/128)) covers
//      the 128 intermediate rows [128j, 128j + 128) of one expert: its gate/up
//      rows and the matching 128 input columns of its down matrix.  Cluster c
//      takes units c, c + 74, c + 148, ...  Inside the cluster, CTA r computes
//      gate/up rows [64r, 64r + 64) of the chunk (warp w: 16-row tile w/2 of
//      gate (w even) or up (w odd) over the whole input dimension), writes the
//      h rows into both CTAs' shared memory, and multiplies the chunk's 128 h
//      values by down rows [r d/2, (r+1) d/2).  Every expert byte is read
//      once and h never leaves the cluster.  The down partial sums, times the
//      routing weight, are stored (no atomics) per (token, slot, chunk).
//   4. Combine.  After a second arrival count, every CTA sums a slice of the
//      partial sums in a fixed order (slot, then chunk) and writes y, so the
//      result does not depend on timing.
//
// Warp 8 is the producer: it moves the weights by bulk copies (TMA) into two
// rings of shared-memory slots (gate/up items: one 16-row tile of gate and of
// up; down items: d/64 row tiles x one 128-column super-tile, fetched through
// a 3-D tensor map), as far ahead as the rings allow.  Warps 0-7 compute:
// warp MMAs on exact 16-bit integer codes (bf16 for gate/up against bf16 x,
// fp16 for down against fp16 h) with the fp16 block scale applied in fp32 per
// 32-block.  Slots, h buffers and the pair's h exchange are tracked by
// mbarriers (the peer's h rows arrive by st.async stores that complete
// bytes on this CTA's barrier), so no wait involves the producer and the
// consumers together.
//
// Every wait is bounded: an mbarrier or counter wait gives up after a limit,
// sets the status word and carries on (a copy wait then waits once more,
// bounded, for its bytes).  The only hardware cluster barriers are one at the
// start and one at the end, run by every thread.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace pair {

constexpr int kCWarps = 8;                 // compute (consumer) warps
constexpr int kConsumers = kCWarps * 32;
constexpr int kProducer = kCWarps;         // warp index of the producer
constexpr int kThreads = kConsumers + 32;
constexpr int kCS = 2;                     // CTAs per cluster
constexpr int kMaxSlots = 16;              // ring slots of each kind (upper bound)
constexpr int kXPad = 32;                  // 16-bit elements of padding per staged row
constexpr int kHRow = 128 + kXPad;
constexpr int kCandBytes = 64 * 16;        // per-warp top-k candidate buffer
constexpr int kMaxKS = 2;                  // input super-tiles per warp of a gate/up tile (d <= 2048)
constexpr int kRouterIt = 4;               // 16-byte router loads per lane per half row (d <= 2048)

// Optional phase trace (build with -DMOE_PAIR_TRACE): thread 0 of every CTA
// records the global timer at phase boundaries and adds clock64() differences
// per phase into shared memory (no global round trip inside a phase), written
// out once at the end; moe_debug_pair_trace() / moe_debug_pair_cycles() copy
// them to the host.
#ifdef MOE_PAIR_TRACE
constexpr int kTraceSlots = 48;
__device__ unsigned long long g_trace[1024 * kTraceSlots];
__device__ unsigned long long g_cyc[1024 * 32];
MOE_DEV unsigned long long* cyc_acc() {
    __shared__ unsigned long long acc[32];
    return acc;
}
MOE_DEV void trace(int slot) {
    if (threadIdx.x == 0 && slot < kTraceSlots) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_trace[blockIdx.x * kTraceSlots + slot] = t;
    }
}
MOE_DEV unsigned long long cyc() { return (unsigned long long)clock64(); }
MOE_DEV void cyc_add(int slot, unsigned long long t0) {
    if (threadIdx.x == 0) cyc_acc()[slot] += cyc() - t0;
}
MOE_DEV void cyc_reset() {
    if (threadIdx.x == 0)
        for (int i = 0; i < 32; ++i) cyc_acc()[i] = 0;
}
MOE_DEV void cyc_flush() {
    if (threadIdx.x == 0)
        for (int i = 0; i < 32; ++i) g_cyc[blockIdx.x * 32 + i] = cyc_acc()[i];
}
#else
MOE_DEV void trace(int) {}
MOE_DEV unsigned long long cyc() { return 0; }
MOE_DEV void cyc_add(int, unsigned long long) {}
MOE_DEV void cyc_reset() {}
MOE_DEV void cyc_flush() {}
#endif

struct Args {
    int T, d, f, E, k, n_shared;
    const uint16_t* x;  // bf16 [T x d]
    void* y;
    int out_fp32, accumulate;
    const uint8_t* codes;
    const uint16_t* scales;
    int64_t code_stride;   // code bytes per expert (gate, up, down)
    int64_t scale_stride;  // fp16 scales per expert
    const uint16_t* wr;    // bf16 [E x d]
    const float* bias;
    double* logits64;      // [T x E]
    int32_t* ids;          // [T x k] (written by CTA 0)
    float* w;
    Meta* meta;
    uint32_t* status;
    float* part;           // [T x (k + n_shared) x f/128 x d] partial sums
    unsigned long long* ctr;  // [0] router arrivals, [1] partial sums written
    int skip_rank;
    int e_begin, e_end;
    int nc;                // clusters in the grid
    uint32_t spin_limit;   // polls before a wait gives up
    int withhold;          // test only: this CTA never announces its router rows (-1: off)
    int norm_input;        // normalise x (rmsnorm, as launch_rms_normalize) before the router
    // shared memory layout (bytes from the dynamic base)
    int ng, nd;            // ring slots
    int g_bytes, d_bytes;  // item sizes
    int off_x, off_h, off_gus, off_cand, off_route, off_emask, off_slots, off_pos, off_g, off_d;
};

// ---------------------------------------------------------------- cluster, mbarrier and memory-order helpers
MOE_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
MOE_DEV uint32_t cluster_idx() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
MOE_DEV void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
MOE_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
MOE_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
// address of the same shared-memory location in CTA `rank` of the cluster
MOE_DEV uint32_t peer_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
MOE_DEV void fence_mbar_init_cluster() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// store 4 bytes into the peer's shared memory; the store completes 4 bytes
// of transactions on the peer's mbarrier (no fence needed before the peer reads)
MOE_DEV void st_async_remote(uint32_t addr, uint32_t v, uint32_t bar_addr) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
                 "r"(bar_addr)
                 : "memory");
}
MOE_DEV void mbar_arrive_relaxed_remote(uint32_t addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
MOE_DEV bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, "
        "p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
MOE_DEV unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
MOE_DEV unsigned long long atom_add_acqrel_u64(unsigned long long* p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.add.acq_rel.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}
MOE_DEV void fence_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
MOE_DEV void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// Bounded waits.  A copy wait that gives up waits once more (bounded) so that
// no copy is still landing when the caller moves on.
MOE_DEV void copy_wait(uint64_t* bar, uint32_t parity, const Args& a) {
    for (uint32_t it = 0; it <= a.spin_limit; ++it)
        if (mbar_try_wait(bar, parity)) return;
    if ((threadIdx.x & 31) == 0) flag_status(a.status, kStatusTimeout);
    for (uint32_t it = 0; it <= a.spin_limit; ++it)
        if (mbar_try_wait(bar, parity)) return;
}
MOE_DEV void slot_wait(uint64_t* bar, uint32_t parity, const Args& a) {
    for (uint32_t it = 0; it <= a.spin_limit; ++it)
        if (mbar_try_wait(bar, parity)) return;
    if ((threadIdx.x & 31) == 0) flag_status(a.status, kStatusTimeout);
}
MOE_DEV void pair_wait(uint64_t* bar, uint32_t parity, const Args& a) {
    for (uint32_t it = 0; it <= a.spin_limit; ++it)
        if (mbar_try_wait_cluster(bar, parity)) return;
    if ((threadIdx.x & 31) == 0) flag_status(a.status, kStatusTimeout);
}
// One thread per CTA: add this CTA's arrival (unless withheld) to a counter
// that only grows; the launch's full count is the next multiple of the grid
// size above the value found at arrival.
MOE_DEV unsigned long long grid_arrive(unsigned long long* ctr, bool arrive) {
    const unsigned long long G = gridDim.x;
    fence_gpu();
    const unsigned long long old = arrive ? atom_add_acqrel_u64(ctr, 1ull) : ld_acquire_u64(ctr);
    return (old / G + 1ull) * G;
}
MOE_DEV void grid_wait(const unsigned long long* ctr, unsigned long long target, const Args& a) {
    uint32_t ns = 32;
    for (uint32_t it = 0; it <= a.spin_limit; ++it) {
        if (ld_acquire_u64(ctr) >= target) return;
        if (it >= 32) {  // back-to-back polls first (the usual wait is a few of them), then back off
            __nanosleep(ns);
            if (ns < 128) ns <<= 1;
        }
    }
    flag_status(a.status, kStatusTimeout);
}

// ---------------------------------------------------------------- code decoding (faster form, 2-bit)
// Each A-fragment register holds two codes u at bits [2p, 2p+1] and
// [16+2p, 17+2p] of the lane's 32-bit code word.  Instead of shifting every
// pair down to bit 0, the word is masked in place and OR-ed into a 16-bit
// float whose exponent makes bit 2p the unit: 2^E + u exactly; subtracting
// 2^E + 2 leaves q = u - 2 exactly.  Pairs whose bits reach the exponent
// field are first shifted down once.
//   bf16 (7 mantissa bits): bits 0-1, 2-3, 4-5 with 2^E = 128, 32, 8
//   fp16 (10 mantissa bits): bits 0-1 .. 8-9 with 2^E = 1024, 256, 64, 16, 4
template <bool F16>
MOE_DEV uint32_t sub2(uint32_t v, uint32_t c) {
    uint32_t r;
    if (F16)
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(c));
    else
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(c));
    return r;
}
MOE_DEV uint32_t dup16(uint32_t h) { return h | (h << 16); }

template <bool F16>
MOE_DEV void decode2_fast(uint32_t lo, uint32_t (&q)[8]) {
    if (F16) {
        const uint32_t s10 = lo >> 10;
        q[0] = sub2<true>((lo & 0x00030003u) | dup16(0x6400u), dup16(0x6402u));
        q[1] = sub2<true>((lo & 0x000C000Cu) | dup16(0x5C00u), dup16(0x5C08u));
        q[2] = sub2<true>((lo & 0x00300030u) | dup16(0x5400u), dup16(0x5420u));
        q[3] = sub2<true>((lo & 0x00C000C0u) | dup16(0x4C00u), dup16(0x4C80u));
        q[4] = sub2<true>((lo & 0x03000300u) | dup16(0x4400u), dup16(0x4600u));
        q[5] = sub2<true>((s10 & 0x00030003u) | dup16(0x6400u), dup16(0x6402u));
        q[6] = sub2<true>((s10 & 0x000C000Cu) | dup16(0x5C00u), dup16(0x5C08u));
        q[7] = sub2<true>((s10 & 0x00300030u) | dup16(0x5400u), dup16(0x5420u));
    } else {
        const uint32_t s6 = lo >> 6, s12 = lo >> 12;
        q[0] = sub2<false>((lo & 0x00030003u) | dup16(0x4300u), dup16(0x4302u));
        q[1] = sub2<false>((lo & 0x000C000Cu) | dup16(0x4200u), dup16(0x4208u));
        q[2] = sub2<false>((lo & 0x00300030u) | dup16(0x4100u), dup16(0x4120u));
        q[3] = sub2<false>((s6 & 0x00030003u) | dup16(0x4300u), dup16(0x4302u));
        q[4] = sub2<false>((s6 & 0x000C000Cu) | dup16(0x4200u), dup16(0x4208u));
        q[5] = sub2<false>((s6 & 0x00300030u) | dup16(0x4100u), dup16(0x4120u));
        q[6] = sub2<false>((s12 & 0x00030003u) | dup16(0x4300u), dup16(0x4302u));
        q[7] = sub2<false>((s12 & 0x000C000Cu) | dup16(0x4200u), dup16(0x4208u));
    }
}

template <bool F16, int BITS>
MOE_DEV void decode_any(uint32_t lo, uint32_t hi, uint32_t (&q)[8]) {
    if (BITS == 2)
        decode2_fast<F16>(lo, q);
    else
        decode_block<F16, BITS>(lo, hi, q);
}

MOE_DEV void scale_acc(float (&acc)[4], const float (&t)[4], uint32_t sc) {
    const float slo = __half2float(__ushort_as_half((unsigned short)(sc & 0xFFFFu)));
    const float shi = __half2float(__ushort_as_half((unsigned short)(sc >> 16)));
    acc[0] = fmaf(slo, t[0], acc[0]);
    acc[1] = fmaf(slo, t[1], acc[1]);
    acc[2] = fmaf(shi, t[2], acc[2]);
    acc[3] = fmaf(shi, t[3], acc[3]);
}

// position of element k (0..31) of a 32-element block in the staged row layout:
// the four pairs a lane's B fragment needs (k = 2c + 8j + e, j = 0..3) sit
// together at 8c + 2j + e, so one 16-byte load fetches them.
MOE_DEV int perm32(int k) { return ((k & 7) >> 1) * 8 + (k >> 3) * 2 + (k & 1); }

// ---------------------------------------------------------------- top-k of one token (warp)
MOE_DEV uint64_t order_key64(double v) {
    if (isnan(v)) v = -INFINITY;
    v = v + 0.0;  // -0 -> +0
    const uint64_t b = (uint64_t)__double_as_longlong(v);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
MOE_DEV bool better64(uint64_t ka, int ia, uint64_t kb, int ib) { return ka > kb || (ka == kb && ia < ib); }
// 32-bit key: order-preserving image of fp32(l) with the low 10 bits replaced
// by 1023 - e.  A strictly larger prefix (the upper 22 bits) means a strictly
// larger logit; keys are unique.
MOE_DEV uint32_t key32(double v, int e) {
    float f = (float)(isnan(v) ? -INFINITY : v);
    f = f + 0.0f;
    const uint32_t b = __float_as_uint(f);
    const uint32_t o = (b >> 31) ? ~b : (b | 0x80000000u);
    return (o & 0xFFFFFC00u) | (uint32_t)(1023 - e);
}

struct Cand {
    double v;
    int e;
    int pad;
};

// Slow exact selection (when more than 32 logits share the candidate prefix).
MOE_DEV void topk_scan(const double* lg, int E, int k, int lane, int& sel, double& lsel, double& top) {
    int prev_e = -1;
    uint64_t prev_k = 0;
    for (int r = 0; r < k; ++r) {
        uint64_t bk = 0;
        int bi = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const uint64_t ke = order_key64(__ldcg(lg + e));
            if (prev_e >= 0 && !better64(prev_k, prev_e, ke, e)) continue;  // not strictly worse than the last pick
            if (bi == 0x7fffffff || better64(ke, e, bk, bi)) {
                bk = ke;
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi != 0x7fffffff && (bi == 0x7fffffff || better64(ok, oi, bk, bi))) {
                bk = ok;
                bi = oi;
            }
        }
        const double lv = __ldcg(lg + bi);
        if (lane == r) {
            sel = bi;
            lsel = lv;
        }
        if (r == 0) top = lv;
        prev_e = bi;
        prev_k = bk;
    }
}

// Exact top-k of one token's E fp64 logits (global memory, read through L2).
// Each lane holds KPL logits and their 32-bit keys (fp32 prefix | 1023 - e,
// unique).  Rounds r = 0 .. k take the warp's largest remaining key with one
// max-reduction; the index is read back from the key, and the lane that held
// it parks (logit, index) at cand[r] and drops the key.  The k largest keys
// are the exact top k when the k-th key's prefix is strictly above the
// (k+1)-th's: every logit left behind then has a smaller prefix than each
// selected one, hence a smaller value.  Their order is the keys' order when
// adjacent prefixes differ; where two selected keys share a prefix the k
// entries are ranked again by (fp64 logit desc, index asc).  A tie of the
// k-th and (k+1)-th prefixes (rare: equal fp32 images) takes the exact
// scan.  Lane r < k returns id r and l_r - l_0 (its logit less the top one),
// from which w_r = softmax over the k selected logits is finished later.
template <int KPL>
MOE_DEV void topk_token(const double* lg, int E, int k, int lane, Cand* cand, int& id_out, float& w_out) {
    unsigned long long tc = cyc();
    double v[KPL];
    uint32_t key[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) v[j] = __ldcg(lg + min(lane + 32 * j, E - 1));
    uint32_t lmax = 0u;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const int e = lane + 32 * j;
        key[j] = e < E ? key32(v[j], e) : 0u;
        lmax = max(lmax, key[j]);
    }
    cyc_add(10, tc);  // loads + keys
    tc = cyc();
    const int rounds = min(k + 1, E);
    uint32_t my_key = 0u;       // lane r < k: the r-th largest key
    uint32_t pk = 0u, pn = 0u;  // prefixes of the k-th and (k+1)-th largest keys
    for (int r = 0; r < rounds; ++r) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, lmax);
        if (lane == r) my_key = m;
        if (r == k - 1) pk = m & 0xFFFFFC00u;
        if (r == k) pn = m & 0xFFFFFC00u;
        // the holder of key m (keys are unique: one lane, one j) parks it
        lmax = 0u;
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
            if (key[j] == m) {
                cand[r].v = v[j];
                cand[r].e = 1023 - (int)(m & 1023u);
                key[j] = 0u;
            }
            lmax = max(lmax, key[j]);
        }
    }
    __syncwarp();
    cyc_add(11, tc);  // k + 1 extraction rounds
    tc = cyc();
    int sel = -1;
    double lsel = 0.0, top = 0.0;
    if (rounds == k || pk > pn) {
        double my_v = 0.0;
        int my_e = 0;
        if (lane < k) {
            my_v = cand[lane].v;
            my_e = cand[lane].e;
        }
        // adjacent selected keys with one prefix: rank the k exactly
        const uint32_t prev = __shfl_up_sync(0xffffffffu, my_key, 1);
        const bool tie = lane >= 1 && lane < k && (prev & 0xFFFFFC00u) == (my_key & 0xFFFFFC00u);
        if (__any_sync(0xffffffffu, tie)) {
            int rank = 0;
            if (lane < k) {
                const uint64_t mk = order_key64(my_v);
                for (int j = 0; j < k; ++j) {
                    const Cand o = cand[j];
                    if (j != lane && better64(order_key64(o.v), o.e, mk, my_e)) ++rank;
                }
            }
            __syncwarp();
            if (lane < k) {
                cand[32 + rank].v = my_v;
                cand[32 + rank].e = my_e;
            }
            __syncwarp();
            if (lane < k) {
                my_v = cand[32 + lane].v;
                my_e = cand[32 + lane].e;
            }
        }
        sel = lane < k ? my_e : -1;
        lsel = my_v;
        top = __shfl_sync(0xffffffffu, my_v, 0);
        cyc_add(13, tc);  // ranking
    } else {
        topk_scan(lg, E, k, lane, sel, lsel, top);
        cyc_add(15, tc);  // slow path taken
    }
    __syncwarp();  // cand is reused by the next token of this warp
    id_out = sel;
    // the weight's logit less the top one; the softmax is finished after the
    // schedule, which needs only the ids
    w_out = lane < k ? (float)(lsel - top) : 0.0f;
}

MOE_DEV double bf16_to_f64(uint32_t bits16) { return (double)__uint_as_float(bits16 << 16); }

// ---------------------------------------------------------------- the kernel
template <int BG, int BD, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const __grid_constant__ Args a, const __grid_constant__ CUtensorMap dmap_c,
                       const __grid_constant__ CUtensorMap dmap_s) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t fullG[kMaxSlots], emptyG[kMaxSlots], fullD[kMaxSlots], emptyD[kMaxSlots];
    __shared__ __align__(8) uint64_t hfull[3], hempty[3], barX, sched;
    __shared__ int s_nslots, s_nunits, s_stride, s_wcnt[kCWarps];
    __shared__ float s_w[2][16];
    __shared__ uint32_t s_mask[2];
    __shared__ int s_slot[2];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    trace(0);
    cyc_reset();
    const uint32_t rank = cluster_ctarank();
    const int q = (int)cluster_idx();
    const int nc = a.nc, G = (int)gridDim.x, b = (int)blockIdx.x;
    const int T = a.T, d = a.d, f = a.f, E = a.E, k = a.k, ns = a.n_shared;
    const int KT = d / 128, FC = f / 128, RT = d / 16, RTI = RT / 4, KS = k + ns;
    constexpr int GCB = 256 * BG, DCB = 256 * BD;  // code bytes of one super-tile
    const int64_t mg = (int64_t)f * d * BG / 8;    // code bytes of one gate/up matrix
    const int64_t msc = (int64_t)f * d / 32;       // scales of one matrix
    const int xstride = d + kXPad;

    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + a.off_x);     // [T][d + pad] bf16
    uint16_t* hb = reinterpret_cast<uint16_t*>(smem + a.off_h);     // [3][T][128 + pad] fp16, permuted
    float* gus = reinterpret_cast<float*>(smem + a.off_gus);        // gate/up outputs / router partials
    Cand* cand = reinterpret_cast<Cand*>(smem + a.off_cand);        // [8 warps][64]
    int* sids = reinterpret_cast<int*>(smem + a.off_route);         // [T * k]
    float* sw = reinterpret_cast<float*>(sids + T * k);             // [T * k]
    uint32_t* emask = reinterpret_cast<uint32_t*>(smem + a.off_emask);  // [E] tokens selecting e
    int* ebest = reinterpret_cast<int*>(emask + E);                 // [E] best rank of e in the batch
    int* slot_e = reinterpret_cast<int*>(smem + a.off_slots);       // [n_slots] expert of each slot
    int* tn = reinterpret_cast<int*>(smem + a.off_pos);             // [16] slots of token t
    unsigned char* pos = smem + a.off_pos + 64;                     // [n_slots][T] place of slot s in t's list
    uint8_t* gring = smem + a.off_g;
    uint8_t* dring = smem + a.off_d;

    if (tid == 0) {
        for (int i = 0; i < a.ng; ++i) {
            mbar_init(&fullG[i], 1);
            mbar_init(&emptyG[i], kCWarps);  // every warp reads its slice of every item
        }
        for (int i = 0; i < a.nd; ++i) {
            mbar_init(&fullD[i], 1);
            mbar_init(&emptyD[i], kCWarps);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(&hfull[i], 1);   // armed here with the bytes the peer's h stores bring
            mbar_init(&hempty[i], 1);  // the peer has read its copy of the buffer
        }
        mbar_init(&barX, 1);
        mbar_init(&sched, 1);
        fence_mbar_init_cluster();
        fence_proxy_async_smem();
    }
    for (int e = tid; e < E; e += kThreads) {
        emask[e] = 0u;
        ebest[e] = k;
    }
    if (tid == 0) s_stride = nc;
    __syncthreads();
    cluster_arrive();  // the peer's barriers are initialised once this completes (waited below)

    // ---- work units of this cluster: u = q + i * stride -> (slot u / FC, chunk u % FC).
    // The stride is nc until the schedule is known (the shared-expert units, slot
    // 0, are units 0 .. FC*ns - 1 of clusters 0 ..); the schedule may then keep
    // the routed units off the clusters that ran shared-expert units (stride
    // nc - FC*ns), which reach the routing step late.
    const int n_pre = (q < FC * ns) ? (FC * ns - 1 - q) / nc + 1 : 0;  // shared-expert units
    auto unit_expert = [&](int i, int& e, int& j, int& s) {
        const int u = q + i * s_stride;
        s = u / FC;
        j = u - s * FC;
        e = s < ns ? E : slot_e[s];
    };

    if (warp == kProducer) {
        // ================================================================ producer
        int item = 0;
        auto issue_items = [&](int end) {
            for (; item < end; ++item) {
                const int i = item / 6, r6 = item - 6 * i;
                int e, j, s;
                unit_expert(i, e, j, s);
                const uint8_t* ce = a.codes + (int64_t)e * a.code_stride;
                const uint8_t* se = reinterpret_cast<const uint8_t*>(a.scales + (int64_t)e * a.scale_stride);
                if (r6 < 4) {
                    const int gi = 4 * i + r6, sl = gi % a.ng, use = gi / a.ng;
                    if (use > 0) slot_wait(&emptyG[sl], (uint32_t)(use - 1) & 1u, a);
                    if (lane == 0) {
                        uint8_t* dst = gring + (size_t)sl * a.g_bytes;
                        const int rtg = 8 * j + 4 * (int)rank + r6;  // 16-row tile of the gate/up matrices
                        const uint32_t cb = KT * GCB, sb = KT * 128;
                        mbar_arrive_expect_tx(&fullG[sl], 2 * (cb + sb));
                        bulk_g2s(dst, ce + (int64_t)rtg * cb, cb, &fullG[sl]);
                        bulk_g2s(dst + cb, se + (int64_t)rtg * sb, sb, &fullG[sl]);
                        bulk_g2s(dst + cb + sb, ce + mg + (int64_t)rtg * cb, cb, &fullG[sl]);
                        bulk_g2s(dst + 2 * cb + sb, se + 2 * msc + (int64_t)rtg * sb, sb, &fullG[sl]);
                    }
                } else {
                    const int di = 2 * i + (r6 - 4), sl = di % a.nd, use = di / a.nd;
                    if (use > 0) slot_wait(&emptyD[sl], (uint32_t)(use - 1) & 1u, a);
                    if (lane == 0) {
                        // RTI row tiles x super-tile column j of expert e's down matrix
                        uint8_t* dst = dring + (size_t)sl * a.d_bytes;
                        const int rt0 = (int)rank * (RT / 2) + (r6 - 4) * RTI;
                        mbar_arrive_expect_tx(&fullD[sl], (uint32_t)RTI * (DCB + 128));
                        tma_load_3d(dst, &dmap_c, j * 64 * BD, rt0, e, &fullD[sl]);
                        tma_load_3d(dst + (size_t)RTI * DCB, &dmap_s, j * 64, rt0, e, &fullD[sl]);
                    }
                }
                __syncwarp();
            }
        };
        auto issue_until = [&](int n_units) { issue_items(6 * n_units); };
        if (lane == 0) {
            mbar_arrive_expect_tx(&barX, (uint32_t)T * d * 2);
            for (int t = 0; t < T; ++t) bulk_g2s(xs + t * xstride, a.x + (int64_t)t * d, d * 2, &barX);
        }
        __syncwarp();
        issue_until(n_pre);
        slot_wait(&sched, 0u, a);  // the consumers published the schedule
        issue_until(s_nunits);
        cluster_wait();  // the producer's half of the first cluster barrier
    } else {
        // ================================================================ consumers
        const unsigned long long c_start = cyc();
        // ---- 0. pre-norm (MOE_NORM_INPUT): x <- bf16(x / sqrt(mean(x^2) + 1e-6)) in
        // shared memory, token by token, with the same 256 threads, the same
        // order of fp32 operations and the same rounding as the stand-alone
        // norm kernel, so the result is bit-identical to it
        if (a.norm_input) {
            copy_wait(&barX, 0u, a);
            float* red = gus;
            for (int t = 0; t < T; ++t) {
                uint16_t* xr = xs + t * xstride;
                float ss = 0.f;
                for (int i = tid * 8; i < d; i += kConsumers * 8) {
                    const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
                    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const float lo = __uint_as_float(u[qq] << 16), hi = __uint_as_float(u[qq] & 0xFFFF0000u);
                        ss = fmaf(lo, lo, ss);
                        ss = fmaf(hi, hi, ss);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                if (lane == 0) red[warp] = ss;
                consumer_sync();
                float tot = 0.f;
#pragma unroll
                for (int w = 0; w < kCWarps; ++w) tot += red[w];
                const float inv = rsqrtf(tot / (float)d + 1e-6f);
                for (int i = tid * 8; i < d; i += kConsumers * 8) {
                    uint4* p4 = reinterpret_cast<uint4*>(xr + i);
                    const uint4 v = *p4;
                    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o4[4];
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) {
                        const __nv_bfloat162 r2 = __floats2bfloat162_rn(__uint_as_float(u[qq] << 16) * inv,
                                                                        __uint_as_float(u[qq] & 0xFFFF0000u) * inv);
                        o4[qq] = *reinterpret_cast<const uint32_t*>(&r2);
                    }
                    *p4 = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
                consumer_sync();  // red is reused by the next token; the router reads the normalised rows
            }
        }

        // ---- 1. router rows [r0, r1): exact logits.  Warp task = (row, 4
        // tokens, half of the input dimension): a lane holds 8 of every 256
        // inputs of its half (all its weight loads issued at once) and sums
        // exact bf16 products in fp64; the two halves meet in shared memory
        // and are added in a fixed order.
        {
            const int r0 = (int)((int64_t)b * E / G), r1 = (int)((int64_t)(b + 1) * E / G), R = r1 - r0;
            const int TG = (T + 3) / 4, NP = R * TG, hd = d / 2;
            double* part = reinterpret_cast<double*>(gus);  // [NP][2 halves][4 tokens]
            bool x_ready = false;
            for (int task = warp; task < 2 * NP; task += kCWarps) {
                const int pr = task >> 1, hf = task & 1;
                const int r = pr / TG, t0 = 4 * (pr - r * TG), nt4 = min(4, T - t0);
                const uint16_t* wrow = a.wr + (int64_t)(r0 + r) * d + hf * hd;
                uint4 wv[kRouterIt];
#pragma unroll
                for (int it = 0; it < kRouterIt; ++it) {
                    const int i = lane * 8 + 256 * it;
                    wv[it] = i < hd ? __ldg(reinterpret_cast<const uint4*>(wrow + i)) : make_uint4(0, 0, 0, 0);
                }
                if (!x_ready) {
                    copy_wait(&barX, 0u, a);
                    x_ready = true;
                }
                double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                for (int it = 0; it < kRouterIt; ++it) {
                    const int i = lane * 8 + 256 * it;
                    if (i < hd) {
                        const uint32_t wu[4] = {wv[it].x, wv[it].y, wv[it].z, wv[it].w};
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            if (t < nt4) {
                                const uint4 xv =
                                    *reinterpret_cast<const uint4*>(xs + (t0 + t) * xstride + hf * hd + i);
                                const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                                for (int h2 = 0; h2 < 4; ++h2) {
                                    acc[t] = fma(bf16_to_f64(wu[h2] & 0xFFFFu), bf16_to_f64(xu[h2] & 0xFFFFu), acc[t]);
                                    acc[t] = fma(bf16_to_f64(wu[h2] >> 16), bf16_to_f64(xu[h2] >> 16), acc[t]);
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
                if (lane < 4) {
                    double v = acc[0];
#pragma unroll
                    for (int t = 1; t < 4; ++t)
                        if (lane == t) v = acc[t];
                    part[(pr * 2 + hf) * 4 + lane] = v;
                }
            }
            if (!x_ready) copy_wait(&barX, 0u, a);  // a warp without router work
            consumer_sync();
            for (int idx = tid; idx < NP * 4; idx += kConsumers) {
                const int pr = idx >> 2, t = idx & 3, r = pr / TG, tt = 4 * (pr - r * TG) + t;
                if (tt < T) {
                    const int e = r0 + r;
                    const double bb = a.bias ? (double)a.bias[e] : 0.0;
                    a.logits64[(int64_t)tt * E + e] = (part[(pr * 2) * 4 + t] + part[(pr * 2 + 1) * 4 + t]) + bb;
                }
            }
            consumer_sync();  // every logit is written before thread 0 announces them
        }
        cyc_add(27, c_start);
        trace(1);
        // announce the logits (release), unless this CTA is the test's withheld one
        unsigned long long router_target = 0;
        if (tid == 0) router_target = grid_arrive(a.ctr, b != a.withhold);
        // x in place: permute every 32-element block so that a lane's B fragment
        // (pairs 2c + 8j, j = 0..3) is one 16-byte load (u32 pair 4j + c -> 4c + j)
        for (int blk = tid; blk < T * (d / 32); blk += kConsumers) {
            const int t = blk / (d / 32), kb = blk - t * (d / 32);
            uint4* p4 = reinterpret_cast<uint4*>(xs + t * xstride + kb * 32);
            const uint4 v0 = p4[0], v1 = p4[1], v2 = p4[2], v3 = p4[3];  // one thread per block
            p4[0] = make_uint4(v0.x, v1.x, v2.x, v3.x);
            p4[1] = make_uint4(v0.y, v1.y, v2.y, v3.y);
            p4[2] = make_uint4(v0.z, v1.z, v2.z, v3.z);
            p4[3] = make_uint4(v0.w, v1.w, v2.w, v3.w);
        }
        consumer_sync();
        cluster_wait();  // the peer is running and its barriers are initialised

        // routing weight and token mask of unit i's expert (kept for its down step)
        auto unit_weights = [&](int i) {
            if (warp != 0) return;
            int e, j, s;
            unit_expert(i, e, j, s);
            uint32_t bit = 0u;
            float wt = 0.f;
            if (lane < T) {
                if (e == E) {
                    wt = 1.f;
                    bit = 1u;
                } else {
                    for (int r = 0; r < k; ++r)
                        if (sids[lane * k + r] == e) {
                            wt = sw[lane * k + r];
                            bit = 1u;
                        }
                }
                s_w[i & 1][lane] = wt;
            }
            const uint32_t m = __ballot_sync(0xffffffffu, bit != 0u);
            if (lane == 0) {
                s_mask[i & 1] = m;
                s_slot[i & 1] = s;
            }
        };

        // ---- gate/up of unit i, one 16-row tile at a time: warp w adds its
        // slice of the input dimension for gate and up, the CTA sums the slices
        // and writes the tile's h rows into both CTAs' h buffer.
        auto gate_up = [&](int i) {
            const int hb3 = i % 3;
            // x fragments of this warp's slice of the input dimension (super-tiles
            // warp, warp + 8, ...), loaded once and used by all 8 tiles of the unit
            uint4 xf[kMaxKS][4][NT];
#pragma unroll
            for (int js = 0; js < kMaxKS; ++js)
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int st = warp + kCWarps * js, tok = nt * 8 + g;
                        xf[js][kb][nt] = (st < KT && tok < T) ? *reinterpret_cast<const uint4*>(
                                                                    xs + tok * xstride + st * 128 + kb * 32 + 8 * c)
                                                              : make_uint4(0, 0, 0, 0);
                    }
            unit_weights(i);
            // before writing the peer's copy of buffer hb3: the peer is done with unit i - 3
            if (tid == 0 && i >= 3) pair_wait(&hempty[hb3], (uint32_t)((i - 3) / 3) & 1u, a);
            const uint32_t peer_full = peer_addr(&hfull[hb3], rank ^ 1u);
            for (int qt = 0; qt < 4; ++qt) {
                const int gi = 4 * i + qt, sl = gi % a.ng, use = gi / a.ng;
                unsigned long long c0 = cyc();
                copy_wait(&fullG[sl], (uint32_t)use & 1u, a);
                cyc_add(1, c0);
                c0 = cyc();
                const uint8_t* gb = gring + (size_t)sl * a.g_bytes;
                const uint8_t* ub = gb + (size_t)KT * (GCB + 128);
                float accg[NT][4], accu[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) accg[nt][r] = accu[nt][r] = 0.f;
#pragma unroll
                for (int js = 0; js < kMaxKS; ++js) {
                    const int st = warp + kCWarps * js;
                    if (st < KT) {
                        TileRegs<BG> tg, tu;
                        load_tile_smem<BG>(gb + st * GCB, gb + KT * GCB + st * 128, lane, tg);
                        load_tile_smem<BG>(ub + st * GCB, ub + KT * GCB + st * 128, lane, tu);
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            uint32_t qq[8];
                            decode_any<false, BG>(tg.lo[kb], tg.hi[kb], qq);
                            {
                                const uint32_t q0[4] = {qq[0], qq[1], qq[2], qq[3]};
                                const uint32_t q1[4] = {qq[4], qq[5], qq[6], qq[7]};
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt) {
                                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                                    mma_bf16(t4, q0, xf[js][kb][nt].x, xf[js][kb][nt].y, t4);
                                    mma_bf16(t4, q1, xf[js][kb][nt].z, xf[js][kb][nt].w, t4);
                                    scale_acc(accg[nt], t4, tg.sc[kb]);
                                }
                            }
                            decode_any<false, BG>(tu.lo[kb], tu.hi[kb], qq);
                            {
                                const uint32_t q0[4] = {qq[0], qq[1], qq[2], qq[3]};
                                const uint32_t q1[4] = {qq[4], qq[5], qq[6], qq[7]};
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt) {
                                    float t4[4] = {0.f, 0.f, 0.f, 0.f};
                                    mma_bf16(t4, q0, xf[js][kb][nt].x, xf[js][kb][nt].y, t4);
                                    mma_bf16(t4, q1, xf[js][kb][nt].z, xf[js][kb][nt].w, t4);
                                    scale_acc(accu[nt], t4, tu.sc[kb]);
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&emptyG[sl]);  // this warp is done with the slot
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        gus[(((warp * 2 + 0) * NT + nt) * 4 + r) * 32 + lane] = accg[nt][r];
                        gus[(((warp * 2 + 1) * NT + nt) * 4 + r) * 32 + lane] = accu[nt][r];
                    }
                cyc_add(2, c0);
                c0 = cyc();
                consumer_sync();
                // h rows (2m2, 2m2 + 1) of tile qt and token n -> both CTAs' h buffer
                for (int id = tid; id < 8 * T; id += kConsumers) {
                    const int m2 = id & 7, n = id >> 3, nt = n >> 3;
                    float hv[2];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int m = 2 * m2 + e2;  // row within the 16-row tile
                        const int rr = 2 * (m >> 3) + (n & 1), ln = 4 * (m & 7) + ((n & 7) >> 1);
                        float gsum = 0.f, usum = 0.f;
#pragma unroll
                        for (int w = 0; w < kCWarps; ++w) {
                            gsum += gus[(((w * 2 + 0) * NT + nt) * 4 + rr) * 32 + ln];
                            usum += gus[(((w * 2 + 1) * NT + nt) * 4 + rr) * 32 + ln];
                        }
                        hv[e2] = silu(gsum) * usum;
                    }
                    const __half2 h2 = __floats2half2_rn(hv[0], hv[1]);
                    const uint32_t hw = *reinterpret_cast<const uint32_t*>(&h2);
                    const int rl = 64 * (int)rank + 16 * qt + 2 * m2;  // chunk-local row (even)
                    uint16_t* dst = hb + (hb3 * T + n) * kHRow + (rl & ~31) + perm32(rl & 31);
                    *reinterpret_cast<uint32_t*>(dst) = hw;
                    st_async_remote(peer_addr(dst, rank ^ 1u), hw, peer_full);
                }
                consumer_sync();  // the partial sums may be overwritten by the next tile
                cyc_add(3, c0);
            }
            // arm this CTA's barrier for the peer's 32 * T stores (their completion may come first)
            if (tid == 0) mbar_arrive_expect_tx(&hfull[hb3], 128u * (uint32_t)T);
        };

        // ---- down of unit i: the chunk's 128 h values times this CTA's d/2 down rows
        auto down = [&](int i) {
            const int hb3 = i % 3;
            unsigned long long c0 = cyc();
            pair_wait(&hfull[hb3], (uint32_t)(i / 3) & 1u, a);
            int e, j, s;
            unit_expert(i, e, j, s);
            const uint32_t mask = s_mask[i & 1];
            const int slot = s_slot[i & 1];
            const uint16_t* hbuf = hb + hb3 * T * kHRow;
            // the h fragments (the same for every down row tile) and, per token of
            // this lane, the routing weight and the partial-sum row (-1: none)
            uint4 hf[4][NT];
            int64_t pbase[NT][2];
            float wtok[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = nt * 8 + g;
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
                    hf[kb][nt] = tok < T ? *reinterpret_cast<const uint4*>(hbuf + tok * kHRow + kb * 32 + 8 * c)
                                         : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int t = nt * 8 + 2 * c + e2;
                    pbase[nt][e2] = -1;
                    wtok[nt][e2] = 0.f;
                    if (t < T && ((mask >> t) & 1u)) {
                        // the shared expert comes first in every token's list; the
                        // routed slots' places exist once the schedule is built
                        const int pl = slot < ns ? 0 : pos[slot * T + t];
                        if (pl < KS) {
                            pbase[nt][e2] = (((int64_t)t * KS + pl) * FC + j) * d;
                            wtok[nt][e2] = s_w[i & 1][t];
                        } else {
                            flag_status(a.status, kStatusBounds);
                        }
                    }
                }
            }
            const int di0 = 2 * i;
            copy_wait(&fullD[di0 % a.nd], (uint32_t)(di0 / a.nd) & 1u, a);
            copy_wait(&fullD[(di0 + 1) % a.nd], (uint32_t)((di0 + 1) / a.nd) & 1u, a);
            cyc_add(4, c0);
            c0 = cyc();
#pragma unroll
            for (int qi = 0; qi < 2; ++qi) {
                const int di = di0 + qi;
                const uint8_t* dc = dring + (size_t)(di % a.nd) * a.d_bytes;
                const uint8_t* ds = dc + (size_t)RTI * DCB;
                const int rt0 = (int)rank * (RT / 2) + qi * RTI;
#pragma unroll 2
                for (int lt = warp; lt < RTI; lt += kCWarps) {
                    TileRegs<BD> td;
                    load_tile_smem<BD>(dc + lt * DCB, ds + lt * 128, lane, td);
                    float acc[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) acc[nt][r] = 0.f;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        uint32_t qq[8];
                        decode_any<true, BD>(td.lo[kb], td.hi[kb], qq);
                        const uint32_t q0[4] = {qq[0], qq[1], qq[2], qq[3]}, q1[4] = {qq[4], qq[5], qq[6], qq[7]};
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            float t4[4] = {0.f, 0.f, 0.f, 0.f};
                            mma_f16(t4, q0, hf[kb][nt].x, hf[kb][nt].y, t4);
                            mma_f16(t4, q1, hf[kb][nt].z, hf[kb][nt].w, t4);
                            scale_acc(acc[nt], t4, td.sc[kb]);
                        }
                    }
                    // partial sums of (token, slot, chunk j) for output rows n, n + 8
                    const int n = (rt0 + lt) * 16 + g;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int e2 = r & 1;
                            if (pbase[nt][e2] >= 0) a.part[pbase[nt][e2] + n + 8 * (r >> 1)] = wtok[nt][e2] * acc[nt][r];
                        }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&emptyD[di0 % a.nd]);
                mbar_arrive(&emptyD[(di0 + 1) % a.nd]);
            }
            cyc_add(5, c0);
            consumer_sync();  // every warp is done with h buffer hb3: the peer may refill it
            if (tid == 0) mbar_arrive_relaxed_remote(peer_addr(&hempty[hb3], rank ^ 1u));
        };

        // ---- 2. every CTA's router rows, then top-k and the schedule (run once,
        // between the shared-expert units and the first routed unit); returns
        // this cluster's unit count
        auto routing = [&]() -> int {
            if (tid == 0) grid_wait(a.ctr, router_target, a);
            consumer_sync();
            trace(3);
            const unsigned long long ctk = cyc();
            for (int t = warp; t < T; t += kCWarps) {
                const double* lg = a.logits64 + (int64_t)t * E;
                int id;
                float wt;
                if (E <= 512)
                    topk_token<16>(lg, E, k, lane, cand + warp * 64, id, wt);
                else
                    topk_token<32>(lg, E, k, lane, cand + warp * 64, id, wt);
                if (lane < k) {
                    sids[t * k + lane] = id;
                    sw[t * k + lane] = wt;  // l_r - l_0 until the weights are finished
                    if (b == 0) a.ids[(int64_t)t * k + lane] = id;
                }
            }
            cyc_add(6, ctk);
            unsigned long long csc = cyc();
            consumer_sync();
            cyc_add(16, csc);  // wait for the other warps' top-k
            csc = cyc();
            trace(4);
            for (int p = tid; p < T * k; p += kConsumers) {
                const int e = sids[p], t = p / k, r = p - t * k;
                if (e >= 0 && e < E) {
                    atomicOr(&emask[e], 1u << t);
                    atomicMin(&ebest[e], r);
                } else {
                    flag_status(a.status, kStatusBounds);
                }
            }
            consumer_sync();
            {
                // kept experts in ascending order: warp w owns a contiguous chunk
                const int chunk = ((E + kCWarps - 1) / kCWarps + 31) & ~31;
                const int e0 = warp * chunk, e1 = min(E, e0 + chunk);
                auto keep = [&](int e) {
                    return e < e1 && emask[e] != 0u && !(a.skip_rank > 0 && ebest[e] >= a.skip_rank) &&
                           e >= a.e_begin && e < a.e_end;
                };
                int cnt = 0;
                for (int base = e0; base < e1; base += 32) cnt += __popc(__ballot_sync(0xffffffffu, keep(base + lane)));
                if (lane == 0) s_wcnt[warp] = cnt;
                consumer_sync();
                int p0 = ns;
                for (int w = 0; w < warp; ++w) p0 += s_wcnt[w];
                for (int base = e0; base < e1; base += 32) {
                    const bool kp = keep(base + lane);
                    const unsigned bal = __ballot_sync(0xffffffffu, kp);
                    if (kp) slot_e[p0 + __popc(bal & ((1u << lane) - 1u))] = base + lane;
                    p0 += __popc(bal);
                }
                if (tid == 0) {
                    int tot = ns;
                    for (int w = 0; w < kCWarps; ++w) tot += s_wcnt[w];
                    s_nslots = tot;
                }
                consumer_sync();
            }
            const int n_slots = s_nslots;
            cyc_add(17, csc);  // masks + compaction
            csc = cyc();
            // place of each slot in its tokens' lists (slot order): the partial sums'
            // row index.  Warp 0, lane = slot: per token, a ballot over the slots
            // that hold it gives each slot's place by a prefix count.
            if (warp == 0) {
                // tn[t] is the running count of token t's places (rolled loops:
                // this code runs once per launch, so it is kept short)
                for (int t = lane; t < T; t += 32) tn[t] = 0;
                __syncwarp();
                int big = 0;
                const uint32_t lt = (1u << lane) - 1u;
                for (int s0 = 0; s0 < n_slots; s0 += 32) {
                    const int sl = s0 + lane;
                    const uint32_t m = sl >= n_slots ? 0u : (sl < ns ? 0xFFFFFFFFu : emask[slot_e[sl]]);
                    if (sl >= ns && sl < n_slots) big = max(big, __popc(m));
#pragma unroll 1
                    for (int t = 0; t < T; ++t) {
                        const uint32_t bit = (m >> t) & 1u;
                        const uint32_t bal = __ballot_sync(0xffffffffu, bit);
                        const int base = tn[t];
                        if (bit) pos[sl * T + t] = (unsigned char)(base + __popc(bal & lt));
                        __syncwarp();
                        if (lane == 0) tn[t] = base + __popc(bal);
                        __syncwarp();
                    }
                }
                big = (int)__reduce_max_sync(0xffffffffu, (unsigned)big);
                if (lane == 0) {
                    // Routed units on the clusters without shared-expert units only,
                    // when that takes no more rounds than spreading them over all.
                    const int U = n_slots * FC, S = FC * ns;
                    const bool apart = S > 0 && S < nc && (U - S + nc - S - 1) / (nc - S) <= (U + nc - 1) / nc;
                    int nu;
                    if (!apart) {
                        nu = U > q ? (U - 1 - q) / nc + 1 : 0;
                    } else if (q < S) {
                        nu = 1;  // its shared-expert unit, u = q
                    } else {
                        nu = U > q ? (U - 1 - q) / (nc - S) + 1 : 0;
                        s_stride = nc - S;
                    }
                    s_nunits = max(nu, n_pre);
                    if (b == 0) {
                        a.meta->n_active = n_slots - ns;
                        a.meta->max_count = big;
                        a.meta->n_fixup = 0;  // the fp64 logits are ranked exactly
                    }
                }
            }
            cyc_add(18, csc);  // places + meta
            consumer_sync();
            if (tid == 0) mbar_arrive(&sched);  // the producer may issue the routed units
            cyc_add(7, ctk);
            trace(5);
            // routing weights = softmax over each token's k selected logits, off the
            // schedule's path: the producer is already issuing the routed units' copies
            const unsigned long long cw = cyc();
            for (int t = warp; t < T; t += kCWarps) {  // the warp that ranked token t
                const float ex = lane < k ? expf(sw[t * k + lane]) : 0.0f;
                float z = ex;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (lane < k) {
                    const float wv = ex / z;
                    sw[t * k + lane] = wv;
                    if (b == 0) a.w[(int64_t)t * k + lane] = wv;
                }
            }
            consumer_sync();  // every token's weights are in sw before the units read them
            cyc_add(14, cw);
            return s_nunits;
        };

        // ---- 3. units, pipelined: gate/up of unit i, then the down of unit i - 1.
        // The shared-expert units (i < n_pre) need no routing and overlap the
        // router hand-off; each unit step is inlined once, which keeps the
        // kernel's instruction footprint small.
        int n_units = n_pre;
        bool routed = false;
        for (int i = 0;; ++i) {
            if (i == n_pre && !routed) {
                trace(2);
                n_units = routing();
                routed = true;
            }
            if (i >= n_units) break;
            gate_up(i);
            if (i >= n_pre) trace(6 + 2 * min(i - n_pre, 15));
            if (i > 0) down(i - 1);
        }
        if (n_units > 0) down(n_units - 1);
        trace(38);

        // ---- 4. every CTA's partial sums, then this CTA's slice of y
        unsigned long long ctl = cyc();
        consumer_sync();
        if (tid == 0) grid_wait(a.ctr + 1, grid_arrive(a.ctr + 1, true), a);
        consumer_sync();
        cyc_add(19, ctl);
        ctl = cyc();
        trace(39);
        {
            // output quads (t, n..n+3); a half-warp per quad, lane `sub` summing
            // contributions sub, sub + 16, ... in order, then a fixed-order tree
            const int NG4 = T * (d / 4);
            const int g0 = (int)((int64_t)b * NG4 / G), g1 = (int)((int64_t)(b + 1) * NG4 / G);
            const int sub = lane & 15;
            for (int base = g0 + 2 * warp; base < g1; base += 2 * kCWarps) {  // warp-uniform trip count
                const int gq = base + (lane >> 4);
                const bool valid = gq < g1;
                const int t = valid ? gq / (d / 4) : 0, n = valid ? 4 * (gq - t * (d / 4)) : 0;
                const int ncon = valid ? tn[t] * FC : 0;
                const float* pr = a.part + (int64_t)t * KS * FC * d + n;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int cc = sub; cc < ncon; cc += 16) {
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(pr + (int64_t)cc * d));
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) {
                    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
                    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
                    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
                    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
                }
                if (valid && sub == 0) {
                    if (a.out_fp32) {
                        float4* y4 = reinterpret_cast<float4*>(static_cast<float*>(a.y) + (int64_t)t * d + n);
                        if (a.accumulate) {
                            const float4 yi = *y4;
                            acc.x += yi.x;
                            acc.y += yi.y;
                            acc.z += yi.z;
                            acc.w += yi.w;
                        }
                        *y4 = acc;
                    } else {
                        uint2* y2 = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.y) + (int64_t)t * d + n);
                        if (a.accumulate) {
                            const uint2 yi = *y2;
                            acc.x += __uint_as_float(yi.x << 16);
                            acc.y += __uint_as_float(yi.x & 0xFFFF0000u);
                            acc.z += __uint_as_float(yi.y << 16);
                            acc.w += __uint_as_float(yi.y & 0xFFFF0000u);
                        }
                        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y);
                        const __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc.z, acc.w);
                        uint2 out;
                        out.x = *reinterpret_cast<const uint32_t*>(&lo2);
                        out.y = *reinterpret_cast<const uint32_t*>(&hi2);
                        *y2 = out;
                    }
                }
            }
        }
        cyc_add(20, ctl);
        trace(40);
        cyc_flush();
    }
    // every thread of both CTAs: no remote access is still in flight when a CTA exits
    cluster_arrive();
    cluster_wait();
}

// ---------------------------------------------------------------- launcher
static size_t round128(size_t n) { return (n + 127) & ~size_t(127); }

struct Layout {
    int ng, nd, g_bytes, d_bytes;
    int off_x, off_h, off_gus, off_cand, off_route, off_emask, off_slots, off_pos, off_g, off_d;
    size_t total;
};

// Shared memory: staged x | h buffers | gate/up outputs | top-k candidates |
// routing | expert masks | slot list | slot places | gate/up ring | down ring.
// The rings take what is left of the per-CTA limit, two thirds of it for
// gate/up items.  Items are issued in order (G0..G3, D0, D1 of each unit) and
// the down of unit i runs after the gate/up of unit i + 1, so the down ring
// needs two slots for the gate/up items of unit i + 1 to be issued in time.
static bool make_layout(int BG, int BD, int NT, int T, int d, int f, int E, int k, int smem_max, Layout* L) {
    const int KT = d / 128, RTI = d / 64;
    const int maxS = std::min(T * k, E) + 1;
    (void)f;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += round128(bytes);
        return (int)o;
    };
    L->off_x = take((size_t)T * (d + kXPad) * 2);
    L->off_h = take((size_t)3 * T * kHRow * 2);
    L->off_gus = take(std::max((size_t)kCWarps * 2 * NT * 4 * 32 * 4, (size_t)kCWarps * 16 * 8));
    L->off_cand = take((size_t)kCWarps * kCandBytes);
    L->off_route = take((size_t)T * k * 8);
    L->off_emask = take((size_t)E * 8);
    L->off_slots = take((size_t)maxS * 4);
    L->off_pos = take(64 + (size_t)maxS * T);  // token counts [16], then the places
    L->g_bytes = 2 * KT * (256 * BG + 128);
    L->d_bytes = RTI * (256 * BD + 128);
    const long avail = (long)smem_max - (long)off;
    if (avail < (long)(L->g_bytes + 2 * L->d_bytes)) return false;
    int ng = std::max(1, (int)((avail * 2 / 3) / L->g_bytes));
    ng = std::min(ng, kMaxSlots);
    int nd = (int)((avail - (long)ng * L->g_bytes) / L->d_bytes);
    if (nd < 2) {
        ng = (int)((avail - 2L * L->d_bytes) / L->g_bytes);
        nd = 2;
    }
    nd = std::min(nd, kMaxSlots);
    if (ng < 1) return false;
    L->ng = ng;
    L->nd = nd;
    L->off_g = take((size_t)ng * L->g_bytes);
    L->off_d = take((size_t)nd * L->d_bytes);
    L->total = off;
    return true;
}

struct Occ {
    int dev;
    const void* fn;
    size_t smem;
    int clusters;
};
// The dynamic shared-memory limit is one setting per kernel and device: it is
// raised to the largest size any launch needed and never lowered.
struct SmemAttr {
    int dev;
    const void* fn;
    size_t smem;
};

template <int BG, int BD, int NT>
static cudaError_t launch_t(const DecodeLaunch& L, cudaStream_t st) {
    auto kern = decode_pair_kernel<BG, BD, NT>;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int smem_max = 0;
    e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    // static shared memory of the kernel (barriers and a few words) comes off the limit
    Layout lay;
    if (!make_layout(BG, BD, NT, L.T, L.d, L.f, L.E, L.k, smem_max - 1024, &lay)) return cudaErrorInvalidConfiguration;

    static std::mutex mu;
    static std::vector<Occ> cache;
    static std::vector<SmemAttr> attrs;
    int clusters = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        SmemAttr* at_set = nullptr;
        for (SmemAttr& s2 : attrs)
            if (s2.dev == dev && s2.fn == (const void*)kern) at_set = &s2;
        if (!at_set || at_set->smem < lay.total) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total);
            if (e != cudaSuccess) return e;
            if (at_set)
                at_set->smem = lay.total;
            else
                attrs.push_back({dev, (const void*)kern, lay.total});
        }
        for (const Occ& o : cache)
            if (o.dev == dev && o.fn == (const void*)kern && o.smem == lay.total) clusters = o.clusters;
        if (clusters == 0) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = kCS;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(kCS);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = lay.total;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
            if (e != cudaSuccess) return e;
            if (clusters < 1) return cudaErrorInvalidConfiguration;
            cache.push_back({dev, (const void*)kern, lay.total, clusters});
        }
    }

    Args a;
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
    a.code_stride = (int64_t)L.f * L.d * (2 * BG + BD) / 8;
    a.scale_stride = (int64_t)3 * L.f * L.d / 32;
    a.wr = static_cast<const uint16_t*>(L.wr);
    a.bias = L.bias;
    a.logits64 = L.logits64;
    a.ids = L.ids;
    a.w = L.w;
    a.meta = L.meta;
    a.status = L.status;
    a.part = L.part;
    a.ctr = L.ctr;
    a.skip_rank = L.skip_rank;
    a.e_begin = std::max(0, L.e_begin);
    a.e_end = std::min(L.E, L.e_end);
    a.nc = clusters;
    a.spin_limit = L.spin_limit;
    a.withhold = L.withhold;
    a.norm_input = L.norm_input;
    a.ng = lay.ng;
    a.nd = lay.nd;
    a.g_bytes = lay.g_bytes;
    a.d_bytes = lay.d_bytes;
    a.off_x = lay.off_x;
    a.off_h = lay.off_h;
    a.off_gus = lay.off_gus;
    a.off_cand = lay.off_cand;
    a.off_route = lay.off_route;
    a.off_emask = lay.off_emask;
    a.off_slots = lay.off_slots;
    a.off_pos = lay.off_pos;
    a.off_g = lay.off_g;
    a.off_d = lay.off_d;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kCS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeCooperative;
    at[1].val.cooperative = 1;
    cfg.gridDim = dim3(kCS * clusters);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lay.total;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    // The grid barriers need every CTA resident at once, which the cooperative
    // launch guarantees.  Where fewer clusters fit than the occupancy query
    // reported (another client holding SMs, a profiler), the launch is refused:
    // retry with fewer clusters (the work split follows the cluster count) and
    // remember the count that was accepted.
    for (int attempt = 0; attempt < 16; ++attempt) {
        a.nc = clusters;
        cfg.gridDim = dim3(kCS * clusters);
        e = cudaLaunchKernelEx(&cfg, kern, a, *L.down_codes_map, *L.down_scales_map);
        if (e != cudaErrorCooperativeLaunchTooLarge || clusters <= 1) break;
        (void)cudaGetLastError();
        clusters = std::max(1, clusters - std::max(1, clusters / 16));
        std::lock_guard<std::mutex> lk(mu);
        for (Occ& o : cache)
            if (o.dev == dev && o.fn == (const void*)kern && o.smem == lay.total) o.clusters = clusters;
    }
    return e;
}

template <int BG, int BD>
static cudaError_t launch_bits(const DecodeLaunch& L, cudaStream_t s) {
    return L.T <= 8 ? launch_t<BG, BD, 1>(L, s) : launch_t<BG, BD, 2>(L, s);
}

template <int BG>
static cudaError_t launch_gu(const DecodeLaunch& L, cudaStream_t s) {
    switch (L.bits_down) {
        case 2: return launch_bits<BG, 2>(L, s);
        case 3: return launch_bits<BG, 3>(L, s);
        case 4: return launch_bits<BG, 4>(L, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pair

#ifdef MOE_PAIR_TRACE
extern "C" int moe_debug_pair_trace(unsigned long long* host, int n) {
    return cudaMemcpyFromSymbol(host, pair::g_trace, sizeof(unsigned long long) * (size_t)n) == cudaSuccess ? 0 : 2;
}
extern "C" int moe_debug_pair_cycles(unsigned long long* host, int n) {  // [1024][32]
    return cudaMemcpyFromSymbol(host, pair::g_cyc, sizeof(unsigned long long) * (size_t)n) == cudaSuccess ? 0 : 2;
}
#endif

size_t pair_part_floats(int max_tokens, int k, int n_shared, int d, int f) {
    return (size_t)std::min(max_tokens, kPairMaxTokens) * (size_t)(k + n_shared) * (size_t)(f / 128) * (size_t)d;
}

bool pair_decode_supported(const DecodeLaunch& L) {
    if (!L.down_codes_map || !L.down_scales_map || !L.part) return false;
    int smem_max = 232448;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    pair::Layout lay;
    const int bd = L.bits_down ? L.bits_down : L.bits;
    return L.T >= 1 && L.T <= kPairMaxTokens && L.E <= 1024 && L.k <= 32 && L.d % 128 == 0 && L.f % 128 == 0 &&
           L.d <= 128 * pair::kCWarps * pair::kMaxKS &&
           pair::make_layout(L.bits, bd, L.T <= 8 ? 1 : 2, L.T, L.d, L.f, L.E, L.k, smem_max - 1024, &lay);
}

cudaError_t launch_decode_pair(const DecodeLaunch& L, cudaStream_t s) {
    if (!pair_decode_supported(L)) return cudaErrorInvalidValue;
    DecodeLaunch M = L;
    if (!M.bits_down) M.bits_down = M.bits;
    switch (M.bits) {
        case 2: return pair::launch_gu<2>(M, s);
        case 3: return pair::launch_gu<3>(M, s);
        case 4: return pair::launch_gu<4>(M, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe

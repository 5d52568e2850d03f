// tiles.cuh -- the tile list of the tensor-core expert GEMMs, built by one
// CTA of kTileListThreads threads (a kernel of its own, or the tail of the
// single-CTA bucketing kernel, which already holds the groups).
//
// Slots: the shared expert (if any), then the active routed experts in
// ascending order.  A slot with c tokens holds ceil(c / kExpertTileN) token
// tiles; token tile q of the layer times the JT row-tiles of a weight gives
// tiles q * JT .. q * JT + JT - 1, so CTAs that take consecutive tiles read
// the same activation rows.  One descriptor per tile:
//   x = expert (E for the shared one), y = row0 (h / partial-output row of
//   the tile's first token = its first pair position), z = n | jt << 16,
//   w = first token for the shared expert, -1 for a routed one (whose rows'
//   tokens are pairs[row0 + r] / k).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kExpertTileN = 256;  // tokens per expert tile (at most; the MMA's N)
constexpr int kTileListThreads = 1024;
constexpr int kTileMaxSlots = 1024 + 1;

// Shared memory of build_tile_list.
struct TileListSmem {
    int pre[kTileMaxSlots + 1];
    int wsum[kTileListThreads / 32];
    int carry;
};

// Every thread of a kTileListThreads-thread CTA calls this (it synchronises
// the CTA).  offsets [E + 1] and active [n_active] are the bucketing's groups,
// readable by every thread of the CTA.
MOE_DEV void build_tile_list(int T, int k, int E, int n_shared, int n_active, const int32_t* offsets,
                             const int32_t* active, int jt_gateup, int jt_down, int4* __restrict__ desc_gu,
                             int4* __restrict__ desc_dn, int32_t* __restrict__ counts, TileListSmem& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_slots = n_shared + n_active;
    if (tid == 0) sm.carry = 0;
    __syncthreads();
    for (int base = 0; base < n_slots; base += kTileListThreads) {
        const int s = base + tid;
        int tt = 0;
        if (s < n_slots) {
            int count;
            if (s < n_shared) count = T;
            else {
                const int e = active[s - n_shared];
                count = offsets[e + 1] - offsets[e];
            }
            tt = (count + kExpertTileN - 1) / kExpertTileN;
        }
        int inc = tt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) sm.wsum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int v = sm.wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            sm.wsum[lane] = v;  // inclusive over warps
        }
        __syncthreads();
        const int carry = sm.carry;
        if (s < n_slots) sm.pre[s] = carry + (warp ? sm.wsum[warp - 1] : 0) + inc - tt;
        __syncthreads();
        if (tid == 0) sm.carry = carry + sm.wsum[kTileListThreads / 32 - 1];
        __syncthreads();
    }
    const int total_tt = sm.carry;
    if (tid == 0) {
        sm.pre[n_slots] = total_tt;
        counts[0] = total_tt * jt_gateup;
        counts[1] = total_tt * jt_down;
    }
    __syncthreads();
    for (int q = tid; q < total_tt; q += kTileListThreads) {
        int lo = 0, hi = n_slots - 1;  // last slot with pre[s] <= q
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sm.pre[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int tt = q - sm.pre[lo];
        int expert, row0, count, tok0;
        if (lo < n_shared) {
            expert = E;
            count = T;
            row0 = T * k + tt * kExpertTileN;
            tok0 = tt * kExpertTileN;
        } else {
            expert = active[lo - n_shared];
            const int p0 = offsets[expert];
            count = offsets[expert + 1] - p0;
            row0 = p0 + tt * kExpertTileN;
            tok0 = -1;
        }
        const int n = min(kExpertTileN, count - tt * kExpertTileN);
        for (int jt = 0; jt < jt_gateup; ++jt) desc_gu[q * jt_gateup + jt] = make_int4(expert, row0, n | (jt << 16), tok0);
        for (int jt = 0; jt < jt_down; ++jt) desc_dn[q * jt_down + jt] = make_int4(expert, row0, n | (jt << 16), tok0);
    }
}

}  // namespace moe

// gemm_sm100.cu -- tcgen05 (5th-generation tensor core) GEMMs for large token counts.
//
// Prefill chunks (thousands of tokens; the pages read prompts in chunks of up
// to 8192 tokens -- molayo1419.me summary, section "Distributed model
// execution across the PC") turn the layer into three dense contractions:
//   router    logits[t, e] = x_t . W_r[e] + bias_e           (bf16 x bf16)
//   gate/up   h[p, j] = silu(Wg_e[j] . x_t) * (Wu_e[j] . x_t)   per expert group
//   down      o[p, n] = w_p * (Wd_e[n] . h_p)                  per expert group
// (p: an expert slot's (token, rank) pair, or the token for the shared expert.)
//
// Each CTA owns one tile at a time: 128 weight rows (the MMA's M, "swap AB")
// by up to 256 tokens (the MMA's N, rounded up to a multiple of 16 for small
// expert groups), accumulated in tensor memory (TMEM) over K in steps of 64.
// The tokens' activation rows (h, or x gathered into group order) arrive by
// 2-D TMA straight into the 128-byte-swizzled K-major layout the MMA reads;
// the packed codes and scales arrive by 1-D bulk copies; the CTA's threads
// turn codes into fp16(q * s) in the same swizzled layout; one thread issues
// tcgen05.mma (kind::f16, fp32 accumulate); the epilogue reads TMEM with
// tcgen05.ld.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace moe {
namespace tc {

constexpr uint32_t kSpin = 1u << 24;  // polls of a non-blocking test (about 0.5 s)

MOE_DEV uint64_t sdesc(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row atoms of 1024 B, 16-B LBO, SM100 version 1
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
// byte offset of element (r, k) in a [rows x 64] 16-bit tile, K-major SW128
MOE_DEV uint32_t sw128(int r, int k) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((k >> 3) ^ (r & 7)) & 7) << 4) + (k & 7) * 2);
}
// 16-byte chunk c (8 elements) of row r
MOE_DEV uint32_t sw128_chunk(int r, int c) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + (((c ^ r) & 7) << 4)); }

MOE_DEV uint32_t idesc_f16(int M, int N, bool bf16) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

MOE_DEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
MOE_DEV void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

MOE_DEV void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
MOE_DEV void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
// 16 consecutive 32-bit columns of the warp's 32 TMEM lanes (no wait)
MOE_DEV void ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
MOE_DEV void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
MOE_DEV void ld16(uint32_t taddr, uint32_t (&r)[16]) {
    ld16_nowait(taddr, r);
    ld_wait();
}

MOE_DEV void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
MOE_DEV void cp8(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
MOE_DEV void cp4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
MOE_DEV void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEV void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

MOE_DEV bool test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// bounded wait on an mbarrier phase; false if it gave up.  A non-blocking
// test in a loop: the waiting thread sees the phase flip at once (a blocking
// try_wait can leave it suspended for a while after the flip).
MOE_DEV bool bar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
    for (uint32_t it = 0; it < kSpin; ++it)
        if (test_wait(bar, parity)) return true;
    flag_status(status, kStatusTimeout);
    return false;
}

}  // namespace tc

constexpr int kTileM = 128;  // weight rows per tile (the MMA's M)
constexpr int kStepK = 64;   // K per pipeline step (one SW128 atom of 16-bit values)
constexpr int kRouterTileN = 128;  // tokens per router tile

// ---------------------------------------------------------------- tile list
// (tiles.cuh: the slots, token tiles and descriptors)
static inline int max_token_tiles(int T, int k, int E, int n_shared) {
    return (T * k + kExpertTileN - 1) / kExpertTileN + E + n_shared * ((T + kExpertTileN - 1) / kExpertTileN) + 1;
}

__global__ void __launch_bounds__(kTileListThreads)
    build_tiles_kernel(const ExpertArgs a, int jt_gateup, int jt_down, int4* __restrict__ desc_gu,
                       int4* __restrict__ desc_dn, int32_t* __restrict__ counts) {
    __shared__ TileListSmem sm;
    build_tile_list(a.T, a.k, a.E, a.n_shared, a.meta->n_active, a.offsets, a.active, jt_gateup, jt_down, desc_gu,
                    desc_dn, counts, sm);
}

struct GemmArgs {
    ExpertArgs e;
    const float* wsorted;    // routing weight of each pair, in group order [T*k]
    __half* o;               // fp16 weighted expert outputs [rows x d]
    const int4* desc;        // tile descriptors
    const int32_t* n_tiles;  // number of descriptors
};

// ---------------------------------------------------------------- grouped expert GEMM
// GATEUP: A0 = W_g rows, A1 = W_u rows (row-tile jt of f), B = x rows of the
// slot's tokens (gathered, fp16); epilogue h = silu(g) * u -> fp16.
// Otherwise: A0 = W_d rows (row-tile jt of d), B = h rows; epilogue
// o = w_p * acc -> fp16.
//
// Warp roles (persistent; every role walks the same tile sequence
// blockIdx.x, blockIdx.x + gridDim.x, ...):
//   warp 13     loader (one thread): for each K = 64 step, once the MMAs that
//               last read the stage are done, TMA loads of the B rows and bulk
//               copies of the 8 row-tiles' code super-tiles and scales (into the
//               stage's A area), all completing on load[stage]
//   warps 0-7   dequant: copy their codes and scales to registers, then write
//               fp16(q * s) over the same area in the swizzled A layout;
//               signal full[stage]
//   warp 12     MMA issuer (one thread): wait full[stage], issue the step's
//               MMAs, commit to empty[stage]; at the end of a tile commit to
//               acc_full[buffer]
//   warps 8-11  epilogue: wait for a finished accumulator, tcgen05.ld, SwiGLU
//               or weighting, fp16 stores; signal acc_empty[buffer]
//
// A pipeline step is kSK of K: 64 for gate/up (one SW128 atom; a step's codes
// are half a 128-wide super-tile, so each super-tile is staged twice), 128
// for down (two atoms side by side in A and in B; the whole super-tile once,
// and half the steps, so half the per-step barriers, for the same K).
template <int BITS, bool GATEUP>
struct GemmCfg {
    static constexpr int kN = kExpertTileN;
    static constexpr int kSK = GATEUP ? 64 : 128;  // K per step
    static constexpr int kAtoms = kSK / 64;         // SW128 atoms per row of a step's tile
    static constexpr int kStages = GATEUP ? 3 : 2;
    static constexpr int kMats = GATEUP ? 2 : 1;
    static constexpr int kAtomA = kTileM * 128, kAtomB = kN * 128;  // one atom of A / of B
    static constexpr int kA = kAtoms * kAtomA, kB = kAtoms * kAtomB;
    static constexpr int kCodeBytes = 8 * 256 * BITS;  // 8 row-tiles x one super-tile, in the A area
    static constexpr int kScaleBytes = 8 * 128;
    static_assert(kCodeBytes + kScaleBytes <= kA, "codes fit in the A area");
    static constexpr int kStageBytes = kMats * kA + kB;
    static constexpr int kSmem = kStages * kStageBytes + 1024;  // + alignment slack
    static constexpr int kAccCols = kMats * kN;                 // one accumulator set
    static constexpr int kAccBufs = 512 / kAccCols;             // 1 (gate/up) or 2 (down)
    static constexpr uint32_t kStageTxFixed = kMats * (kCodeBytes + kScaleBytes);
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static_assert(kAccBufs >= 1, "tensor memory");
};
constexpr int kBRowsSmall = 32;   // rows of the small B TMA box (groups of <= 64 tokens)
constexpr int kBRowsBig = 256;    // rows of the large B TMA box
constexpr int kEpilogueWarp0 = 8;
constexpr int kMmaWarp = 12;
constexpr int kLoaderWarp = 13;
constexpr int kExpertThreads = 14 * 32;

MOE_DEV void producer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// warp-uniform bounded wait (lane 0 polls)
MOE_DEV bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
    bool okw = true;
    if ((threadIdx.x & 31) == 0) okw = tc::bar_wait(bar, parity, status);
    return __shfl_sync(0xffffffffu, okw ? 1 : 0, 0) != 0;
}

// 2-D TMA tile load into this CTA's shared memory, completing on `bar`
MOE_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// 3-D TMA tile load into this CTA's shared memory, completing on `bar`
MOE_DEV void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

MOE_DEV int4 load_desc(const GemmArgs& g, int tile) { return __ldg(&g.desc[tile]); }

template <int BITS, bool GATEUP>
__global__ void __launch_bounds__(kExpertThreads, 1)
    expert_gemm_kernel(const GemmArgs g, const __grid_constant__ CUtensorMap bmap_s,
                       const __grid_constant__ CUtensorMap bmap_b, const __grid_constant__ CUtensorMap cmap,
                       const __grid_constant__ CUtensorMap smap) {
    using C = GemmCfg<BITS, GATEUP>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t load_bar[C::kStages];
    __shared__ __align__(8) uint64_t full_bar[C::kStages];
    __shared__ __align__(8) uint64_t empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t accf_bar[C::kAccBufs];
    __shared__ __align__(8) uint64_t acce_bar[C::kAccBufs];
    __shared__ uint32_t tmem_slot;
    __shared__ float w_s[GATEUP ? 1 : kExpertTileN];  // routing weights of the epilogue's tile
    __shared__ __align__(16) __half ep_stage[4][16][32];  // epilogue transpose, one [token][row] block per warp
    const ExpertArgs& a = g.e;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int K = GATEUP ? a.d : a.f;  // contraction length
    const int KS = K / C::kSK;         // pipeline steps per tile

    if (tid == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(&load_bar[i], 1);
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        for (int i = 0; i < C::kAccBufs; ++i) {
            mbar_init(&accf_bar[i], 1);
            mbar_init(&acce_bar[i], 128);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) tc::tmem_alloc(&tmem_slot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = tmem_slot;

    const int total_tiles = *g.n_tiles;
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
    const int my_tiles = total_tiles > bid ? (total_tiles - 1 - bid) / grid + 1 : 0;
    const int total = my_tiles * KS;  // K steps of this CTA

    if (warp < kEpilogueWarp0) {
        // ======================= dequant
        bool ok = true;
        const int rt = tid >> 5, ln = tid & 31, gg = ln >> 2, c = ln & 3;
        constexpr int NKB = C::kSK / 32;  // 32-wide K blocks per step: 2 (half a super-tile) or 4
        for (int gs = 0; gs < total; ++gs) {
            const int st = gs % C::kStages;
            const int kbs = C::kSK == 64 ? 2 * ((gs % KS) & 1) : 0;  // first K block of the super-tile
            if (tid == 0 && ok) ok = tc::bar_wait(&load_bar[st], (gs / C::kStages) & 1, a.status);
            producer_sync();  // codes, scales and B rows of step gs have landed
            uint8_t* sb = smem + st * C::kStageBytes;
            uint32_t lo[C::kMats][NKB], hi[C::kMats][NKB], sc[C::kMats][NKB];
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
                const uint8_t* cs = sb + m * C::kA + rt * (256 * BITS);
                const uint8_t* ss = sb + m * C::kA + C::kCodeBytes + rt * 128 + 16 * gg;
#pragma unroll
                for (int j = 0; j < NKB; ++j) {
                    const int kb = kbs + j;
                    lo[m][j] = *reinterpret_cast<const uint32_t*>(cs + 16 * ln + 4 * kb);
                    if (BITS == 3) {
                        const uint32_t hv = *reinterpret_cast<const uint32_t*>(cs + 512 + 8 * ln + 4 * (kb >> 1));
                        hi[m][j] = (kb & 1) ? hv >> 16 : hv & 0xFFFFu;
                    } else if (BITS == 4) {
                        hi[m][j] = *reinterpret_cast<const uint32_t*>(cs + 512 + 16 * ln + 4 * kb);
                    } else {
                        hi[m][j] = 0;
                    }
                    sc[m][j] = *reinterpret_cast<const uint32_t*>(ss + 4 * kb);
                }
            }
            producer_sync();  // every read of the staged codes is done before A overwrites them
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
#pragma unroll
                for (int kbl = 0; kbl < NKB; ++kbl) {
                    uint8_t* A = sb + m * C::kA + (kbl >> 1) * C::kAtomA;  // the block's atom
                    uint32_t q[8];
                    decode_block<true, BITS>(lo[m][kbl], hi[m][kbl], q);
                    const __half2 s_lo = __half2half2(__ushort_as_half((unsigned short)(sc[m][kbl] & 0xFFFFu)));
                    const __half2 s_hi = __half2half2(__ushort_as_half((unsigned short)(sc[m][kbl] >> 16)));
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        // pair p = 4 ks + 2 (m / 8) + r / 8 of the A-fragment layout
                        const int ks = p >> 2, hi8 = (p >> 1) & 1, half = p & 1;
                        const int r = rt * 16 + gg + 8 * half;
                        const int kk = 32 * (kbl & 1) + 16 * ks + 8 * hi8 + 2 * c;  // within the atom
                        const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&q[p]), half ? s_hi : s_lo);
                        *reinterpret_cast<__half2*>(A + tc::sw128(r, kk)) = v;
                    }
                }
            }
            fence_proxy_async_smem();  // A tiles visible to the tensor core
            producer_sync();
            if (tid == 0) mbar_arrive(&full_bar[st]);
        }
    } else if (warp < kMmaWarp) {
        // ======================= epilogue
        // Thread = weight row (TMEM lane); per 16-token chunk the next chunk's
        // TMEM loads are in flight while this one is converted, staged as
        // [token][32 rows] fp16 in shared memory and written out as 16-byte
        // vectors (4 lanes cover the warp's 64 contiguous bytes of a token row).
        const int q = warp & 3;  // TMEM lanes 32 q .. 32 q + 31 = weight rows
        const int et = tid - 32 * kEpilogueWarp0;  // 0 .. 127
        __half* stg = &ep_stage[q][0][0];
        const int vt = lane >> 2, seg = lane & 3;  // vector store: token vt (+8), 16-byte segment seg
        bool ok = true;
        int4 nd = my_tiles > 0 ? load_desc(g, bid) : make_int4(0, 0, 0, 0);
        for (int it = 0; it < my_tiles; ++it) {
            const int4 ds = nd;
            if (it + 1 < my_tiles) nd = load_desc(g, bid + (it + 1) * grid);
            const int n = ds.z & 0xFFFF, jt = ds.z >> 16, nmma = (n + 15) & ~15;
            if (!GATEUP) {
                for (int i = et; i < n; i += 128) w_s[i] = ds.w >= 0 ? 1.0f : __ldg(&g.wsorted[ds.y + i]);
                asm volatile("bar.sync 2, 128;" ::: "memory");
            }
            const int b = it % C::kAccBufs, use = it / C::kAccBufs;
            if (ok) ok = warp_wait(&accf_bar[b], use & 1, a.status);
            tc::fence_after();
            const uint32_t tb = tmem + ((uint32_t)(32 * q) << 16) + b * C::kAccCols;
            const int ld_cols = GATEUP ? a.f : a.d;  // row length of h / o
            __half* dst = (GATEUP ? static_cast<__half*>(a.h) : g.o) + (int64_t)ds.y * ld_cols + jt * kTileM + 32 * q +
                          seg * 8;
            uint32_t r0[16], r1[16];
            if (ok && nmma > 0) {
                tc::ld16_nowait(tb, r0);
                if (GATEUP) tc::ld16_nowait(tb + C::kN, r1);
                tc::ld_wait();
            }
            bool finite = true;
            for (int c0 = 0; c0 < nmma && ok; c0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float acc = __uint_as_float(r0[i]);
                    if (GATEUP) {
                        const float hv = __fdividef(acc, 1.0f + __expf(-acc)) * __uint_as_float(r1[i]);
                        finite = finite && fabsf(hv) <= 65504.0f;
                        v[i] = hv;
                    } else {
                        v[i] = w_s[min(c0 + i, kExpertTileN - 1)] * acc;
                    }
                }
                const bool more = c0 + 16 < nmma;
                if (more) {  // next chunk's accumulators load while this one is stored
                    tc::ld16_nowait(tb + c0 + 16, r0);
                    if (GATEUP) tc::ld16_nowait(tb + C::kN + c0 + 16, r1);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) stg[i * 32 + lane] = __float2half_rn(v[i]);
                __syncwarp();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int tl = vt + 8 * hh, tok = c0 + tl;
                    if (tok < n)
                        *reinterpret_cast<uint4*>(dst + (int64_t)tok * ld_cols) =
                            *reinterpret_cast<const uint4*>(stg + tl * 32 + seg * 8);
                }
                __syncwarp();
                if (more) tc::ld_wait();
            }
            if (GATEUP && !finite) flag_status(a.status, kStatusRange);
            tc::fence_before();
            mbar_arrive(&acce_bar[b]);
            if (!GATEUP) asm volatile("bar.sync 2, 128;" ::: "memory");  // w_s reads done
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            // ======================= MMA issuer
            bool ok = true;
            int gs = 0;
            int4 nd = my_tiles > 0 ? load_desc(g, bid) : make_int4(0, 0, 0, 0);
            for (int it = 0; it < my_tiles; ++it) {
                const int4 ds = nd;
                if (it + 1 < my_tiles) nd = load_desc(g, bid + (it + 1) * grid);
                const int nmma = ((ds.z & 0xFFFF) + 15) & ~15;
                const uint32_t idesc = tc::idesc_f16(kTileM, nmma, false);
                const int b = it % C::kAccBufs, use = it / C::kAccBufs;
                if (use > 0 && ok) ok = tc::bar_wait(&acce_bar[b], (use - 1) & 1, a.status);
                tc::fence_after();
                const uint32_t acc_addr = tmem + b * C::kAccCols;
                for (int s = 0; s < KS; ++s, ++gs) {
                    const int st = gs % C::kStages;
                    if (ok) ok = tc::bar_wait(&full_bar[st], (gs / C::kStages) & 1, a.status);
                    tc::fence_after();
                    uint8_t* sb = smem + st * C::kStageBytes;
                    const uint32_t a_addr = smem_addr(sb), b_addr = smem_addr(sb + C::kMats * C::kA);
#pragma unroll
                    for (int kk = 0; kk < C::kSK / 16; ++kk) {
                        const uint32_t ao = (kk >> 2) * C::kAtomA + (kk & 3) * 32;  // atom, then 16-wide K slice
                        const uint64_t bd = tc::sdesc(b_addr + (kk >> 2) * C::kAtomB + (kk & 3) * 32);
                        const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                        tc::mma(acc_addr, tc::sdesc(a_addr + ao), bd, idesc, acc);
                        if (GATEUP) tc::mma(acc_addr + C::kN, tc::sdesc(a_addr + C::kA + ao), bd, idesc, acc);
                    }
                    tc::commit(&empty_bar[st]);
                }
                tc::commit(&accf_bar[b]);
            }
        }
    } else if (warp == kLoaderWarp && lane == 0) {
        // ======================= loader
        // Per step: the B rows (one 256-row box, or 32-row boxes for small
        // groups) and, per matrix, one box of 8 row-tiles x one super-tile of
        // codes and one of scales (the codes and scales tensor maps view a
        // matrix as rows of 16-row tiles, columns of 128-wide super-tiles).
        bool ok = true;
        const int mrows = (GATEUP ? a.f : a.d) / 16;  // map rows per matrix
        int4 ds = make_int4(0, 0, 0, 0);
        int4 nd = my_tiles > 0 ? load_desc(g, bid) : make_int4(0, 0, 0, 0);
        int cur = -1, nmma = 0;
        for (int j = 0; j < total; ++j) {
            const int ti_local = j / KS, s = j - ti_local * KS, st = j % C::kStages;
            if (ti_local != cur) {
                cur = ti_local;
                ds = nd;
                if (ti_local + 1 < my_tiles) nd = load_desc(g, bid + (ti_local + 1) * grid);
                nmma = ((ds.z & 0xFFFF) + 15) & ~15;
            }
            if (j >= C::kStages && ok)  // the MMAs of step j - S have read the stage
                ok = tc::bar_wait(&empty_bar[st], ((j / C::kStages) - 1) & 1, a.status);
            uint8_t* sb = smem + st * C::kStageBytes;
            uint8_t* Bs = sb + C::kMats * C::kA;
            const bool big = nmma > 2 * kBRowsSmall;
            const int nsmall = (nmma + kBRowsSmall - 1) / kBRowsSmall;
            mbar_arrive_expect_tx(&load_bar[st], C::kStageTxFixed + (uint32_t)C::kAtoms *
                                                                        (big ? kBRowsBig : nsmall * kBRowsSmall) * 128);
#pragma unroll
            for (int at = 0; at < C::kAtoms; ++at) {  // one 64-wide K atom of the B rows at a time
                uint8_t* Ba = Bs + at * C::kAtomB;
                const int kx = s * C::kSK + at * 64;
                if (big) {
                    tma_load_2d(Ba, &bmap_b, kx, ds.y, &load_bar[st]);
                } else {
                    for (int i = 0; i < nsmall; ++i)
                        tma_load_2d(Ba + i * kBRowsSmall * 128, &bmap_s, kx, ds.y + i * kBRowsSmall, &load_bar[st]);
                }
            }
            const int expert = ds.x, jt = ds.z >> 16, kt = (s * C::kSK) / 128;  // the step's super-tile
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
                uint8_t* A = sb + m * C::kA;
                // codes: (word, row tile of this kernel's matrices, expert); scales: every
                // expert's three matrices stacked as rows of 16-row tiles
                tma_load_3d(A, &cmap, kt * 64 * BITS, m * mrows + jt * 8, expert, &load_bar[st]);
                tma_load_2d(A + C::kCodeBytes, &smap, kt * 64, (expert * 3 + (GATEUP ? m : 2)) * mrows + jt * 8,
                            &load_bar[st]);
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == kMmaWarp) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- router GEMM
// logits[t][e] = W_r[e] . x_t + bias_e for 128-expert x 128-token tiles, bf16
// operands loaded by TMA straight into the SW128 tiles.  The contraction is
// split into `chunks` consecutive K ranges, each accumulated in its own
// tensor-memory columns; the epilogue adds the chunk sums in chunk order.  A
// chunk's rounding error grows with its own length, so the logits' error bound
// is that many times tighter than one running sum over all of d
// (router_gemm_depth).  split != 0 (small batches, whose few tiles would leave
// most SMs idle): every (tile, chunk) is a work item of its own, and its raw
// chunk sums go to logits[chunk][t][e]; the reader adds the chunks in chunk
// order, then the bias -- the same operations, so the same logits, as the
// unsplit epilogue.
//
// Warp roles (every role walks the same items blockIdx.x, + gridDim.x, ...):
//   warp 0     loader (one thread): per K step, once the MMAs that last read
//              the stage are done, one TMA box of router rows and one of x
//              rows (rows past E or T read as zeros)
//   warp 1     MMA issuer (one thread), after the epilogue has drained the
//              previous item's accumulators
//   warps 2-5  epilogue: tcgen05.ld of the chunk sums, in chunk order, then
//              the bias; fp32 stores
constexpr int kRouterStages = 6;
constexpr int kRouterStage = kTileM * 128 + kRouterTileN * 128;
constexpr int kRouterThreads = 6 * 32;

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, int T,
                       int d, const float* __restrict__ bias, int E, float* __restrict__ logits, int chunks, int split,
                       uint32_t* status) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kRouterStages], empty_bar[kRouterStages], accf_bar, acce_bar,
        drain_bar;
    __shared__ uint32_t tmem_slot;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int KS = d / kStepK;
    const int MT = (E + kTileM - 1) / kTileM, NT = (T + kRouterTileN - 1) / kRouterTileN;
    if (tid == 0) {
        for (int i = 0; i < kRouterStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&acce_bar, 128);
        mbar_init(&drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tc::tmem_alloc(&tmem_slot, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = tmem_slot;
    const int csteps = KS / chunks;        // K steps per chunk
    const uint32_t ccols = 512u / chunks;  // tensor-memory columns per chunk (>= the tile's width)
    const int items = MT * NT * (split ? chunks : 1);
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;
    // item -> tile (mt, nt) and its K steps [s0, s0 + ns); ich: its chunk when split
    auto item_of = [&](int item, int& mt, int& nt, int& ich, int& s0, int& ns) {
        const int tile = item % (MT * NT);
        ich = item / (MT * NT);
        mt = tile % MT;
        nt = tile / MT;
        s0 = split ? ich * csteps : 0;
        ns = split ? csteps : KS;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ======================= loader
            bool ok = true;
            int j = 0;  // K steps issued
            for (int item = bid; item < items && ok; item += grid) {
                int mt, nt, ich, s0, ns;
                item_of(item, mt, nt, ich, s0, ns);
                for (int s = 0; s < ns; ++s, ++j) {
                    const int st = j % kRouterStages;
                    if (j >= kRouterStages)  // the MMAs of step j - S have read the stage
                        ok = tc::bar_wait(&empty_bar[st], ((j / kRouterStages) - 1) & 1, status);
                    if (!ok) break;
                    uint8_t* As = smem + st * kRouterStage;
                    mbar_arrive_expect_tx(&full_bar[st], (uint32_t)kRouterStage);
                    tma_load_2d(As, &wmap, (s0 + s) * kStepK, mt * kTileM, &full_bar[st]);
                    tma_load_2d(As + kTileM * 128, &xmap, (s0 + s) * kStepK, nt * kRouterTileN, &full_bar[st]);
                }
            }
            // no copy may still be landing in shared memory when the CTA leaves
            for (int jj = j > kRouterStages ? j - kRouterStages : 0; jj < j; ++jj)
                tc::bar_wait(&full_bar[jj % kRouterStages], (jj / kRouterStages) & 1, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ======================= MMA issuer
            bool ok = true;
            int j = 0, it = 0;
            for (int item = bid; item < items && ok; item += grid, ++it) {
                int mt, nt, ich, s0, ns;
                item_of(item, mt, nt, ich, s0, ns);
                const int n = min(kRouterTileN, T - nt * kRouterTileN), nmma = (n + 15) & ~15;
                const uint32_t idesc = tc::idesc_f16(kTileM, nmma, true);
                if (it > 0) ok = tc::bar_wait(&acce_bar, (it - 1) & 1, status);  // accumulators drained
                if (!ok) break;
                tc::fence_after();
                for (int s = 0; s < ns && ok; ++s, ++j) {
                    const int st = j % kRouterStages;
                    ok = tc::bar_wait(&full_bar[st], (j / kRouterStages) & 1, status);
                    if (!ok) break;
                    tc::fence_after();
                    const uint32_t a_addr = smem_addr(smem + st * kRouterStage), b_addr = a_addr + kTileM * 128;
                    const int ch = split ? 0 : s / csteps;  // this step's accumulator
#pragma unroll
                    for (int kk = 0; kk < kStepK / 16; ++kk)
                        tc::mma(tmem + ch * ccols, tc::sdesc(a_addr + kk * 32), tc::sdesc(b_addr + kk * 32), idesc,
                                (s > ch * csteps || kk > 0) ? 1u : 0u);
                    tc::commit(&empty_bar[st]);
                }
                if (!ok) break;
                tc::commit(&accf_bar);
            }
            // every MMA issued has finished before tensor memory is released
            tc::commit(&drain_bar);
            tc::bar_wait(&drain_bar, 0, status);
        }
    } else {
        // ======================= epilogue: warp w reads TMEM lanes 32 (w % 4) ..
        const int q = warp & 3;
        bool ok = true;
        int it = 0;
        for (int item = bid; item < items && ok; item += grid, ++it) {
            int mt, nt, ich, s0, ns;
            item_of(item, mt, nt, ich, s0, ns);
            const int t0 = nt * kRouterTileN, n = min(kRouterTileN, T - t0), nmma = (n + 15) & ~15;
            ok = warp_wait(&accf_bar, it & 1, status);
            if (!ok) break;
            tc::fence_after();
            const int e = mt * kTileM + 32 * q + lane;
            const float b = (bias && e < E) ? bias[e] : 0.0f;
            const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
            for (int c0 = 0; c0 < nmma; c0 += 16) {
                float v[16];
                if (split) {  // the item's raw chunk sums
                    uint32_t r0[16];
                    tc::ld16(tl + c0, r0);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r0[i]);
                } else {
                    for (int ch0 = 0; ch0 < chunks; ch0 += 4) {  // chunk sums in chunk order, 4 loads in flight
                        uint32_t r[4][16];
                        const int nc = min(4, chunks - ch0);
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            if (jj < nc) tc::ld16_nowait(tl + (ch0 + jj) * ccols + c0, r[jj]);
                        tc::ld_wait();
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            if (jj < nc) {
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    v[i] = (ch0 + jj == 0) ? __uint_as_float(r[jj][i]) : v[i] + __uint_as_float(r[jj][i]);
                            }
                    }
                }
                float* lp = split ? logits + (int64_t)ich * T * E : logits;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < n && e < E) lp[(int64_t)(t0 + c0 + i) * E + e] = split ? v[i] : v[i] + b;
            }
            tc::fence_before();
            mbar_arrive(&acce_bar);
        }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- activation gather, combine
// xg[row] = fp16(x[token of row]) in group order: rows [0, offsets[E]) are
// the routed pairs (token pairs[row] / k), rows T*k + t the shared expert's.
// One warp per RPW rows (32 lanes x 16 bytes per step, eight steps in flight),
// 8 warps per CTA: RPW = 4 for large batches (a few thousand CTAs that each
// stream whole rows), 1 for small ones (more warps, each one round of loads).
constexpr int kGatherWarps = 8;
constexpr int kGatherSmallRows = 148 * kGatherWarps * 16;  // below this many rows: one row per warp

template <int RPW>
__global__ void __launch_bounds__(kGatherWarps * 32)
    gather_f16_kernel(const __nv_bfloat16* __restrict__ x, int T, int d, int k, int n_shared,
                      const int32_t* __restrict__ pairs, const int32_t* __restrict__ n_pairs,
                      __half* __restrict__ xg, uint32_t* status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = T * k + n_shared * T, np = *n_pairs;
    const int r0 = (blockIdx.x * kGatherWarps + warp) * RPW;
    int tok[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int row = r0 + i;
        tok[i] = -1;
        if (row < T * k) {
            if (row < np) tok[i] = __ldg(&pairs[row]) / k;
        } else if (row < rows) {
            tok[i] = row - T * k;
        }
    }
    bool finite = true;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        if (tok[i] < 0) continue;
        const __nv_bfloat16* src = x + (int64_t)tok[i] * d;
        __half* dst = xg + (int64_t)(r0 + i) * d;
#pragma unroll 8
        for (int c = lane * 8; c < d; c += 256) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + c));
            const uint32_t in[4] = {v.x, v.y, v.z, v.w};
            uint32_t out[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(in[j] << 16), hi = __uint_as_float(in[j] & 0xFFFF0000u);
                finite = finite && fabsf(lo) <= 65504.0f && fabsf(hi) <= 65504.0f;
                const __half2 hv = __floats2half2_rn(lo, hi);
                out[j] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(dst + c) = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
    if (!finite) flag_status(status, kStatusRange);
}

// y[t] = o[shared row of t] + sum_r o[row of (t, r)] (already weighted), fixed order
__global__ void combine_f16_kernel(const CombineArgs a, const __half* __restrict__ o) {
    const int t = blockIdx.y;
    const int n = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (n >= a.d) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    auto add_row = [&](int64_t row) {
        const uint4 v = *reinterpret_cast<const uint4*>(o + row * a.d + n);
        const __half2* h2 = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __half22float2(h2[j]);
            acc[2 * j] += f.x;
            acc[2 * j + 1] += f.y;
        }
    };
    if (a.n_shared) add_row((int64_t)a.T * a.k + t);
    for (int r0 = 0; r0 < a.k; r0 += 4) {  // slots in order, four positions and rows in flight
        int pos[4];
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) pos[j] = r0 + j < a.k ? a.inv[(int64_t)t * a.k + r0 + j] : -1;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (pos[j] >= 0) v[j] = *reinterpret_cast<const uint4*>(o + (int64_t)pos[j] * a.d + n);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (pos[j] >= 0) {
                const __half2* h2 = reinterpret_cast<const __half2*>(&v[j]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __half22float2(h2[q]);
                    acc[2 * q] += f.x;
                    acc[2 * q + 1] += f.y;
                }
            }
    }
    if (a.out_fp32) {
        float* y = static_cast<float*>(a.y) + (int64_t)t * a.d + n;
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = a.accumulate ? y[j] + acc[j] : acc[j];
    } else {
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y) + (int64_t)t * a.d + n;
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v0 = acc[2 * j], v1 = acc[2 * j + 1];
            if (a.accumulate) {
                v0 += __bfloat162float(y[2 * j]);
                v1 += __bfloat162float(y[2 * j + 1]);
            }
            const __nv_bfloat162 b = __floats2bfloat162_rn(v0, v1);
            out[j] = *reinterpret_cast<const uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(y) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ---------------------------------------------------------------- launchers
static int num_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return sms;
}

template <int BITS, bool GATEUP>
static cudaError_t gemm_bits(const GemmArgs& g, const GemmMaps& m, cudaStream_t s) {
    using C = GemmCfg<BITS, GATEUP>;
    auto kern = expert_gemm_kernel<BITS, GATEUP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<num_sms(), kExpertThreads, C::kSmem, s>>>(g, m.b_small, m.b_big, m.codes, m.scales);
    return cudaGetLastError();
}

size_t tile_desc_count(int T, int k, int E, int n_shared, int jt) {
    return (size_t)max_token_tiles(T, k, E, n_shared) * (size_t)jt;
}

cudaError_t launch_build_tiles(const ExpertArgs& a, int4* desc_gu, int4* desc_dn, int32_t* counts, cudaStream_t s) {
    if (a.n_shared + a.E > kTileMaxSlots) return cudaErrorInvalidValue;
    build_tiles_kernel<<<1, kTileListThreads, 0, s>>>(a, a.f / kTileM, a.d / kTileM, desc_gu, desc_dn, counts);
    return cudaGetLastError();
}

cudaError_t launch_gemm_gateup(const ExpertArgs& a, const GemmMaps& maps, const int4* desc, const int32_t* counts,
                               cudaStream_t s) {
    GemmArgs g;
    g.e = a;
    g.wsorted = nullptr;
    g.o = nullptr;
    g.desc = desc;
    g.n_tiles = counts;
    switch (a.bits) {
        case 2: return gemm_bits<2, true>(g, maps, s);
        case 3: return gemm_bits<3, true>(g, maps, s);
        case 4: return gemm_bits<4, true>(g, maps, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_down(const ExpertArgs& a, const GemmMaps& maps, const float* wsorted, void* o,
                             const int4* desc, const int32_t* counts, cudaStream_t s) {
    GemmArgs g;
    g.e = a;
    g.wsorted = wsorted;
    g.o = static_cast<__half*>(o);
    g.desc = desc;
    g.n_tiles = counts + 1;
    switch (a.bits_down ? a.bits_down : a.bits) {
        case 2: return gemm_bits<2, false>(g, maps, s);
        case 3: return gemm_bits<3, false>(g, maps, s);
        case 4: return gemm_bits<4, false>(g, maps, s);
        default: return cudaErrorInvalidValue;
    }
}

using Encode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                            const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                            CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static Encode encoder() {
    static Encode encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return nullptr;
        encode = reinterpret_cast<Encode>(fn);
    }
    return encode;
}

static cudaError_t encode_2d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base,
                             int64_t rows, int64_t row_elems, int box_inner, int box_rows, CUtensorMapSwizzle swz) {
    Encode encode = encoder();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)row_elems, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_elems * elem_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Maps of a row-major fp16 activation matrix [rows x cols] (xg or h) for
// boxes of 64 columns (128 B) x 32 or 256 rows, 128-byte swizzle (the MMA's
// K-major layout); rows past the end read as zeros.
cudaError_t make_row_maps(GemmMaps* m, const void* base, int64_t rows, int cols) {
    cudaError_t e = encode_2d(&m->b_small, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, rows, cols, 64, kBRowsSmall,
                              CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    return encode_2d(&m->b_big, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, rows, cols, 64, kBRowsBig,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

static cudaError_t encode_3d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base,
                             const cuuint64_t (&dims)[3], const cuuint64_t (&strides_bytes)[2], const cuuint32_t (&box)[3]);

// Maps of a layer's packed codes and scales for one kernel of the expert
// GEMM: gate/up (N = f rows per matrix, K = d) or down (N = d, K = f).  Every
// matrix is N/16 row tiles of K/128 super-tiles (256 b bytes of codes and 64
// fp16 scales each), at its own code width b.
//   codes:  a 3-D view (32-bit word, row tile, expert) starting at the
//           kernel's first matrix -- gate and up are adjacent at the same
//           width, so their 2N/16 row tiles form one plane -- with the
//           expert stride f*d*(2*bits + bits_down)/8 bytes, so the two
//           kernels may read different widths.  One box = 8 row tiles x one
//           super-tile.
//   scales: every expert's three matrices stacked as rows of 16-row tiles
//           (the scales do not depend on the code width), row
//           (expert * 3 + mat) * N/16 + tile.  One box = 8 row tiles x 64.
cudaError_t make_weight_maps(GemmMaps* m, const void* codes, const void* scales, int n_experts_total, int d, int f,
                             int bits, int bits_down, bool gateup) {
    const int N = gateup ? f : d, K = gateup ? d : f, b = gateup ? bits : bits_down;
    const int64_t code_stride = (int64_t)f * d * (2 * bits + bits_down) / 8;
    const uint8_t* base = static_cast<const uint8_t*>(codes) + (gateup ? 0 : 2 * (int64_t)f * d * bits / 8);
    const int64_t words = (int64_t)(K / 128) * 64 * b;  // per row tile
    const cuuint64_t cdims[3] = {(cuuint64_t)words, (cuuint64_t)((gateup ? 2 : 1) * (N / 16)),
                                 (cuuint64_t)n_experts_total};
    const cuuint64_t cstr[2] = {(cuuint64_t)words * 4, (cuuint64_t)code_stride};
    const cuuint32_t cbox[3] = {(cuuint32_t)(64 * b), 8, 1};
    cudaError_t e = encode_3d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, base, cdims, cstr, cbox);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)n_experts_total * 3 * (N / 16);
    return encode_2d(&m->scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, scales, rows, (int64_t)(K / 128) * 64, 64, 8,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Maps of the down matrices for the clustered decode kernel: a 3-D view
// (super-tile words, 16-row tile, expert) of every expert's down codes and
// scales, any code widths.  One box = RTI row tiles x one super-tile column,
// so a kernel fetches the 128 input columns [128j, 128j + 128) of RTI
// consecutive row tiles with one instruction per map.
static cudaError_t encode_3d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base,
                             const cuuint64_t (&dims)[3], const cuuint64_t (&strides_bytes)[2], const cuuint32_t (&box)[3]) {
    Encode encode = encoder();
    if (!encode) return cudaErrorNotSupported;
    (void)elem_bytes;
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(map, type, 3, const_cast<void*>(base), dims, strides_bytes, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_pair_down_maps(CUtensorMap* codes_map, CUtensorMap* scales_map, const void* codes,
                                const void* scales, int n_experts_total, int d, int f, int bits, int bits_down) {
    const int FC = f / 128, RT = d / 16, RTI = d / 64;
    if (RTI < 1 || RTI > 256) return cudaErrorInvalidValue;
    const int64_t mg = (int64_t)f * d * bits / 8, msc = (int64_t)f * d / 32;
    const int64_t code_stride = (int64_t)f * d * (2 * bits + bits_down) / 8;
    const cuuint64_t cdims[3] = {(cuuint64_t)FC * 64 * bits_down, (cuuint64_t)RT, (cuuint64_t)n_experts_total};
    const cuuint64_t cstr[2] = {(cuuint64_t)FC * 256 * bits_down, (cuuint64_t)code_stride};
    const cuuint32_t cbox[3] = {(cuuint32_t)(64 * bits_down), (cuuint32_t)RTI, 1};
    cudaError_t e = encode_3d(codes_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4,
                              static_cast<const uint8_t*>(codes) + 2 * mg, cdims, cstr, cbox);
    if (e != cudaSuccess) return e;
    const cuuint64_t sdims[3] = {(cuuint64_t)FC * 64, (cuuint64_t)RT, (cuuint64_t)n_experts_total};
    const cuuint64_t sstr[2] = {(cuuint64_t)FC * 128, (cuuint64_t)(3 * msc * 2)};
    const cuuint32_t sbox[3] = {64, (cuuint32_t)RTI, 1};
    return encode_3d(scales_map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, static_cast<const uint16_t*>(scales) + 2 * msc,
                     sdims, sstr, sbox);
}

cudaError_t launch_router_gemm(const RouteArgs& a, uint32_t* status, cudaStream_t s) {
    const int smem = kRouterStages * kRouterStage + 1024;
    cudaError_t e = cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // row-major bf16 [E x d] and [T x d], boxes of 64 columns (128 B) x 128 rows, 128-byte swizzle
    CUtensorMap wmap, xmap;
    e = encode_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.wr, a.E, a.d, 64, kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.x, a.T, a.d, 64, kRouterTileN,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const int tiles = ((a.E + kTileM - 1) / kTileM) * ((a.T + kRouterTileN - 1) / kRouterTileN);
    const int chunks = router_gemm_chunks(a.T, a.d), split = router_gemm_split(a.T) ? 1 : 0;
    if (split && a.logit_parts != chunks) return cudaErrorInvalidValue;  // the caller sized logits for the chunks
    const int items = tiles * (split ? chunks : 1);
    router_gemm_kernel<<<min(items, num_sms()), kRouterThreads, smem, s>>>(wmap, xmap, a.T, a.d, a.bias, a.E,
                                                                          a.logits, chunks, split, status);
    return cudaGetLastError();
}

// Batches of at most one token tile are split by K chunk over the CTAs.
bool router_gemm_split(int T) { return T <= kRouterTileN; }

// K chunks of the router GEMM for T tokens, a power of two dividing the d / 64
// steps, at most 32.  Split (T <= 128): 32, one step each at d = 2048.  Else as
// many as the 512 tensor-memory columns hold at the tile's 128 columns: 4.
int router_gemm_chunks(int T, int d) {
    const int cols = router_gemm_split(T) ? 16 : kRouterTileN;  // split: one accumulator per CTA
    const int steps = d / kStepK;
    int c = 1;
    while (2 * c <= 512 / cols && 2 * c <= 32 && steps % (2 * c) == 0) c *= 2;
    return c;
}

// logits[t][e] = (sum over chunks c, in order, of parts[c][t][e]) + bias_e: the
// split router GEMM's chunk sums reduced as its unsplit epilogue would.
__global__ void router_reduce_kernel(const float* __restrict__ parts, int chunks, int T, int E,
                                     const float* __restrict__ bias, float* __restrict__ logits) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, n = (int64_t)T * E;
    if (i >= n) return;
    float v = parts[i];
#pragma unroll 8
    for (int c = 1; c < chunks; ++c) v += parts[(int64_t)c * n + i];
    logits[i] = v + (bias ? bias[i % E] : 0.0f);
}

cudaError_t launch_router_reduce(const float* parts, int chunks, int T, int E, const float* bias, float* logits,
                                 cudaStream_t s) {
    const int64_t n = (int64_t)T * E;
    if (n == 0) return cudaSuccess;
    router_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(parts, chunks, T, E, bias, logits);
    return cudaGetLastError();
}

// Error bound of the tensor-core logits, in the units of the top-k kernel's
// certificate delta = 2 * depth * 2^-24 * (||W_r,e|| ||x|| + |bias_e|).
// Model: each MMA adds 16 exact bf16 x bf16 products to its chunk's fp32
// accumulator; aligning the 17 terms to the largest exponent and truncating
// costs at most one fp32 ulp of that largest term per term, and every term is
// at most the chunk's sum_i |w_i x_i| <= ||w|| ||x||.  Summed over a chunk's
// d / (16 c) steps (doubled for margin), the chunk errors together stay
// within 34 * d / (16 c) units of the whole sum; then c - 1 fp32 adds of the
// chunk sums and the bias add, one unit each.
float router_gemm_depth(int d, int chunks) {
    return 34.0f * (float)(d / 16 / chunks) + (float)(chunks - 1) + 2.0f;
}

cudaError_t launch_gather_f16(const void* x, int T, int d, int k, int n_shared, const int32_t* pairs,
                              const int32_t* n_pairs, void* xg, uint32_t* status, cudaStream_t s) {
    const int rows = T * k + n_shared * T;
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    if (rows < kGatherSmallRows)
        gather_f16_kernel<1><<<(rows + kGatherWarps - 1) / kGatherWarps, kGatherWarps * 32, 0, s>>>(
            xb, T, d, k, n_shared, pairs, n_pairs, static_cast<__half*>(xg), status);
    else
        gather_f16_kernel<4><<<(rows + 4 * kGatherWarps - 1) / (4 * kGatherWarps), kGatherWarps * 32, 0, s>>>(
            xb, T, d, k, n_shared, pairs, n_pairs, static_cast<__half*>(xg), status);
    return cudaGetLastError();
}

cudaError_t launch_combine_f16(const CombineArgs& a, const void* o, cudaStream_t s) {
    dim3 grid((a.d / 8 + 127) / 128, a.T);
    combine_f16_kernel<<<grid, 128, 0, s>>>(a, static_cast<const __half*>(o));
    return cudaGetLastError();
}

}  // namespace moe

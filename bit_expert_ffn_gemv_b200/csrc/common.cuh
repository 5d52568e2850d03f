// common.cuh -- device helpers shared by the routed-MoE kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "moe.h"

#define MOE_DEV __device__ __forceinline__

namespace moe {

// ---------------------------------------------------------------- status word
// bit 0: a bounded wait gave up; bit 1: an index was out of range;
// bit 2: a value did not fit an fp16 operand.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;
constexpr uint32_t kStatusRange = 4u;

MOE_DEV void flag_status(uint32_t* status, uint32_t bit) { atomicOr(status, bit); }

// ---------------------------------------------------------------- scratch meta
// Small integer block written by the bucket kernel and read by later kernels.
struct Meta {
    int32_t n_active;   // distinct routed experts with >= 1 token
    int32_t max_count;  // largest routed group
    int32_t n_fixup;    // tokens re-ranked in fp64 by the last routing
    int32_t pad[5];
};

// ---------------------------------------------------------------- packed format
// Bytes of one 16 x 128 super-tile of codes for b-bit weights.
__host__ __device__ constexpr int tile_code_bytes(int bits) { return 256 * bits; }
constexpr int kTileScaleHalfs = 64;

// ---------------------------------------------------------------- warp MMA
// D = A(16x16) * B(16x8) + C, fp32 accumulate, A row-major, B column-major.
MOE_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

MOE_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// ---------------------------------------------------------------- code decoding
// Two codes sit at bits [0..w) and [16..16+w) of `v`; OR-ing them into the
// mantissa of a 16-bit float whose value is 2^M gives (2^M + u) exactly, and
// subtracting (2^M + 2^(b-1)) leaves the signed code q exactly.
//   bf16: 0x4300 = 128.0 ; fp16: 0x6400 = 1024.0
template <bool F16>
MOE_DEV uint32_t codes_to_pair(uint32_t v, uint32_t sub2) {
    uint32_t r;
    if (F16) {
        uint32_t m = v | 0x64006400u;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(sub2));
    } else {
        uint32_t m = v | 0x43004300u;
        asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(sub2));
    }
    return r;
}

// bias constant (2^M + 2^(b-1)) in both halves
template <bool F16, int BITS>
MOE_DEV uint32_t code_sub2() {
    constexpr uint32_t h = F16 ? (0x6400u | (1u << (BITS - 1))) : (0x4300u | (1u << (BITS - 1)));
    return h | (h << 16);
}

// The 8 A-fragment registers (two k-steps of 16) of one 32-weight block for
// the calling lane.  lo: the lane's 32-bit code word (b = 2, 3: low 2 bits of
// each code; b = 4: pairs 0..3), hi: b = 3: the 16-bit plane; b = 4: the word
// holding pairs 4..7.
template <bool F16, int BITS>
MOE_DEV void decode_block(uint32_t lo, uint32_t hi, uint32_t (&a)[8]) {
    const uint32_t sub2 = code_sub2<F16, BITS>();
    if (BITS == 2) {
#pragma unroll
        for (int p = 0; p < 8; ++p) a[p] = codes_to_pair<F16>((lo >> (2 * p)) & 0x00030003u, sub2);
    } else if (BITS == 3) {
        // spread the 16-bit plane: bit p -> bit 2+p... as bit (p) of each half, then << 2
        uint32_t h32 = ((hi & 0x00FFu) | ((hi & 0xFF00u) << 8)) << 2;
#pragma unroll
        for (int p = 0; p < 8; ++p)
            a[p] = codes_to_pair<F16>(((lo >> (2 * p)) & 0x00030003u) | ((h32 >> p) & 0x00040004u), sub2);
    } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) a[p] = codes_to_pair<F16>((lo >> (4 * p)) & 0x000F000Fu, sub2);
#pragma unroll
        for (int p = 0; p < 4; ++p) a[4 + p] = codes_to_pair<F16>((hi >> (4 * p)) & 0x000F000Fu, sub2);
    }
}

// Per-lane view of one super-tile: code words and scales for kb = 0..3.
template <int BITS>
struct TileRegs {
    uint32_t lo[4];
    uint32_t hi[4];
    uint32_t sc[4];  // fp16 pair (row g, row g+8) of block kb
};

// Load the calling lane's part of super-tile `st` (global memory).
template <int BITS>
MOE_DEV void load_tile(const uint8_t* __restrict__ codes, const __half* __restrict__ scales, int64_t st, int lane,
                       TileRegs<BITS>& t) {
    const uint8_t* base = codes + st * tile_code_bytes(BITS);
    uint4 w = __ldg(reinterpret_cast<const uint4*>(base + 16 * lane));
    t.lo[0] = w.x;
    t.lo[1] = w.y;
    t.lo[2] = w.z;
    t.lo[3] = w.w;
    if (BITS == 3) {
        uint2 hv = __ldg(reinterpret_cast<const uint2*>(base + 512 + 8 * lane));
        t.hi[0] = hv.x & 0xFFFFu;
        t.hi[1] = hv.x >> 16;
        t.hi[2] = hv.y & 0xFFFFu;
        t.hi[3] = hv.y >> 16;
    } else if (BITS == 4) {
        uint4 w2 = __ldg(reinterpret_cast<const uint4*>(base + 512 + 16 * lane));
        t.hi[0] = w2.x;
        t.hi[1] = w2.y;
        t.hi[2] = w2.z;
        t.hi[3] = w2.w;
    } else {
        t.hi[0] = t.hi[1] = t.hi[2] = t.hi[3] = 0;
    }
    uint4 s = __ldg(reinterpret_cast<const uint4*>(scales + st * kTileScaleHalfs + 8 * (lane >> 2)));
    t.sc[0] = s.x;
    t.sc[1] = s.y;
    t.sc[2] = s.z;
    t.sc[3] = s.w;
}

// The calling lane's part of one super-tile already staged in shared memory:
// `code` points at the super-tile's 256*BITS code bytes, `scale` at its 64
// fp16 scales.
template <int BITS>
MOE_DEV void load_tile_smem(const uint8_t* code, const uint8_t* scale, int lane, TileRegs<BITS>& t) {
    const uint4 w = *reinterpret_cast<const uint4*>(code + 16 * lane);
    t.lo[0] = w.x;
    t.lo[1] = w.y;
    t.lo[2] = w.z;
    t.lo[3] = w.w;
    if (BITS == 3) {
        const uint2 hv = *reinterpret_cast<const uint2*>(code + 512 + 8 * lane);
        t.hi[0] = hv.x & 0xFFFFu;
        t.hi[1] = hv.x >> 16;
        t.hi[2] = hv.y & 0xFFFFu;
        t.hi[3] = hv.y >> 16;
    } else if (BITS == 4) {
        const uint4 w2 = *reinterpret_cast<const uint4*>(code + 512 + 16 * lane);
        t.hi[0] = w2.x;
        t.hi[1] = w2.y;
        t.hi[2] = w2.z;
        t.hi[3] = w2.w;
    } else {
        t.hi[0] = t.hi[1] = t.hi[2] = t.hi[3] = 0;
    }
    const uint4 sv = *reinterpret_cast<const uint4*>(scale + 16 * (lane >> 2));
    t.sc[0] = sv.x;
    t.sc[1] = sv.y;
    t.sc[2] = sv.z;
    t.sc[3] = sv.w;
}

// ---------------------------------------------------------------- bulk copies (TMA, 1-D) and mbarriers
MOE_DEV uint32_t smem_addr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// one arrival that also announces `bytes` of transactions still to land
MOE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
MOE_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
MOE_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// global -> shared copy completed on `bar` (16-byte aligned, bytes % 16 == 0)
MOE_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
// order earlier generic-proxy accesses before later async-proxy (bulk copy) ones
MOE_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
MOE_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

MOE_DEV float silu(float g) { return g / (1.0f + __expf(-g)); }

MOE_DEV float bf16_bits_to_float(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

}  // namespace moe

// synth_gpu.cu -- device twin of synth.c: the same seeded inputs, bit for bit.
//
// Generates a whole layer's packed expert weights (and bf16 normal tensors)
// directly in device memory, for workloads too large to generate on the host
// (one full-shape layer is 2.4e9 weights; the 48-layer set is 1.2e11).  Every
// value follows the definitions in synth.c: splitmix64 counters, the polar
// method with the series logarithm evaluated in the same order with explicit
// round-to-nearest double operations (no FMA contraction; built with
// -fmad=false as well), the block quantiser and the tiled packing.  Inputs
// only: nothing here is part of the layer's arithmetic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define G64 0x9E3779B97F4A7C15ULL

__host__ __device__ static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__host__ __device__ static inline uint64_t key_of(uint64_t master, uint32_t layer, uint32_t tensor, uint32_t expert) {
    uint64_t k = mix64(master + G64);
    k = mix64(k + G64 * (1 + (uint64_t)layer));
    k = mix64(k + G64 * (1 + (uint64_t)tensor));
    k = mix64(k + G64 * (1 + (uint64_t)expert));
    return k;
}

__device__ static double dev_ln(double s) {
    uint64_t b = (uint64_t)__double_as_longlong(s);
    int e = (int)((b >> 52) & 0x7FF) - 1023;
    uint64_t mb = (b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL;
    double m = __longlong_as_double((long long)mb);
    if (m > 1.4142135623730951) {
        m = __dmul_rn(m, 0.5);
        e += 1;
    }
    double z = __ddiv_rn(__dsub_rn(m, 1.0), __dadd_rn(m, 1.0));
    double w = __dmul_rn(z, z);
    double p = __ddiv_rn(1.0, 23.0);
    for (int j = 21; j >= 1; j -= 2) p = __dadd_rn(__dmul_rn(p, w), __ddiv_rn(1.0, (double)j));
    double lm = __dmul_rn(__dmul_rn(2.0, z), p);
    return __dadd_rn(__dmul_rn((double)e, 0.6931471805599453), lm);
}

__device__ static void dev_pair(uint64_t key, uint64_t n, double& z0, double& z1) {
    for (uint64_t a = 0; a < 64; ++a) {
        uint64_t r = mix64(key + G64 * (((n << 6) | a) + 1));
        double u = __dsub_rn(__dmul_rn(__dadd_rn((double)(uint32_t)r, 0.5), 4.656612873077392578125e-10), 1.0);
        double v =
            __dsub_rn(__dmul_rn(__dadd_rn((double)(uint32_t)(r >> 32), 0.5), 4.656612873077392578125e-10), 1.0);
        double s = __dadd_rn(__dmul_rn(u, u), __dmul_rn(v, v));
        if (s >= 1.0 || s == 0.0) continue;
        double f = __dsqrt_rn(__ddiv_rn(__dmul_rn(-2.0, dev_ln(s)), s));
        z0 = __dmul_rn(u, f);
        z1 = __dmul_rn(v, f);
        return;
    }
    z0 = 0.0;
    z1 = 0.0;
}

// One CTA of 64 threads per 16 x 128 super-tile of one matrix.  Thread t
// generates and quantises the 32-weight block (row t/4, block t%4); lanes
// 0..31 then pack the super-tile.
// Matrices mat0 .. mat0 + gridDim.y - 1 of each expert, all at width BITS:
// expert e's codes start at e * code_stride, matrix mat0's at code_off within
// them (the next matrices follow at f*d*BITS/8 apart).
template <int BITS>
__global__ void __launch_bounds__(64) gen_matrix_kernel(uint64_t master, uint32_t layer, int d, int f, int expert0,
                                                        int mat0, int64_t code_stride, int64_t code_off,
                                                        uint8_t* __restrict__ codes, uint16_t* __restrict__ scales) {
    __shared__ uint8_t us[16][128];
    __shared__ uint16_t ss[16][4];
    const int mat = mat0 + (int)blockIdx.y;     // 0 gate, 1 up, 2 down
    const int expert = expert0 + blockIdx.z;
    const int N = mat < 2 ? f : d, K = mat < 2 ? d : f;
    const int KT = K / 128;
    const int st = blockIdx.x;
    if (st >= (N / 16) * KT) return;
    const int R = st / KT, C = st % KT;
    const uint64_t key = key_of(master, layer, 3u + (uint32_t)mat, (uint32_t)expert);
    const int bias = 1 << (BITS - 1);

    {
        const int r = threadIdx.x >> 2, kb = threadIdx.x & 3;
        const int64_t n = 16 * R + r;
        const int64_t i0 = n * K + 128 * C + 32 * kb;  // even
        float w[32];
        for (int p = 0; p < 16; ++p) {
            double z0, z1;
            dev_pair(key, (uint64_t)(i0 / 2 + p), z0, z1);
            w[2 * p] = __double2float_rn(__dmul_rn(0.02, z0));
            w[2 * p + 1] = __double2float_rn(__dmul_rn(0.02, z1));
        }
        float amax = 0.0f;
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(w[k]));
        const __half sh = __float2half_rn(__fdiv_rn(amax, (float)bias));
        const float sf = __half2float(sh);
        for (int k = 0; k < 32; ++k) {
            int q = 0;
            if (sf != 0.0f) {
                q = __float2int_rn(__fdiv_rn(w[k], sf));
                q = q < -bias ? -bias : (q > bias - 1 ? bias - 1 : q);
            }
            us[r][32 * kb + k] = (uint8_t)(q + bias);
        }
        ss[r][kb] = __half_as_ushort(sh);
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x, g = lane >> 2, c = lane & 3;
    const int64_t mat_codes = (int64_t)f * d * BITS / 8, mat_scales = (int64_t)f * d / 32;
    uint8_t* cb = codes + (int64_t)blockIdx.z * code_stride + code_off + (int64_t)(mat - mat0) * mat_codes +
                  (int64_t)st * 256 * BITS;
    uint16_t* sb = scales + ((int64_t)blockIdx.z * 3 + mat) * mat_scales + (int64_t)st * 64;
    uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
    for (int kb = 0; kb < 4; ++kb)
        for (int p = 0; p < 8; ++p)
            for (int e = 0; e < 2; ++e) {
                const int ks = p >> 2, reg = p & 3, half = reg & 1, hi8 = reg >> 1;
                const int r = g + 8 * half, kk = 32 * kb + 16 * ks + 8 * hi8 + 2 * c + e;
                const uint32_t u = us[r][kk];
                if (BITS == 4) {
                    const int sh = 4 * (p & 3) + 16 * e;
                    if (p < 4) lo[kb] |= (u & 15u) << sh;
                    else hi[kb] |= (u & 15u) << sh;
                } else {
                    lo[kb] |= (u & 3u) << (2 * p + 16 * e);
                    if (BITS == 3) hi[kb] |= ((u >> 2) & 1u) << (p + 8 * e);
                }
            }
    reinterpret_cast<uint4*>(cb + 16 * lane)[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    if (BITS == 3)
        reinterpret_cast<uint2*>(cb + 512 + 8 * lane)[0] =
            make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
    if (BITS == 4) reinterpret_cast<uint4*>(cb + 512 + 16 * lane)[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    // scales: fp16 number g*8 + kb*2 + half
    reinterpret_cast<uint4*>(sb + 8 * g)[0] =
        make_uint4((uint32_t)ss[g][0] | ((uint32_t)ss[g + 8][0] << 16), (uint32_t)ss[g][1] | ((uint32_t)ss[g + 8][1] << 16),
                   (uint32_t)ss[g][2] | ((uint32_t)ss[g + 8][2] << 16), (uint32_t)ss[g][3] | ((uint32_t)ss[g + 8][3] << 16));
}

__global__ void gen_bf16_kernel(uint64_t key, int64_t n, double stdv, uint16_t* __restrict__ out) {
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (2 * p >= n) return;
    double z0, z1;
    dev_pair(key, (uint64_t)p, z0, z1);
    float a = __double2float_rn(__dmul_rn(stdv, z0)), b = __double2float_rn(__dmul_rn(stdv, z1));
    out[2 * p] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
    if (2 * p + 1 < n) out[2 * p + 1] = __bfloat16_as_ushort(__float2bfloat16_rn(b));
}

template <int B>
static void launch_gen(uint64_t master, uint32_t layer, int d, int f, int expert0, int n_experts, int mat0, int nmat,
                       int64_t code_stride, int64_t code_off, uint8_t* c, uint16_t* sc, cudaStream_t s) {
    const int st_gu = (f / 16) * (d / 128), st_dn = (d / 16) * (f / 128);
    dim3 grid(st_gu > st_dn ? st_gu : st_dn, nmat, n_experts);
    gen_matrix_kernel<B><<<grid, 64, 0, s>>>(master, layer, d, f, expert0, mat0, code_stride, code_off, c, sc);
}

static void gen_mats(int bits, uint64_t master, uint32_t layer, int d, int f, int expert0, int n_experts, int mat0,
                     int nmat, int64_t code_stride, int64_t code_off, uint8_t* c, uint16_t* sc, cudaStream_t s) {
    switch (bits) {
        case 2: launch_gen<2>(master, layer, d, f, expert0, n_experts, mat0, nmat, code_stride, code_off, c, sc, s); break;
        case 3: launch_gen<3>(master, layer, d, f, expert0, n_experts, mat0, nmat, code_stride, code_off, c, sc, s); break;
        default: launch_gen<4>(master, layer, d, f, expert0, n_experts, mat0, nmat, code_stride, code_off, c, sc, s);
    }
}

extern "C" {

// Experts expert0 .. expert0+n_experts-1 of layer `layer` (gate, up, down
// each), written back to back into codes/scales (device): gate and up at
// `bits`, down at `bits_down` (0: bits), so an expert holds
// f*d*(2*bits + bits_down)/8 code bytes.  0 on success.
int synth_gpu_experts(uint64_t master, uint32_t layer, int d, int f, int expert0, int n_experts, int bits,
                      int bits_down, void* codes, void* scales, void* stream) {
    if (bits_down == 0) bits_down = bits;
    if (d % 128 || f % 128 || d <= 0 || f <= 0 || n_experts <= 0 || bits < 2 || bits > 4 || bits_down < 2 ||
        bits_down > 4)
        return -1;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* c = static_cast<uint8_t*>(codes);
    uint16_t* sc = static_cast<uint16_t*>(scales);
    const int64_t stride = (int64_t)f * d * (2 * bits + bits_down) / 8;
    if (bits_down == bits) {
        gen_mats(bits, master, layer, d, f, expert0, n_experts, 0, 3, stride, 0, c, sc, s);
    } else {
        gen_mats(bits, master, layer, d, f, expert0, n_experts, 0, 2, stride, 0, c, sc, s);
        gen_mats(bits_down, master, layer, d, f, expert0, n_experts, 2, 1, stride, 2 * (int64_t)f * d * bits / 8, c,
                 sc, s);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

// n bf16 values bf16_rne((float)(std * normal(key, i))) into out (device).
int synth_gpu_normal_bf16(uint64_t key, int64_t n, double stdv, void* out, void* stream) {
    if (n <= 0) return 0;
    const int64_t pairs = (n + 1) / 2;
    gen_bf16_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        key, n, stdv, static_cast<uint16_t*>(out));
    return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

uint64_t synth_gpu_key(uint64_t master, uint32_t layer, uint32_t tensor, uint32_t expert) {
    return key_of(master, layer, tensor, expert);
}

}  // extern "C"

/*
 * synth.c -- seeded synthetic inputs for the routed-MoE layer (host side).
 *
 * This file generates INPUTS only: activations, router weights, the Zipf
 * log-prior bias, and expert weights quantised into the packed block format.
 * It holds none of the layer's arithmetic (no dequantisation for compute, no
 * routing, no GEMV).  Both the fp64 oracle and the CUDA path consume what it
 * writes; synth_gpu.cu reproduces the same numbers bit for bit on the device
 * for workloads too large to generate on the host.
 *
 * Counter-based generator
 *   mix64(z)         the splitmix64 output function (Steele, Lea, Flood,
 *                    "Fast splittable pseudorandom number generators", 2014)
 *   draw(key, c)     = mix64(key + G*(c+1)),  G = 0x9E3779B97F4A7C15
 *   key(m,l,t,e)     = chained mix64 of master seed, layer, tensor id, expert
 *   normal #i        = Marsaglia polar method on the pair n = i/2:
 *                      attempt a = 0..63 draws r = draw(key, 64n + a);
 *                      u,v = (32-bit halves + 0.5)*2^-31 - 1  (exact doubles)
 *                      s = u*u + v*v, rejected when s >= 1 or s == 0,
 *                      z = (u or v) * sqrt(-2 ln s / s).
 *   ln               is computed here from its series (ln m = 2 atanh((m-1)/(m+1)))
 *                    with a fixed operation order, so host and device agree
 *                    bit for bit (no FMA contraction: build with
 *                    -ffp-contract=off).
 *
 * Value conventions (the readings of "N(0,0.02)", "cast to bf16",
 * "per-block fp16 scale = max|w|/2^(b-1), round-to-nearest"):
 *   weight w  = (float)(0.02 * z)       (std 0.02)
 *   x         = bf16_rne((float)z)      (std 1)
 *   W_r       = bf16_rne((float)(0.02*z))
 *   scale     s = fp16_rne(max|w| / 2^(b-1))  over a block of 32 weights along K
 *   code      q = clamp(rne(w / float(s)), -2^(b-1), 2^(b-1)-1), q = 0 when s == 0
 *   stored    u = q + 2^(b-1)  (unsigned b-bit)
 *
 * Packed tiled format of one matrix W[N x K] (N % 16 == 0, K % 128 == 0):
 *   super-tile (R, C) covers rows 16R..16R+15 and columns 128C..128C+127 and is
 *   stored at index R*(K/128) + C; codes take 256*b bytes per super-tile and
 *   scales 128 bytes.  Inside a super-tile, element (r, kk) maps to
 *     kb = kk/32, ks = (kk%32)/16, k16 = kk%16, hi8 = k16/8, c = (k16%8)/2,
 *     e = k16%2, half = r/8, g = r%8, lane = 4g + c, p = 4ks + 2hi8 + half
 *   (lane/p follow the A-operand register layout of a 16x8x16 warp MMA, so a
 *   thread of a warp loads exactly the codes it multiplies).
 *   b = 2: 32-bit word at byte lane*16 + kb*4, bits [2p + 16e, +1] = u
 *   b = 3: that word holds u & 3; a 16-bit word at byte 512 + lane*8 + kb*2
 *          holds bit (p + 8e) = u >> 2
 *   b = 4: 32-bit word at byte (p/4)*512 + lane*16 + kb*4,
 *          bits [4(p%4) + 16e, +3] = u
 *   scale of (row r, block kb): fp16 at index g*8 + kb*2 + half.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, uint64_t ctr) { return mix64(key + SYNTH_G * (ctr + 1)); }

uint64_t synth_key(uint64_t master, uint32_t layer, uint32_t tensor, uint32_t expert) {
    uint64_t k = mix64(master + SYNTH_G);
    k = mix64(k + SYNTH_G * (1 + (uint64_t)layer));
    k = mix64(k + SYNTH_G * (1 + (uint64_t)tensor));
    k = mix64(k + SYNTH_G * (1 + (uint64_t)expert));
    return k;
}

/* natural log of s in (0, 1], series form, fixed evaluation order */
static double synth_ln(double s) {
    uint64_t b;
    memcpy(&b, &s, 8);
    int e = (int)((b >> 52) & 0x7FF) - 1023;
    uint64_t mb = (b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL;
    double m;
    memcpy(&m, &mb, 8);
    if (m > 1.4142135623730951) {
        m = m * 0.5;
        e += 1;
    }
    double z = (m - 1.0) / (m + 1.0);
    double w = z * z;
    double p = 1.0 / 23.0;
    for (int j = 21; j >= 1; j -= 2) p = p * w + 1.0 / (double)j;
    double lm = (2.0 * z) * p;
    return (double)e * 0.6931471805599453 + lm;
}

/* the two normals of pair n (polar method) */
static void synth_pair(uint64_t key, uint64_t n, double* z0, double* z1) {
    for (uint64_t a = 0; a < 64; ++a) {
        uint64_t r = draw(key, (n << 6) | a);
        double u = ((double)(uint32_t)r + 0.5) * 4.656612873077392578125e-10 - 1.0;
        double v = ((double)(uint32_t)(r >> 32) + 0.5) * 4.656612873077392578125e-10 - 1.0;
        double s = u * u + v * v;
        if (s >= 1.0 || s == 0.0) continue;
        double f = sqrt((-2.0 * synth_ln(s)) / s);
        *z0 = u * f;
        *z1 = v * f;
        return;
    }
    *z0 = 0.0;
    *z1 = 0.0;
}

double synth_normal(uint64_t key, uint64_t i) {
    double z0, z1;
    synth_pair(key, i >> 1, &z0, &z1);
    return (i & 1) ? z1 : z0;
}

/* ---- rounding helpers (IEEE round-to-nearest-even) ---- */
uint16_t synth_f32_to_bf16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    if ((x & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((x >> 16) | 0x40);
    x += 0x7FFFu + ((x >> 16) & 1u);
    return (uint16_t)(x >> 16);
}

uint16_t synth_f32_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u) return (uint16_t)(sign | (ax > 0x7F800000u ? 0x7E00u : 0x7C00u));
    if (ax >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u);
    if (ax < 0x38800000u) {
        if (ax < 0x33000000u) return (uint16_t)sign;
        uint32_t e = ax >> 23;
        uint32_t m = (ax & 0x7FFFFFu) | 0x800000u;
        uint32_t shift = 126u - e;
        uint32_t q = m >> shift;
        uint32_t rem = m & ((1u << shift) - 1u);
        uint32_t half = 1u << (shift - 1u);
        if (rem > half || (rem == half && (q & 1u))) q++;
        return (uint16_t)(sign | q);
    }
    uint32_t e = (ax >> 23) - 127u + 15u;
    uint32_t q = (e << 10) | ((ax & 0x7FFFFFu) >> 13);
    uint32_t rem = ax & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (q & 1u))) q++;
    return (uint16_t)(sign | q);
}

static float f16_bits_to_f32(uint16_t h) {
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t m = h & 0x3FFu;
    float r;
    if (e == 0) {
        r = ldexpf((float)m, -24);
        if (sign) r = -r;
        return r;
    }
    uint32_t bits;
    if (e == 31) bits = sign | 0x7F800000u | (m << 13);
    else bits = sign | ((e - 15u + 127u) << 23) | (m << 13);
    memcpy(&r, &bits, 4);
    return r;
}

/* ---- tiled packing ---- */
typedef struct {
    int lane, kb, p, e, g, half;
} tile_pos;

static inline tile_pos pos_of(int r, int kk) {
    tile_pos t;
    int kin = kk & 31, k16 = kin & 15;
    int ks = kin >> 4, hi8 = k16 >> 3, c = (k16 & 7) >> 1;
    t.kb = kk >> 5;
    t.e = k16 & 1;
    t.half = r >> 3;
    t.g = r & 7;
    t.lane = 4 * t.g + c;
    t.p = 4 * ks + 2 * hi8 + t.half;
    return t;
}

int64_t synth_codes_bytes(int N, int K, int bits) { return (int64_t)N * K * bits / 8; }
int64_t synth_scales_bytes(int N, int K) { return (int64_t)N * (K / 32) * 2; }

static void put_code(uint8_t* st, int bits, tile_pos t, unsigned u) {
    if (bits == 2 || bits == 3) {
        uint32_t* w = (uint32_t*)(st + t.lane * 16 + t.kb * 4);
        int sh = 2 * t.p + 16 * t.e;
        *w = (*w & ~(3u << sh)) | ((u & 3u) << sh);
        if (bits == 3) {
            uint16_t* h = (uint16_t*)(st + 512 + t.lane * 8 + t.kb * 2);
            int hb = t.p + 8 * t.e;
            *h = (uint16_t)((*h & ~(1u << hb)) | (((u >> 2) & 1u) << hb));
        }
    } else {
        uint32_t* w = (uint32_t*)(st + (t.p >> 2) * 512 + t.lane * 16 + t.kb * 4);
        int sh = 4 * (t.p & 3) + 16 * t.e;
        *w = (*w & ~(15u << sh)) | ((u & 15u) << sh);
    }
}

/*
 * Pack signed codes q[N*K] (row-major, q in [-2^(b-1), 2^(b-1)-1]) and fp16
 * scale bits s[N*(K/32)] (row-major) into the tiled format.
 * Returns 0 on success, -1 on a bad shape or bit width.
 */
int synth_pack(int N, int K, int bits, const int8_t* q, const uint16_t* s, uint8_t* codes, uint16_t* scales) {
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || bits < 2 || bits > 4) return -1;
    int KT = K / 128, bias = 1 << (bits - 1);
    int64_t st_bytes = 256 * bits;
#pragma omp parallel for schedule(static)
    for (int R = 0; R < N / 16; ++R) {
        for (int C = 0; C < KT; ++C) {
            int64_t st = (int64_t)R * KT + C;
            uint8_t* cp = codes + st * st_bytes;
            uint16_t* sp = scales + st * 64;
            memset(cp, 0, (size_t)st_bytes);
            for (int r = 0; r < 16; ++r) {
                int n = 16 * R + r;
                for (int kk = 0; kk < 128; ++kk) {
                    int k = 128 * C + kk;
                    tile_pos t = pos_of(r, kk);
                    put_code(cp, bits, t, (unsigned)(q[(int64_t)n * K + k] + bias));
                    if ((kk & 31) == 0) sp[t.g * 8 + t.kb * 2 + t.half] = s[(int64_t)n * (K / 32) + k / 32];
                }
            }
        }
    }
    return 0;
}

/* quantise one block of 32 fp32 weights: writes q[32], returns scale bits */
static uint16_t quant_block(const float* w, int bits, int8_t* q) {
    float amax = 0.0f;
    for (int k = 0; k < 32; ++k) {
        float a = fabsf(w[k]);
        if (a > amax) amax = a;
    }
    int bias = 1 << (bits - 1);
    uint16_t sh = synth_f32_to_f16(amax / (float)bias);
    float sf = f16_bits_to_f32(sh);
    for (int k = 0; k < 32; ++k) {
        int v = 0;
        if (sf != 0.0f) {
            float t = w[k] / sf;
            v = (int)nearbyintf(t);
            if (v < -bias) v = -bias;
            if (v > bias - 1) v = bias - 1;
        }
        q[k] = (int8_t)v;
    }
    return sh;
}

/*
 * Quantise fp32 weights w[N*K] (row-major) and pack them.  q_out / s_out, when
 * not NULL, receive the signed codes and scale bits in row-major order.
 */
int synth_quantize(int N, int K, int bits, const float* w, uint8_t* codes, uint16_t* scales, int8_t* q_out,
                   uint16_t* s_out) {
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || bits < 2 || bits > 4) return -1;
    int8_t* q = q_out ? q_out : (int8_t*)malloc((size_t)N * K);
    uint16_t* s = s_out ? s_out : (uint16_t*)malloc((size_t)N * (K / 32) * 2);
    if (!q || !s) return -2;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        for (int kb = 0; kb < K / 32; ++kb)
            s[(int64_t)n * (K / 32) + kb] = quant_block(w + (int64_t)n * K + 32 * kb, bits, q + (int64_t)n * K + 32 * kb);
    int rc = synth_pack(N, K, bits, q, s, codes, scales);
    if (!q_out) free(q);
    if (!s_out) free(s);
    return rc;
}

/* fp32 weights of a generated matrix: w[i] = (float)(std * normal(key, i)), i = n*K + k */
void synth_normal_f32(uint64_t key, int64_t n, double std, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < (n + 1) / 2; ++p) {
        double z0, z1;
        synth_pair(key, (uint64_t)p, &z0, &z1);
        out[2 * p] = (float)(std * z0);
        if (2 * p + 1 < n) out[2 * p + 1] = (float)(std * z1);
    }
}

void synth_normal_bf16(uint64_t key, int64_t n, double std, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < (n + 1) / 2; ++p) {
        double z0, z1;
        synth_pair(key, (uint64_t)p, &z0, &z1);
        out[2 * p] = synth_f32_to_bf16((float)(std * z0));
        if (2 * p + 1 < n) out[2 * p + 1] = synth_f32_to_bf16((float)(std * z1));
    }
}

/* generate W[N x K] with std 0.02 from key and quantise+pack it */
int synth_expert_matrix(uint64_t key, int N, int K, int bits, uint8_t* codes, uint16_t* scales) {
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || bits < 2 || bits > 4) return -1;
    float* w = (float*)malloc((size_t)N * K * sizeof(float));
    if (!w) return -2;
    synth_normal_f32(key, (int64_t)N * K, 0.02, w);
    int rc = synth_quantize(N, K, bits, w, codes, scales, NULL, NULL);
    free(w);
    return rc;
}

/*
 * Zipf(s) log-prior: bias[e] = ln p(rank(e)), p(r) = r^-s / sum_{r'=1..E} r'^-s,
 * rank = 1 + pi(e) with pi a seeded Fisher-Yates permutation of 0..E-1.
 */
void synth_zipf_bias(uint64_t key, int E, double s, float* bias) {
    int* perm = (int*)malloc(sizeof(int) * (size_t)E);
    for (int i = 0; i < E; ++i) perm[i] = i;
    for (int i = E - 1; i > 0; --i) {
        uint64_t r = draw(key, (uint64_t)i);
        int j = (int)(((unsigned __int128)r * (unsigned __int128)(uint64_t)(i + 1)) >> 64);
        int t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
    }
    double norm = 0.0;
    for (int r = 1; r <= E; ++r) norm += pow((double)r, -s);
    for (int e = 0; e < E; ++e) bias[e] = (float)(-s * log((double)(perm[e] + 1)) - log(norm));
    free(perm);
}

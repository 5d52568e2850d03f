/*
 * oracle.c -- plain fp64 CPU implementation of the routed-MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg call this code.  It shares no code with the CUDA path and
 * reads the packed weights through its own decoder written from the format
 * definition (codes, fp16 scales, tiled layout; see FORMAT below).
 *
 * What it computes, per token t (the layer the Strata pages describe: "the
 * GPU runs the router", "10 experts selected per token", "a shared expert used
 * by every token", "the GPU combines each result" -- discuss.pytorch.kr post,
 * section "Strata's operating principle / experts split across VRAM, RAM,
 * SSD"; 48 layers x (512 routed + 1 shared) -- tech.okbari.net guide, section
 * "Strata, Qwen and GSQ-RCO are different components"), with the formulas of
 * the tiny-layer workload definition (softmax over experts, top-k with ties
 * to the lower index, renormalisation, expert = W_d (silu(W_g x) * W_u x),
 * output = shared expert + sum of renormalised weight x routed expert):
 *   1. l_e   = sum_i double(W_r[e,i]) * double(x[t,i]) + bias_e
 *   2. p_e   = exp(l_e - max l) / sum_e' exp(l_e' - max l)
 *   3. ids   = the k experts first in the order (l desc, e asc)
 *   4. w_r   = p_{ids_r} / sum_{r'} p_{ids_r'}
 *   5. per selected expert and the shared expert:
 *        What[n,k] = q[n,k] * double(s[n, k/32])
 *        g = What_g x, u = What_u x, h = g / (1 + exp(-g)) * u, o = What_d h
 *   6. y = o_shared + sum_r w_r o_r
 *      (with the route-tail skip, the caller passes drop[e] = 1 for the
 *      experts the batch-level rule removes, and their terms leave the sum;
 *      see tail_skip in __init__.py)
 * Everything is in fp64; nothing intermediate is rounded.  Step 3 is a
 * selection scan: repeatedly take the largest remaining l, the lowest index
 * among equals (NaN ranks as -inf).
 *
 * FORMAT (one matrix W[N x K], N % 16 == 0, K % 128 == 0, b = bits):
 *   the weight at (n, k) lies in super-tile (n/16, k/128), stored at index
 *   (n/16)*(K/128) + k/128, 256*b bytes of codes and 64 fp16 scales each.
 *   Inside it, with r = n%16 and j = k%128:
 *     block kb = j/32, step ks = (j%32)/16, m = j%16,
 *     lane = 4*(r%8) + (m%8)/2, pair p = 4*ks + 2*(m/8) + r/8, elem e = m%2
 *   the unsigned code u (q = u - 2^(b-1)) is:
 *     b=2: bits 2p+16e .. +1 of the LE 32-bit word at byte 16*lane + 4*kb
 *     b=3: those two bits are u%4; bit p+8e of the LE 16-bit word at byte
 *          512 + 8*lane + 2*kb is u/4
 *     b=4: bits 4(p%4)+16e .. +3 of the LE 32-bit word at byte
 *          512*(p/4) + 16*lane + 4*kb
 *   and its block scale is fp16 number 8*(r%8) + 2*kb + r/8 of the
 *   super-tile's 64 scales.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t d, f, E, k, n_shared, bits;
    int32_t bits_down; /* code width of the down matrices; 0: bits (gate, up and down alike) */
} oracle_shape;

/* ---- scalar decoders ---- */
double oracle_fp16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int ex = (h >> 10) & 31;
    int man = h & 1023;
    double v;
    if (ex == 0) v = ldexp((double)man, -24);
    else if (ex == 31) v = man ? NAN : INFINITY;
    else v = ldexp(1024.0 + man, ex - 25);
    return sign ? -v : v;
}

double oracle_bf16(uint16_t b) {
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* signed code q at (n, k) of a packed matrix */
int oracle_code(const uint8_t* codes, int N, int K, int bits, int n, int k) {
    (void)N;
    int64_t st = (int64_t)(n / 16) * (K / 128) + k / 128;
    const uint8_t* t = codes + st * 256 * bits;
    int r = n % 16, j = k % 128;
    int kb = j / 32, ks = (j % 32) / 16, m = j % 16;
    int lane = 4 * (r % 8) + (m % 8) / 2;
    int p = 4 * ks + 2 * (m / 8) + r / 8;
    int e = m % 2;
    unsigned u;
    if (bits == 4) {
        const uint8_t* w = t + 512 * (p / 4) + 16 * lane + 4 * kb;
        uint32_t word = (uint32_t)w[0] | ((uint32_t)w[1] << 8) | ((uint32_t)w[2] << 16) | ((uint32_t)w[3] << 24);
        u = (word >> (4 * (p % 4) + 16 * e)) & 15u;
    } else {
        const uint8_t* w = t + 16 * lane + 4 * kb;
        uint32_t word = (uint32_t)w[0] | ((uint32_t)w[1] << 8) | ((uint32_t)w[2] << 16) | ((uint32_t)w[3] << 24);
        u = (word >> (2 * p + 16 * e)) & 3u;
        if (bits == 3) {
            const uint8_t* hw = t + 512 + 8 * lane + 2 * kb;
            uint32_t hword = (uint32_t)hw[0] | ((uint32_t)hw[1] << 8);
            u += 4u * ((hword >> (p + 8 * e)) & 1u);
        }
    }
    return (int)u - (1 << (bits - 1));
}

double oracle_scale(const uint16_t* scales, int N, int K, int n, int k) {
    (void)N;
    int64_t st = (int64_t)(n / 16) * (K / 128) + k / 128;
    int r = n % 16, kb = (k % 128) / 32;
    return oracle_fp16(scales[st * 64 + 8 * (r % 8) + 2 * kb + r / 8]);
}

/* one dequantised row What[n, 0..K-1] */
static void dequant_row(const uint8_t* codes, const uint16_t* scales, int N, int K, int bits, int n, double* out) {
    for (int k = 0; k < K; ++k)
        out[k] = (double)oracle_code(codes, N, K, bits, n, k) * oracle_scale(scales, N, K, n, k);
}

/* dequantised matrix What[N x K] (row-major) */
int oracle_dequant(int N, int K, int bits, const uint8_t* codes, const uint16_t* scales, double* out) {
    if (N <= 0 || K <= 0 || N % 16 || K % 128 || bits < 2 || bits > 4) return -1;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) dequant_row(codes, scales, N, K, bits, n, out + (int64_t)n * K);
    return 0;
}

static int shape_ok(const oracle_shape* s) {
    return s && s->d > 0 && s->f > 0 && s->d % 128 == 0 && s->f % 128 == 0 && s->E > 0 && s->k >= 1 &&
           s->k <= s->E && (s->n_shared == 0 || s->n_shared == 1) && s->bits >= 2 && s->bits <= 4 &&
           (s->bits_down == 0 || (s->bits_down >= 2 && s->bits_down <= 4));
}

/* ---- routing of one token ---- */
static void route_token(const oracle_shape* s, const uint16_t* x, const uint16_t* wr, const float* bias,
                        double* logits, int32_t* ids, double* w, unsigned char* taken) {
    int E = s->E, d = s->d;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += oracle_bf16(wr[(int64_t)e * d + i]) * oracle_bf16(x[i]);
        if (bias) acc += (double)bias[e];
        logits[e] = acc;
    }
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (logits[e] > mx) mx = logits[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += exp(logits[e] - mx);
    memset(taken, 0, (size_t)E);
    double psel = 0.0;
    for (int r = 0; r < s->k; ++r) {
        int best = -1;
        double bv = 0.0;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            double v = isnan(logits[e]) ? -INFINITY : logits[e];
            if (best < 0 || v > bv) {
                best = e;
                bv = v;
            }
        }
        taken[best] = 1;
        ids[r] = best;
        w[r] = exp(logits[best] - mx) / z;
        psel += w[r];
    }
    for (int r = 0; r < s->k; ++r) w[r] /= psel;
}

/*
 * Routing only: ids[T*k] (int32), w[T*k] and logits[T*E] (may be NULL).
 * x: bf16 bits [T*d]; wr: bf16 bits [E*d]; bias: [E] or NULL.
 */
int oracle_route(const oracle_shape* s, const uint16_t* x, int T, const uint16_t* wr, const float* bias,
                 int32_t* ids, double* w, double* logits) {
    if (!shape_ok(s) || T < 0 || (T > 0 && (!x || !wr || !ids || !w))) return -1;
    int E = s->E;
#pragma omp parallel
    {
        double* lg = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            route_token(s, x + (int64_t)t * s->d, wr, bias, lg, ids + (int64_t)t * s->k, w + (int64_t)t * s->k, taken);
            if (logits) memcpy(logits + (int64_t)t * E, lg, sizeof(double) * (size_t)E);
        }
        free(lg);
        free(taken);
    }
    return 0;
}

/* o = What_d (silu(What_g x) * What_u x) for one expert; row scratch of max(d, f) */
static void expert_eval(const oracle_shape* s, const uint8_t* codes, const uint16_t* scales, const double* x,
                        double* h, double* row, double* o) {
    /* per-tensor widths: gate and up at b, down at bd (the mixed precision of GSQ-RCO) */
    int d = s->d, f = s->f, b = s->bits, bd = s->bits_down ? s->bits_down : s->bits;
    int64_t mc = (int64_t)f * d * b / 8, ms = (int64_t)f * d / 32;
    const uint8_t *cg = codes, *cu = codes + mc, *cd = codes + 2 * mc;
    const uint16_t *sg = scales, *su = scales + ms, *sd = scales + 2 * ms;
    for (int j = 0; j < f; ++j) {
        double g = 0.0, u = 0.0;
        dequant_row(cg, sg, f, d, b, j, row);
        for (int i = 0; i < d; ++i) g += row[i] * x[i];
        dequant_row(cu, su, f, d, b, j, row);
        for (int i = 0; i < d; ++i) u += row[i] * x[i];
        h[j] = g / (1.0 + exp(-g)) * u;
    }
    for (int n = 0; n < d; ++n) {
        double acc = 0.0;
        dequant_row(cd, sd, d, f, bd, n, row);
        for (int j = 0; j < f; ++j) acc += row[j] * h[j];
        o[n] = acc;
    }
}

/*
 * The whole layer for T tokens.
 *   codes[e], scales[e] (e < E + n_shared; the shared expert is index E):
 *     host pointers to expert e's packed gate, up, down matrices back to back,
 *     or NULL for an expert no token may select (an error if one does).
 *   y: [T*d] fp64 output; ids/w: [T*k] (may be NULL).
 * Returns 0, -1 on bad arguments, -2 when a needed expert is NULL.
 */
int oracle_layer(const oracle_shape* s, const uint16_t* x, int T, const uint16_t* wr, const float* bias,
                 const uint8_t* const* codes, const uint16_t* const* scales, const unsigned char* drop, double* y,
                 int32_t* ids_out, double* w_out) {
    if (!shape_ok(s) || T < 0 || (T > 0 && (!x || !wr || !codes || !scales || !y))) return -1;
    int d = s->d, E = s->E, k = s->k;
    int bad = 0;
    int big = d > s->f ? d : s->f;
#pragma omp parallel
    {
        double* lg = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        double* xd = (double*)malloc(sizeof(double) * (size_t)d);
        double* h = (double*)malloc(sizeof(double) * (size_t)s->f);
        double* row = (double*)malloc(sizeof(double) * (size_t)big);
        double* o = (double*)malloc(sizeof(double) * (size_t)d);
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
        double* w = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            const uint16_t* xt = x + (int64_t)t * d;
            double* yt = y + (int64_t)t * d;
            route_token(s, xt, wr, bias, lg, ids, w, taken);
            for (int i = 0; i < d; ++i) xd[i] = oracle_bf16(xt[i]);
            for (int i = 0; i < d; ++i) yt[i] = 0.0;
            if (s->n_shared) {
                if (!codes[E] || !scales[E]) {
#pragma omp atomic write
                    bad = 1;
                } else {
                    expert_eval(s, codes[E], scales[E], xd, h, row, o);
                    for (int i = 0; i < d; ++i) yt[i] = o[i];
                }
            }
            for (int r = 0; r < k; ++r) {
                int e = ids[r];
                if (drop && drop[e]) continue; /* route-tail skip: the pair leaves the sum, w keeps its value */
                if (!codes[e] || !scales[e]) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                expert_eval(s, codes[e], scales[e], xd, h, row, o);
                for (int i = 0; i < d; ++i) yt[i] += w[r] * o[i];
            }
            if (ids_out) memcpy(ids_out + (int64_t)t * k, ids, sizeof(int32_t) * (size_t)k);
            if (w_out) memcpy(w_out + (int64_t)t * k, w, sizeof(double) * (size_t)k);
        }
        free(lg);
        free(taken);
        free(xd);
        free(h);
        free(row);
        free(o);
        free(ids);
        free(w);
    }
    return bad ? -2 : 0;
}

/* number of threads a parallel region will use; n > 0 sets it first */
int oracle_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
    int used = 1;
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
    }
    return used;
}

/*
 * moe.h -- C ABI of the B200 routed Mixture-of-Experts layer.
 *
 * One routed-MoE layer of a Qwen3.8-Flash-Next-shaped model: per token, a
 * router picks k of E experts (10 of 512 per layer), each a SwiGLU FFN with
 * 2-4-bit block-quantised weights, plus one shared expert that every token
 * uses; the GPU combines the results before the next layer.  The operation is
 * the one the Strata pages describe -- discuss.pytorch.kr post, section
 * "Strata's operating principle / experts split across VRAM, RAM and SSD"
 * ("the GPU runs the router and writes the numbers of the 10 selected
 * experts ... the GPU combines each result, then moves to the next layer"),
 * and tech.okbari.net guide, section "Strata, Qwen and GSQ-RCO are different
 * components" (48 layers, 10 of 512 routed experts plus 1 shared expert
 * active per MoE layer).  The formulas are those of the tiny-layer workload
 * definition:
 *   logits  l = W_r x + bias             (W_r bf16 [E x d], bias fp32 or none)
 *   p       = softmax(l) over the E experts
 *   ids     = top-k of l, ties to the lower expert index, in rank order
 *   w_r     = p[ids_r] / sum_r' p[ids_r']
 *   expert  o_e = W_d,e (silu(W_g,e x) * W_u,e x),  silu(a) = a / (1 + e^-a)
 *   y       = o_shared + sum_r w_r o_{ids_r}
 * with What = q * s: b-bit codes q in [-2^(b-1), 2^(b-1)-1] and one fp16
 * scale s per block of 32 weights along the input dimension.
 *
 * Conventions
 *   - Every call returns a moe_status; no exception crosses the ABI.
 *   - All tensor pointers are DEVICE pointers on the handle's device unless
 *     a function says otherwise, and must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); work is
 *     enqueued asynchronously on it.
 *   - A handle is not thread-safe: use one handle per stream.
 *   - Device-side anomalies (an expert id out of range, a bounded wait that
 *     ran out) set a status word in device memory; moe_check_status()
 *     synchronises and reports it.
 *
 * Packed weight layout of one layer (memory owned by the caller, borrowed):
 *   codes : expert-major; expert e (the shared expert is e = E) holds
 *           gate [f x d], up [f x d], down [d x f], each f*d*b/8 bytes
 *           (down: f*d*bits_down/8 when bits_down is set)
 *   scales: same order, each matrix f*d/32 fp16 values
 * Each matrix W[N x K] is tiled into 16 x 128 super-tiles stored at
 * (n/16)*(K/128) + k/128, 256*b code bytes and 64 fp16 scales each.  Inside
 * a super-tile, with r = n%16 and j = k%128:
 *   kb = j/32, ks = (j%32)/16, m = j%16,
 *   lane = 4*(r%8) + (m%8)/2, pair p = 4*ks + 2*(m/8) + r/8, elem e = m%2
 *   b=2: u = bits [2p+16e, +1] of the 32-bit LE word at byte 16*lane + 4*kb
 *   b=3: same two bits = u%4, plus bit (p+8e) of the 16-bit LE word at
 *        byte 512 + 8*lane + 2*kb = u/4
 *   b=4: u = bits [4(p%4)+16e, +3] of the 32-bit LE word at byte
 *        512*(p/4) + 16*lane + 4*kb
 *   q = u - 2^(b-1); the block scale is fp16 number 8*(r%8) + 2*kb + r/8 of
 *   the super-tile's 64.
 * (lane and p follow the A-operand registers of a 16x8x16 warp-level MMA, so
 * each thread of a warp loads exactly the codes it multiplies.)
 */
#ifndef MOE_H
#define MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_handle moe_handle;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* a bad argument; nothing was enqueued */
    MOE_ERR_CUDA = 2,        /* a CUDA runtime call failed */
    MOE_ERR_OOM = 3,         /* device allocation failed */
    MOE_ERR_NOT_LOADED = 4,  /* the layer has no weights loaded */
    MOE_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
    MOE_ERR_BOUNDS = 6,      /* a device-side index was out of range */
    MOE_ERR_RANGE = 7        /* a value left the range of an internal fp16
                                operand (|x| or |h| above 65504, or NaN) */
} moe_status;

typedef struct {
    int32_t d;          /* hidden size, multiple of 128 */
    int32_t f;          /* expert intermediate size, multiple of 128 */
    int32_t n_experts;  /* routed experts E, 1..1024 */
    int32_t top_k;      /* experts per token k, 1..min(E, 32) */
    int32_t n_shared;   /* shared experts, 0 or 1 */
    int32_t n_layers;   /* layers this handle can hold, >= 1 */
    int32_t bits;       /* code width b: 2, 3 or 4 */
    int32_t max_tokens; /* largest T a call may pass, >= 1 */
    int32_t bits_down;  /* code width of the down matrices: 0 (= bits) or 2..4.
                           A width other than `bits` gives per-tensor mixed
                           precision (GSQ-RCO's per-tensor bit allocation, as the
                           tech.okbari.net guide describes it in its GSQ-RCO
                           section).  Every path reads each matrix at its own
                           width: the fused decode kernel (T <= 16; the older
                           persistent kernel takes one width only), the grouped
                           GEMV and the tensor-core grouped GEMM. */
} moe_config;

typedef struct {
    const void* codes;       /* device, packed codes of all E + n_shared experts */
    const void* scales;      /* device, fp16 block scales, same order */
    const void* router_w;    /* device, bf16 [E x d] row-major */
    const float* router_bias;/* device, fp32 [E], or NULL for no bias */
} moe_layer_weights;

/* forward flags */
#define MOE_OUT_FP32 0x1u   /* y is fp32 [T x d] (default: bf16) */
#define MOE_ACCUMULATE 0x2u /* y += layer output (default: y = layer output) */
/* Path selection (default: the fused decode kernel for T <= 16, the
 * tensor-core grouped-GEMM path above -- the measured crossover). */
#define MOE_FORCE_GEMV 0x4u /* CUDA-core paths: a fused kernel up to 64 tokens, grouped GEMV above */
#define MOE_FORCE_GEMM 0x8u /* the tensor-core grouped-GEMM path whatever T is */
#define MOE_FORCE_UNFUSED 0x10u /* one kernel per step (grouped GEMV) instead of the fused persistent kernel */
/*
 * Route-tail skip (an approximation, off by default): a routed expert is not
 * computed when every token of the call that selected it ranked it at
 * position MOE_TAIL_SKIP_RANK or later (0-based, i.e. 7th to 10th of a
 * top-10).  Its (token, rank) pairs drop out of the sum; the remaining
 * weights keep their values (no second renormalisation), and the routing
 * that moe_debug_last_routing reports is unchanged.  The rule is the one the
 * discuss.pytorch.kr post describes in "Strata's operating principle /
 * experts split across VRAM, RAM and SSD" for experts outside the GPU cache;
 * here it applies to every routed expert, since all of them are resident.
 * The decision is per call: it depends on which tokens share the batch.
 */
#define MOE_ROUTE_TAIL_SKIP 0x20u
#define MOE_TAIL_SKIP_RANK 6
/*
 * Pre-norm input: the layer reads u = rmsnorm(x) instead of x, with u exactly
 * as moe_rms_normalize writes it (bf16(x / sqrt(mean(x^2) + 1e-6)), no gain):
 * the model family the pages describe normalises the residual stream before
 * each MoE layer (tech.okbari.net guide, "Strata, Qwen and GSQ-RCO are
 * different components").  With MOE_ACCUMULATE and y == x, one call is a
 * whole residual step x += layer(rmsnorm(x)).  The clustered decode kernel
 * normalises inside its launch; the other paths run the norm first into the
 * handle's scratch.  The output is bit-identical to moe_rms_normalize
 * followed by moe_forward without the flag.
 */
#define MOE_NORM_INPUT 0x40u

/*
 * Create a handle on the current CUDA device.  Checks the configuration and
 * allocates all library-owned scratch for up to cfg->max_tokens tokens.
 * Errors: INVALID_ARG (bad field, NULL pointer), OOM, CUDA.  *out is set to
 * NULL on error.
 */
moe_status moe_layer_init(const moe_config* cfg, moe_handle** out);

/*
 * Attach layer `layer`'s weights (device pointers, layout above).  The memory
 * stays owned by the caller and must outlive the handle or the next load of
 * the same layer.  Precomputes the router row norms used to certify the
 * expert selection (synchronous on the legacy default stream).
 * Errors: INVALID_ARG (NULL handle/weights/pointer, layer out of range,
 * misaligned pointer), CUDA, OOM.
 */
moe_status moe_load_layer(moe_handle* h, int32_t layer, const moe_layer_weights* w);

/*
 * Routing only: ids [T x k] int32 (rank order) and renormalised weights
 * w [T x k] fp32 for bf16 activations x [T x d].  The selection equals the
 * exact (fp64) ranking: tokens whose fp32 logits leave the order uncertain
 * are re-ranked from fp64 logits.  T = 0 is a no-op.
 * Errors: INVALID_ARG (T < 0 or > max_tokens, NULL or misaligned pointer),
 * NOT_LOADED, CUDA.
 */
moe_status moe_route(moe_handle* h, int32_t layer, const void* x, int32_t T, int32_t* ids, float* w,
                     void* stream);

/*
 * The whole layer for bf16 activations x [T x d]: writes (or, with
 * MOE_ACCUMULATE, adds to) y [T x d], bf16 or (MOE_OUT_FP32) fp32.  x and y
 * must not overlap, except y == x (bf16) with MOE_ACCUMULATE, which updates a
 * residual stream in place (x += layer(x)): every read of x is enqueued
 * before the final write of y.  T = 0 is a no-op.
 * Errors: INVALID_ARG (layer out of range, T < 0 or > max_tokens, NULL or
 * misaligned x / y, an unknown flag, MOE_FORCE_GEMV with MOE_FORCE_GEMM),
 * NOT_LOADED, CUDA; nothing is
 * enqueued on an argument error.  Device-side errors (MOE_ERR_TIMEOUT,
 * MOE_ERR_BOUNDS, MOE_ERR_RANGE) surface through moe_check_status.
 */
moe_status moe_forward(moe_handle* h, int32_t layer, const void* x, int32_t T, void* y, uint32_t flags,
                       void* stream);

/*
 * moe_forward for HOST buffers: copies x_host (bf16 [T x d]) to the device,
 * runs the layer and copies y back into y_host ([T x d], bf16 or fp32 per
 * flags), all on `stream`; returns after the result is in y_host.  Pinned
 * host memory makes the copies asynchronous DMA; pageable memory works but is
 * staged by the driver.  MOE_ACCUMULATE adds to the values already in y_host.
 * Errors: as moe_forward.
 */
moe_status moe_forward_host(moe_handle* h, int32_t layer, const void* x_host, int32_t T, void* y_host,
                            uint32_t flags, void* stream);

/*
 * Routing without any device allocation (the Strata pages have no counterpart
 * of this call; it exists for callers of this library that cannot allocate:
 * code running while a CUDA graph is captured, plug-ins whose host framework
 * owns all device memory, loops that cannot pay for cudaMalloc's implicit
 * synchronisation).  Same result as moe_route() -- ids [T x k] int32 and
 * weights w [T x k] fp32 -- but without a handle: the caller passes the router
 * weights (bf16 [n_experts x d], 16-byte aligned), the bias (fp32 [n_experts]
 * or NULL) and the activations x (bf16 [T x d]).  All device pointers.
 *
 * Intermediates live in one fixed device array inside the library (about
 * 260 KB, held by every GPU that loads the library until the process exits):
 * T * n_experts must not exceed 65536 and n_experts not 1024, else
 * MOE_ERR_INVALID_ARG and nothing is enqueued.  d must be a multiple of 128
 * and at most 8192 (the logits kernel stages 16 * d bytes of shared memory),
 * 1 <= top_k <= min(n_experts, 32); outside these limits the call returns
 * MOE_ERR_INVALID_ARG before enqueuing anything.  Every call looks the
 * array's address up on the current device (a host-side lookup that follows
 * a recreated context); the first call on a device may load the library's
 * module, so make it before any stream capture.  All calls share the array: two calls whose work overlaps
 * on the GPU (different streams, no ordering between them) race and give
 * wrong results -- order them on one stream.
 * Errors: INVALID_ARG, CUDA.
 */
moe_status moe_route_noalloc(const void* x, int32_t T, int32_t d, int32_t n_experts, int32_t top_k,
                             const void* router_w, const float* router_bias, int32_t* ids, float* w,
                             void* stream);

/*
 * Helper for callers that chain layers (not a step of the routed-MoE layer):
 * out[t] = bf16(x[t] / sqrt(mean_i x[t,i]^2 + 1e-6)) for bf16 x, out [T x d]
 * (device, 16-byte aligned, d % 8 == 0; out may equal x).  The model family
 * the pages describe normalises the residual stream before each MoE layer;
 * without it, x_{l+1} = x_l + layer(x_l) diverges, the SwiGLU output being
 * quadratic in its input.  Errors: INVALID_ARG, CUDA.
 */
moe_status moe_rms_normalize(const void* x, int32_t T, int32_t d, void* out, void* stream);

/* Free the handle's own memory (never the borrowed weights).  NULL is a no-op. */
moe_status moe_destroy(moe_handle* h);

/*
 * Debug: the fp32 values q * s of matrix `mat` (0 gate [f x d], 1 up [f x d],
 * 2 down [d x f]) of expert `expert` (E = shared) of a loaded layer, written
 * row-major to out (device), each matrix decoded at its own code width.
 * Exact: |q| <= 8 and s is fp16.
 * Errors: INVALID_ARG (expert or mat out of range, NULL or misaligned out),
 * NOT_LOADED, CUDA.
 */
moe_status moe_debug_dequant(moe_handle* h, int32_t layer, int32_t expert, int32_t mat, float* out,
                             void* stream);

/*
 * Debug: the grouping step alone, as the unfused and tensor-core paths run it
 * between routing and the expert kernels (discuss.pytorch.kr post, "how it
 * works": each token's selected experts are gathered per expert before they
 * run).  Input: ids [T x k] int32 in moe_route's layout and, optionally, the
 * routing weights w [T x k] fp32.  Output (device, 16-byte aligned):
 *   offsets [E + 1]  start of each expert's group in pairs; offsets[E] is the
 *                    number of kept pairs
 *   pairs   [T * k]  pair index t * k + r, grouped by expert in ascending
 *                    expert order, ascending t inside a group (a stable
 *                    counting sort); entries past offsets[E] are not written
 *   inv     [T * k]  position of pair t * k + r in pairs, or -1 if dropped
 *   active  [E]      experts with a non-empty group, ascending; entries past
 *                    their count are not written
 *   wsorted [T * k]  w of the pair at each position (only when w and wsorted
 *                    are both non-NULL)
 * A pair is dropped when its expert lies outside the handle's expert range
 * (moe_set_expert_range) or, with MOE_ROUTE_TAIL_SKIP in flags, when no token
 * ranked its expert before MOE_TAIL_SKIP_RANK.  At T * k >= 8192 the grouping
 * runs as three kernels over 128 CTAs, below as one CTA; both give the same
 * result.  Uses the handle's scratch: enqueue it on the stream of the handle's
 * other calls.  Ids outside [0, E) set the device status (MOE_ERR_BOUNDS).
 * Errors: INVALID_ARG (T out of range, NULL or misaligned pointer, unknown
 * flag), CUDA.
 */
moe_status moe_debug_bucket(moe_handle* h, const int32_t* ids, int32_t T, const float* w, int32_t* offsets,
                            int32_t* pairs, int32_t* inv, int32_t* active, float* wsorted, uint32_t flags,
                            void* stream);

/*
 * Debug: copy the routing the last moe_forward computed internally (rank-order
 * ids [T x k] int32 and weights [T x k] fp32, device pointers) for its T
 * tokens.  Enqueued on `stream` after that forward.  Errors: INVALID_ARG.
 */
moe_status moe_debug_last_routing(moe_handle* h, int32_t T, int32_t* ids, float* w, void* stream);

/*
 * Debug: the fp32 router logits l = W_r x + bias [T x n_experts] (device,
 * row-major) of a loaded layer as one of the two router kernels computes
 * them: tensor_cores != 0 the bf16 tcgen05 GEMM (a forward uses it above 16
 * tokens, moe_route above 64), else the CUDA-core kernel.  Each logit is within
 *   delta_e = 2 * depth * 2^-24 * (||W_r,e||_2 ||x||_2 + |bias_e|)
 * of the exact value, depth = moe_router_error_depth(d, T, tensor_cores); the
 * top-k re-ranks every token whose order these intervals leave open.
 * Errors: INVALID_ARG, NOT_LOADED, CUDA.
 */
moe_status moe_debug_router_logits(moe_handle* h, int32_t layer, const void* x, int32_t T, float* logits,
                                   int32_t tensor_cores, void* stream);

/*
 * The `depth` of the logits error bound above for hidden size d and a batch of
 * T tokens (0 if d <= 0).  The tensor-core GEMM sums the contraction in K
 * chunks, more of them for narrower token tiles, so its bound tightens for
 * T < 128; T <= 0 gives the bound that holds for every T.
 */
float moe_router_error_depth(int32_t d, int32_t T, int32_t tensor_cores);

/*
 * Synchronise the device and return the first device-side error recorded
 * since the last call (then clear it): MOE_ERR_TIMEOUT, MOE_ERR_BOUNDS,
 * MOE_ERR_RANGE or MOE_OK; MOE_ERR_CUDA if the synchronisation itself failed.
 */
moe_status moe_check_status(moe_handle* h);

/*
 * Expert parallelism: from now on, moe_forward on this handle computes only
 * the routed experts e with begin <= e < end, plus the shared expert when
 * with_shared is 1; the terms of the other experts leave the sum, which makes
 * y this handle's partial output.  Every rank routes all tokens over all E
 * experts (the router is replicated), so the ranks agree on the selection and
 * weights; summing the ranks' fp32 partial outputs over disjoint ranges that
 * cover [0, E), with the shared expert on exactly one rank, gives the layer
 * (an all-reduce; the expert weights outside the range are never read, so a
 * rank needs only its own experts' bytes at their usual offsets).  Default:
 * [0, E) with the shared expert.  Combines with MOE_ROUTE_TAIL_SKIP.
 * Errors: INVALID_ARG (NULL handle, begin < 0, end < begin, end > E,
 * with_shared not 0 or 1).
 */
moe_status moe_set_expert_range(moe_handle* h, int32_t begin, int32_t end, int32_t with_shared);

/*
 * Test hook for the device watchdog (no counterpart in the pages): from now
 * on the fused decode kernels give up a device-side wait after `spins` polls
 * (default 2^21, about half a second) instead of waiting on, and, when
 * withhold_cta >= 0, that CTA of the clustered decode kernel never announces
 * its router rows, so that every other CTA's wait for them runs out.  The
 * forward then reports MOE_ERR_TIMEOUT through moe_check_status, which also
 * resets the kernels' counters so that the handle computes correctly again
 * once the hook is off (withhold_cta = -1).  Nothing traps or hangs.
 * Errors: INVALID_ARG (NULL handle, spins = 0, withhold_cta < -1).
 */
moe_status moe_debug_wait_limit(moe_handle* h, uint32_t spins, int32_t withhold_cta);

/* Counters (moe_get_stats). */
typedef struct {
    int64_t fixup_tokens;   /* tokens of the last routing re-ranked from fp64 logits */
    int64_t active_experts; /* routed experts the last moe_forward computed (distinct
                               selected experts, less those the route-tail skip or
                               the expert range dropped) */
    int64_t max_group;      /* largest expert group of the last moe_forward */
    int64_t launches;       /* kernels this handle has launched since moe_layer_init */
    int64_t cuda_error;     /* the cudaError_t of the last CUDA call of this handle that failed
                               (0 if none): the detail behind a MOE_ERR_CUDA */
} moe_stats;

/* Synchronise the device and read the counters. */
moe_status moe_get_stats(moe_handle* h, moe_stats* out);

/* Kernel ids for the per-kernel timing of moe_profile_read. */
enum {
    MOE_K_ROUTER_LOGITS = 0,
    MOE_K_TOPK = 1,
    MOE_K_BUCKET = 2,
    MOE_K_GEMV_GATEUP = 3,
    MOE_K_GEMV_DOWN = 4,
    MOE_K_COMBINE = 5,
    MOE_K_GEMM_GATEUP = 6,
    MOE_K_GEMM_DOWN = 7,
    MOE_K_ROUTER_GEMM = 8,
    MOE_K_DECODE = 9,
    MOE_K_GATHER_F16 = 10,
    MOE_K_TILE_LIST = 11,
    MOE_K_RMS_NORM = 12,
    MOE_KERNEL_COUNT = 13
};

/*
 * Per-kernel timing.  moe_profile(h, 1) synchronises, clears the totals and
 * from then on brackets every kernel the handle launches with a pair of CUDA
 * events on the launching stream; moe_profile(h, 0) stops.  Events add a
 * little time between kernels, so time throughput with profiling off.
 */
moe_status moe_profile(moe_handle* h, int32_t enable);

/*
 * Synchronise and add up the recorded events: total_ms[i] and launches[i]
 * (arrays of MOE_KERNEL_COUNT) receive the summed device time and the launch
 * count of kernel i since moe_profile(h, 1).
 */
moe_status moe_profile_read(moe_handle* h, double* total_ms, int64_t* launches);

/* Static name of kernel id i ("unknown" when out of range). */
const char* moe_kernel_name(int32_t kernel);

/* Static text for a status code. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */

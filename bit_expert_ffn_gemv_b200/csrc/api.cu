// api.cu -- the C ABI (include/moe.h): handle, scratch, argument checks and the
// order in which the kernels of one routed-MoE layer are enqueued.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

static const char* const kKernelNames[MOE_KERNEL_COUNT] = {
    "router_logits", "topk", "bucket", "gemv_gateup", "gemv_down", "combine", "gemm_gateup", "gemm_down",
    "router_gemm", "decode_fused", "gather_f16", "tile_list", "rms_norm"};

struct moe_layer_state {
    const uint8_t* codes = nullptr;
    const uint16_t* scales = nullptr;
    const void* router_w = nullptr;
    const float* bias = nullptr;
    float* wnorm = nullptr;  // owned
    moe::GemmMaps w_gu{};    // codes/scales TMA maps, gate/up geometry
    moe::GemmMaps w_dn{};    // codes/scales TMA maps, down geometry
    CUtensorMap pair_dc{};   // down codes / scales maps of the clustered decode kernel
    CUtensorMap pair_ds{};
    bool loaded = false;
};

struct moe_handle {
    moe_config cfg{};
    int device = 0;
    std::vector<moe_layer_state> layers;
    void* arena = nullptr;
    size_t arena_bytes = 0;
    // views into the arena
    float* logits = nullptr;
    float* logit_parts = nullptr;  // chunk sums of the split router GEMM [32][min(T, 128)][E]
    int32_t* ids = nullptr;
    float* w = nullptr;
    int32_t* offsets = nullptr;
    int32_t* pairs = nullptr;
    int32_t* inv = nullptr;
    int32_t* active = nullptr;
    moe::Meta* meta = nullptr;
    uint32_t* status = nullptr;
    __half* h = nullptr;
    float* obuf = nullptr;
    double* logits64 = nullptr;
    int* sync = nullptr;
    float* part = nullptr;               // partial sums of the clustered decode kernel
    unsigned long long* ctr = nullptr;   // its monotonic counters
    uint32_t spin_limit = 1u << 21;      // polls before a device-side wait gives up
    int withhold = -1;                   // test hook: a CTA that never announces its router rows
    void* x_stage = nullptr;
    void* y_stage = nullptr;
    void* x_norm = nullptr;      // rmsnorm(x) for MOE_NORM_INPUT outside the clustered decode kernel
    void* xg = nullptr;          // fp16 x rows in group order (tensor-core path)
    moe::GemmMaps gu_maps{};     // TMA maps of xg (gate/up B) and h (down B); the
    moe::GemmMaps dn_maps{};     // codes/scales maps come from the layer
    int4* desc_gu = nullptr;     // gate/up tile descriptors
    int4* desc_dn = nullptr;     // down tile descriptors
    int32_t* n_tiles = nullptr;  // [2] descriptor counts
    float* wsorted = nullptr;    // routing weights in group order
    int32_t* bucket_cnt = nullptr;  // per-chunk expert counts (multi-CTA bucketing)
    // expert parallelism: the routed experts this handle computes, and whether it adds the shared one
    int32_t ep_begin = 0, ep_end = 1 << 30, ep_shared = 1;
    // launch accounting and optional per-kernel event timing
    int64_t launches = 0;
    int last_cuda_error = 0;  // cudaError_t of the last failed CUDA call (moe_stats.cuda_error)
    bool prof_on = false;
    std::vector<cudaEvent_t> ev;    // pairs (start, stop)
    std::vector<int> ev_kernel;     // kernel id of each recorded pair
    double prof_ms[MOE_KERNEL_COUNT] = {};
    int64_t prof_n[MOE_KERNEL_COUNT] = {};
};

namespace {


constexpr uint32_t kAllFlags = MOE_OUT_FP32 | MOE_ACCUMULATE | MOE_FORCE_GEMV | MOE_FORCE_GEMM | MOE_FORCE_UNFUSED |
                               MOE_ROUTE_TAIL_SKIP | MOE_NORM_INPUT;
constexpr float kNormEps = 1e-6f;  // the pre-norm of MOE_NORM_INPUT and moe_rms_normalize

// Shared experts this handle computes (0 when another rank owns the shared expert).
int eff_shared(const moe_handle* h) { return h->ep_shared ? h->cfg.n_shared : 0; }

// Rank from which the route-tail skip drops an expert (0: off, or no rank of k reaches it).
int skip_rank(const moe_config& c, uint32_t flags) {
    return (flags & MOE_ROUTE_TAIL_SKIP) && MOE_TAIL_SKIP_RANK < c.top_k ? MOE_TAIL_SKIP_RANK : 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// An NVTX range named after a kernel (domain "moe") around its launch, so a
// profiler's timeline shows which library step enqueued it; with no profiler
// attached the range calls return at once.
struct NvtxRange {
    explicit NvtxRange(int kernel) {
        static nvtxDomainHandle_t dom = nvtxDomainCreateA("moe");
        nvtxEventAttributes_t at = {};
        at.version = NVTX_VERSION;
        at.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
        at.messageType = NVTX_MESSAGE_TYPE_ASCII;
        at.message.ascii = moe_kernel_name(kernel);
        nvtxDomainRangePushEx(dom, &at);
        d = dom;
    }
    ~NvtxRange() { nvtxDomainRangePop(d); }
    nvtxDomainHandle_t d;
};

// Enqueue one kernel (via `f`) inside its NVTX range, counting it and, when
// profiling is on, bracketing it with a pair of events on the same stream.
template <class F>
cudaError_t run(moe_handle* h, int kernel, cudaStream_t s, F&& f) {
    h->launches++;
    const NvtxRange range(kernel);
    if (!h->prof_on) {
        const cudaError_t e = f();
        if (e != cudaSuccess) h->last_cuda_error = (int)e;
        return e;
    }
    const size_t i = 2 * h->ev_kernel.size();
    while (h->ev.size() < i + 2) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return cudaErrorMemoryAllocation;
        h->ev.push_back(e);
    }
    cudaError_t e = cudaEventRecord(h->ev[i], s);
    if (e != cudaSuccess) return e;
    e = f();
    if (e != cudaSuccess) {
        h->last_cuda_error = (int)e;
        return e;
    }
    e = cudaEventRecord(h->ev[i + 1], s);
    h->ev_kernel.push_back(kernel);
    return e;
}

moe_status check_layer(moe_handle* h, int32_t layer) {
    if (!h || layer < 0 || layer >= h->cfg.n_layers) return MOE_ERR_INVALID_ARG;
    if (!h->layers[layer].loaded) return MOE_ERR_NOT_LOADED;
    return MOE_OK;
}

// Code width of the down matrices, and whether it differs from gate/up's.
int bits_down(const moe_config& c) { return c.bits_down ? c.bits_down : c.bits; }
bool mixed_widths(const moe_config& c) { return bits_down(c) != c.bits; }

// moe_forward takes the tensor-core path (bf16 tcgen05 router, grouped
// dequant GEMMs) above kFusedMaxTokens tokens, or when forced; any code widths.
bool use_tensor_cores(const moe_config& c, int32_t T, uint32_t flags) {
    (void)c;
    if (flags & (MOE_FORCE_GEMV | MOE_FORCE_UNFUSED)) return false;
    return T > moe::kFusedMaxTokens || (flags & MOE_FORCE_GEMM);
}

// router -> certified top-k; writes ids / w (device)
moe_status do_route(moe_handle* h, int32_t layer, const void* x, int32_t T, int32_t* ids, float* w, bool tc,
                    cudaStream_t s) {
    const moe_layer_state& L = h->layers[layer];
    cudaError_t e = cudaMemsetAsync(h->meta, 0, sizeof(moe::Meta), s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    moe::RouteArgs ra;
    ra.x = x;
    ra.T = T;
    ra.d = h->cfg.d;
    ra.E = h->cfg.n_experts;
    ra.k = h->cfg.top_k;
    ra.wr = L.router_w;
    ra.bias = L.bias;
    ra.wnorm = L.wnorm;
    ra.logits = h->logits;
    ra.ids = ids;
    ra.w = w;
    ra.meta = h->meta;
    if (tc) {
        const int chunks = moe::router_gemm_chunks(T, ra.d);
        ra.depth = moe::router_gemm_depth(ra.d, chunks);
        if (moe::router_gemm_split(T)) {
            // small batch: the GEMM's chunk sums over all SMs, then their fixed-order
            // reduction into the logits (both counted as the router GEMM)
            moe::RouteArgs rp = ra;
            rp.logits = h->logit_parts;
            rp.logit_parts = chunks;
            e = run(h, MOE_K_ROUTER_GEMM, s, [&] {
                cudaError_t r = moe::launch_router_gemm(rp, h->status, s);
                if (r == cudaSuccess) r = moe::launch_router_reduce(rp.logits, chunks, T, ra.E, ra.bias, ra.logits, s);
                return r;
            });
            h->launches++;
        } else {
            e = run(h, MOE_K_ROUTER_GEMM, s, [&] { return moe::launch_router_gemm(ra, h->status, s); });
        }
    } else {
        e = run(h, MOE_K_ROUTER_LOGITS, s, [&] { return moe::launch_router_logits(ra, s); });
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(run(h, MOE_K_TOPK, s, [&] { return moe::launch_topk(ra, s); }));
}

// The fused decode kernels: the clustered kernel (any code widths) up to
// kPairMaxTokens tokens when its shared-memory layout fits, else the older
// persistent kernel (one code width) up to kDecodeMaxTokens.  Returns false,
// enqueueing nothing, when neither applies.
bool try_decode(moe_handle* h, int32_t layer, const void* x, int32_t T, void* y, uint32_t flags, cudaStream_t s,
                moe_status* st) {
    const moe_config& c = h->cfg;
    if (use_tensor_cores(c, T, flags) || (flags & MOE_FORCE_UNFUSED)) return false;
    const moe_layer_state& L = h->layers[layer];
    moe::DecodeLaunch d;
    d.T = T;
    d.d = c.d;
    d.f = c.f;
    d.E = c.n_experts;
    d.k = c.top_k;
    d.n_shared = eff_shared(h);
    d.bits = c.bits;
    d.x = x;
    d.y = y;
    d.out_fp32 = (flags & MOE_OUT_FP32) ? 1 : 0;
    d.accumulate = (flags & MOE_ACCUMULATE) ? 1 : 0;
    d.codes = L.codes;
    d.scales = L.scales;
    d.wr = L.router_w;
    d.bias = L.bias;
    d.wnorm = L.wnorm;
    d.logits = h->logits;
    d.logits64 = h->logits64;
    d.ids = h->ids;
    d.w = h->w;
    d.offsets = h->offsets;
    d.pairs = h->pairs;
    d.inv = h->inv;
    d.active = h->active;
    d.meta = h->meta;
    d.status = h->status;
    d.h = h->h;
    d.obuf = h->obuf;
    d.sync = h->sync;
    d.skip_rank = skip_rank(c, flags);
    d.e_begin = h->ep_begin;
    d.e_end = h->ep_end;
    d.bits_down = bits_down(c);
    d.part = h->part;
    d.ctr = h->ctr;
    d.spin_limit = h->spin_limit;
    d.withhold = h->withhold;
    d.down_codes_map = &L.pair_dc;
    d.down_scales_map = &L.pair_ds;
    if (T <= moe::kPairMaxTokens && moe::pair_decode_supported(d)) {
        d.norm_input = (flags & MOE_NORM_INPUT) ? 1 : 0;  // normalised inside the launch
        *st = cuda_status(run(h, MOE_K_DECODE, s, [&] { return moe::launch_decode_pair(d, s); }));
        return true;
    }
    if (T <= moe::kDecodeMaxTokens && !mixed_widths(c)) {
        if (flags & MOE_NORM_INPUT) {
            if (run(h, MOE_K_RMS_NORM, s,
                    [&] { return moe::launch_rms_normalize(x, T, c.d, h->x_norm, kNormEps, s); }) != cudaSuccess) {
                *st = MOE_ERR_CUDA;
                return true;
            }
            d.x = h->x_norm;
        }
        *st = cuda_status(run(h, MOE_K_DECODE, s, [&] { return moe::launch_decode(d, s); }));
        return true;
    }
    return false;
}

moe_status do_forward(moe_handle* h, int32_t layer, const void* x, int32_t T, void* y, uint32_t flags,
                      cudaStream_t s) {
    const moe_config& c = h->cfg;
    moe_status dst = MOE_OK;
    if (try_decode(h, layer, x, T, y, flags, s, &dst)) return dst;
    if (flags & MOE_NORM_INPUT) {  // the unfused and tensor-core paths read the normalised copy
        if (run(h, MOE_K_RMS_NORM, s, [&] { return moe::launch_rms_normalize(x, T, c.d, h->x_norm, kNormEps, s); }) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        x = h->x_norm;
    }
    const bool tc = use_tensor_cores(c, T, flags);
    cudaError_t e;
    moe_status st = do_route(h, layer, x, T, h->ids, h->w, tc, s);
    if (st != MOE_OK) return st;
    moe::BucketArgs ba;
    ba.ids = h->ids;
    ba.T = T;
    ba.k = c.top_k;
    ba.E = c.n_experts;
    ba.offsets = h->offsets;
    ba.pairs = h->pairs;
    ba.inv = h->inv;
    ba.active = h->active;
    ba.meta = h->meta;
    ba.status = h->status;
    if (tc) {
        ba.w = h->w;
        ba.wsorted = h->wsorted;
    }
    ba.cnt = h->bucket_cnt;
    ba.skip_rank = skip_rank(c, flags);
    ba.e_begin = h->ep_begin;
    ba.e_end = h->ep_end;
    // the single-CTA bucketing also builds the tensor-core path's tile list (one launch fewer)
    const bool tiles_in_bucket = tc && moe::bucket_builds_tiles(ba);
    if (tiles_in_bucket) {
        ba.desc_gu = h->desc_gu;
        ba.desc_dn = h->desc_dn;
        ba.tile_counts = h->n_tiles;
        ba.n_shared = eff_shared(h);
        ba.jt_gateup = c.f / 128;
        ba.jt_down = c.d / 128;
    }
    e = run(h, MOE_K_BUCKET, s, [&] { return moe::launch_bucket(ba, s); });
    h->launches += moe::bucket_kernel_count(ba) - 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;

    const moe_layer_state& L = h->layers[layer];
    moe::ExpertArgs ea;
    ea.T = T;
    ea.d = c.d;
    ea.f = c.f;
    ea.E = c.n_experts;
    ea.k = c.top_k;
    ea.n_shared = eff_shared(h);
    ea.bits = c.bits;
    ea.bits_down = bits_down(c);
    ea.code_stride = (int64_t)c.f * c.d * (2 * c.bits + bits_down(c)) / 8;
    ea.codes = L.codes;
    ea.scales = L.scales;
    ea.x = x;
    ea.offsets = h->offsets;
    ea.pairs = h->pairs;
    ea.active = h->active;
    ea.meta = h->meta;
    ea.h = h->h;
    ea.obuf = h->obuf;
    ea.status = h->status;
    if (tc) {
        e = run(h, MOE_K_GATHER_F16, s, [&] {
            return moe::launch_gather_f16(x, T, c.d, c.top_k, ea.n_shared, h->pairs, h->offsets + c.n_experts, h->xg,
                                          h->status, s);
        });
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        if (!tiles_in_bucket) {
            e = run(h, MOE_K_TILE_LIST, s,
                    [&] { return moe::launch_build_tiles(ea, h->desc_gu, h->desc_dn, h->n_tiles, s); });
            if (e != cudaSuccess) return MOE_ERR_CUDA;
        }
        e = run(h, MOE_K_GEMM_GATEUP, s,
                [&] {
                    moe::GemmMaps m = h->gu_maps;
                    m.codes = L.w_gu.codes;
                    m.scales = L.w_gu.scales;
                    return moe::launch_gemm_gateup(ea, m, h->desc_gu, h->n_tiles, s);
                });
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        // the fp16 partial outputs reuse the fp32 partial-output buffer
        e = run(h, MOE_K_GEMM_DOWN, s,
                [&] {
                    moe::GemmMaps m = h->dn_maps;
                    m.codes = L.w_dn.codes;
                    m.scales = L.w_dn.scales;
                    return moe::launch_gemm_down(ea, m, h->wsorted, h->obuf, h->desc_dn, h->n_tiles, s);
                });
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        e = run(h, MOE_K_GEMV_GATEUP, s, [&] { return moe::launch_gemv_gateup(ea, s); });
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        e = run(h, MOE_K_GEMV_DOWN, s, [&] { return moe::launch_gemv_down(ea, s); });
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }

    moe::CombineArgs ca;
    ca.T = T;
    ca.d = c.d;
    ca.k = c.top_k;
    ca.n_shared = eff_shared(h);
    ca.obuf = h->obuf;
    ca.inv = h->inv;
    ca.w = h->w;
    ca.y = y;
    ca.out_fp32 = (flags & MOE_OUT_FP32) != 0;
    ca.accumulate = (flags & MOE_ACCUMULATE) != 0;
    if (tc) return cuda_status(run(h, MOE_K_COMBINE, s, [&] { return moe::launch_combine_f16(ca, h->obuf, s); }));
    return cuda_status(run(h, MOE_K_COMBINE, s, [&] { return moe::launch_combine(ca, s); }));
}

// Layer, token count and flags of a forward call (both entry points).
moe_status check_forward_call(moe_handle* h, int32_t layer, int32_t T, uint32_t flags) {
    moe_status st = check_layer(h, layer);
    if (st != MOE_OK) return st;
    if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (flags & ~kAllFlags) return MOE_ERR_INVALID_ARG;
    if ((flags & MOE_FORCE_GEMV) && (flags & MOE_FORCE_GEMM)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status check_forward_args(moe_handle* h, int32_t layer, const void* x, int32_t T, const void* y,
                              uint32_t flags) {
    moe_status st = check_forward_call(h, layer, T, flags);
    if (st != MOE_OK) return st;
    if (T > 0 && (!x || !y || !aligned16(x) || !aligned16(y))) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_layer_init(const moe_config* cfg, moe_handle** out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg) return MOE_ERR_INVALID_ARG;
    const moe_config c = *cfg;
    if (c.d <= 0 || c.f <= 0 || c.d % 128 || c.f % 128 || c.n_experts < 1 || c.n_experts > 1024 || c.top_k < 1 ||
        c.top_k > c.n_experts || c.top_k > 32 || (c.n_shared != 0 && c.n_shared != 1) || c.n_layers < 1 ||
        c.n_layers > 4096 || c.bits < 2 || c.bits > 4 || c.max_tokens < 1 || c.max_tokens > (1 << 20) ||
        (c.bits_down != 0 && (c.bits_down < 2 || c.bits_down > 4)))
        return MOE_ERR_INVALID_ARG;
    moe_handle* h = new (std::nothrow) moe_handle();
    if (!h) return MOE_ERR_OOM;
    h->cfg = c;
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        delete h;
        return MOE_ERR_CUDA;
    }
    h->layers.resize(c.n_layers);

    const size_t T = (size_t)c.max_tokens, E = (size_t)c.n_experts, k = (size_t)c.top_k;
    const size_t rows = T * k + T * (size_t)c.n_shared;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += round256(bytes);
        return o;
    };
    const size_t o_logits = take(sizeof(float) * T * E);
    const size_t o_lparts = take(sizeof(float) * 32 * std::min<size_t>(T, 128) * E);
    const size_t o_ids = take(sizeof(int32_t) * T * k);
    const size_t o_w = take(sizeof(float) * T * k);
    const size_t o_off = take(sizeof(int32_t) * (E + 1));
    const size_t o_pairs = take(sizeof(int32_t) * T * k);
    const size_t o_inv = take(sizeof(int32_t) * T * k);
    const size_t o_active = take(sizeof(int32_t) * E);
    const size_t o_meta = take(sizeof(moe::Meta));
    const size_t o_status = take(sizeof(uint32_t) * 4);
    const size_t o_h = take(sizeof(__half) * rows * (size_t)c.f);
    const size_t o_obuf = take(sizeof(float) * rows * (size_t)c.d);
    const size_t o_xs = take(sizeof(uint16_t) * T * (size_t)c.d);
    const size_t o_xn = take(sizeof(uint16_t) * T * (size_t)c.d);
    const size_t o_ys = take(sizeof(float) * T * (size_t)c.d);
    const size_t o_norms = take(sizeof(float) * E * (size_t)c.n_layers);
    const size_t o_l64 = take(sizeof(double) * std::min<size_t>(T, moe::kDecodeMaxTokens) * E);
    const size_t o_xg = take(sizeof(uint16_t) * rows * (size_t)c.d);
    const size_t o_dgu = take(sizeof(int4) * moe::tile_desc_count(c.max_tokens, c.top_k, c.n_experts, c.n_shared,
                                                                   c.f / 128));
    const size_t o_ddn = take(sizeof(int4) * moe::tile_desc_count(c.max_tokens, c.top_k, c.n_experts, c.n_shared,
                                                                   c.d / 128));
    const size_t o_ntiles = take(sizeof(int32_t) * 2);
    const size_t o_wsorted = take(sizeof(float) * T * k);
    const size_t o_bcnt = take(sizeof(int32_t) * moe::bucket_scratch_words(c.n_experts));
    const size_t o_sync =
        take(sizeof(int) * moe::decode_sync_words(std::min(c.max_tokens, moe::kDecodeMaxTokens), c.n_experts, c.d));
    const size_t o_part = take(sizeof(float) * moe::pair_part_floats(c.max_tokens, c.top_k, c.n_shared, c.d, c.f));
    const size_t o_ctr = take(sizeof(unsigned long long) * moe::kPairCounters);
    h->arena_bytes = off;
    cudaError_t e = cudaMalloc(&h->arena, h->arena_bytes);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        delete h;
        return e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;
    }
    char* base = static_cast<char*>(h->arena);
    h->logits = reinterpret_cast<float*>(base + o_logits);
    h->logit_parts = reinterpret_cast<float*>(base + o_lparts);
    h->ids = reinterpret_cast<int32_t*>(base + o_ids);
    h->w = reinterpret_cast<float*>(base + o_w);
    h->offsets = reinterpret_cast<int32_t*>(base + o_off);
    h->pairs = reinterpret_cast<int32_t*>(base + o_pairs);
    h->inv = reinterpret_cast<int32_t*>(base + o_inv);
    h->active = reinterpret_cast<int32_t*>(base + o_active);
    h->meta = reinterpret_cast<moe::Meta*>(base + o_meta);
    h->status = reinterpret_cast<uint32_t*>(base + o_status);
    h->h = reinterpret_cast<__half*>(base + o_h);
    h->obuf = reinterpret_cast<float*>(base + o_obuf);
    h->logits64 = reinterpret_cast<double*>(base + o_l64);
    h->sync = reinterpret_cast<int*>(base + o_sync);
    h->part = reinterpret_cast<float*>(base + o_part);
    h->ctr = reinterpret_cast<unsigned long long*>(base + o_ctr);
    h->x_stage = base + o_xs;
    h->x_norm = base + o_xn;
    h->y_stage = base + o_ys;
    h->xg = base + o_xg;
    h->desc_gu = reinterpret_cast<int4*>(base + o_dgu);
    h->desc_dn = reinterpret_cast<int4*>(base + o_ddn);
    h->n_tiles = reinterpret_cast<int32_t*>(base + o_ntiles);
    h->wsorted = reinterpret_cast<float*>(base + o_wsorted);
    h->bucket_cnt = reinterpret_cast<int32_t*>(base + o_bcnt);
    for (int l = 0; l < c.n_layers; ++l) h->layers[l].wnorm = reinterpret_cast<float*>(base + o_norms) + E * l;
    if (cudaMemset(h->arena, 0, h->arena_bytes) != cudaSuccess ||
        moe::make_row_maps(&h->gu_maps, h->xg, (int64_t)rows, c.d) != cudaSuccess ||
        moe::make_row_maps(&h->dn_maps, h->h, (int64_t)rows, c.f) != cudaSuccess) {
        cudaFree(h->arena);
        delete h;
        return MOE_ERR_CUDA;
    }
    *out = h;
    return MOE_OK;
}

moe_status moe_load_layer(moe_handle* h, int32_t layer, const moe_layer_weights* w) {
    if (!h || !w || layer < 0 || layer >= h->cfg.n_layers) return MOE_ERR_INVALID_ARG;
    if (!w->codes || !w->scales || !w->router_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->codes) || !aligned16(w->scales) || !aligned16(w->router_w) ||
        (w->router_bias && (reinterpret_cast<uintptr_t>(w->router_bias) & 3u)))
        return MOE_ERR_INVALID_ARG;
    moe_layer_state& L = h->layers[layer];
    L.loaded = false;
    L.codes = static_cast<const uint8_t*>(w->codes);
    L.scales = static_cast<const uint16_t*>(w->scales);
    L.router_w = w->router_w;
    L.bias = w->router_bias;
    const int ne = h->cfg.n_experts + h->cfg.n_shared;
    if (moe::make_weight_maps(&L.w_gu, L.codes, L.scales, ne, h->cfg.d, h->cfg.f, h->cfg.bits, bits_down(h->cfg),
                              true) != cudaSuccess ||
        moe::make_weight_maps(&L.w_dn, L.codes, L.scales, ne, h->cfg.d, h->cfg.f, h->cfg.bits, bits_down(h->cfg),
                              false) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::make_pair_down_maps(&L.pair_dc, &L.pair_ds, L.codes, L.scales, ne, h->cfg.d, h->cfg.f, h->cfg.bits,
                                 bits_down(h->cfg)) != cudaSuccess)
        return MOE_ERR_CUDA;
    cudaError_t e = moe::launch_router_norms(L.router_w, h->cfg.n_experts, h->cfg.d, L.wnorm, 0);
    if (e == cudaSuccess) e = cudaStreamSynchronize(0);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    L.loaded = true;
    return MOE_OK;
}

moe_status moe_route(moe_handle* h, int32_t layer, const void* x, int32_t T, int32_t* ids, float* w,
                     void* stream) {
    moe_status st = check_layer(h, layer);
    if (st != MOE_OK) return st;
    if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !ids || !w || !aligned16(x) || !aligned16(ids) || !aligned16(w)) return MOE_ERR_INVALID_ARG;
    // routing alone: the CUDA-core router up to 64 tokens, the tensor-core router above
    return do_route(h, layer, x, T, ids, w, T > moe::kDecodeMaxTokens, static_cast<cudaStream_t>(stream));
}

moe_status moe_debug_router_logits(moe_handle* h, int32_t layer, const void* x, int32_t T, float* logits,
                                   int32_t tensor_cores, void* stream) {
    moe_status st = check_layer(h, layer);
    if (st != MOE_OK) return st;
    if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !logits || !aligned16(x) || !aligned16(logits)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const moe_layer_state& L = h->layers[layer];
    moe::RouteArgs ra;
    ra.x = x;
    ra.T = T;
    ra.d = h->cfg.d;
    ra.E = h->cfg.n_experts;
    ra.k = h->cfg.top_k;
    ra.wr = L.router_w;
    ra.bias = L.bias;
    ra.wnorm = L.wnorm;
    ra.logits = logits;
    ra.ids = nullptr;
    ra.w = nullptr;
    ra.meta = h->meta;
    if (tensor_cores && moe::router_gemm_split(T)) {  // chunk sums, then their fixed-order reduction
        ra.logits = h->logit_parts;
        ra.logit_parts = moe::router_gemm_chunks(T, ra.d);
        cudaError_t e = moe::launch_router_gemm(ra, h->status, s);
        if (e == cudaSuccess) e = moe::launch_router_reduce(ra.logits, ra.logit_parts, T, ra.E, ra.bias, logits, s);
        return cuda_status(e);
    }
    cudaError_t e = tensor_cores ? moe::launch_router_gemm(ra, h->status, s) : moe::launch_router_logits(ra, s);
    return cuda_status(e);
}

float moe_router_error_depth(int32_t d, int32_t T, int32_t tensor_cores) {
    if (d <= 0) return 0.0f;
    if (!tensor_cores) return (float)(d / 32 + 6);
    // T <= 0: the bound for any batch (full 128-token tiles have the fewest chunks)
    return moe::router_gemm_depth(d, moe::router_gemm_chunks(T > 0 ? T : (1 << 20), d));
}

moe_status moe_forward(moe_handle* h, int32_t layer, const void* x, int32_t T, void* y, uint32_t flags,
                       void* stream) {
    moe_status st = check_forward_args(h, layer, x, T, y, flags);
    if (st != MOE_OK || T == 0) return st;
    return do_forward(h, layer, x, T, y, flags, static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_host(moe_handle* h, int32_t layer, const void* x_host, int32_t T, void* y_host,
                            uint32_t flags, void* stream) {
    moe_status st = check_forward_call(h, layer, T, flags);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t xb = sizeof(uint16_t) * (size_t)T * h->cfg.d;
    const size_t yb = ((flags & MOE_OUT_FP32) ? sizeof(float) : sizeof(uint16_t)) * (size_t)T * h->cfg.d;
    if (cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    if ((flags & MOE_ACCUMULATE) &&
        cudaMemcpyAsync(h->y_stage, y_host, yb, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = do_forward(h, layer, h->x_stage, T, h->y_stage, flags, s);
    if (st != MOE_OK) return st;
    if (cudaMemcpyAsync(y_host, h->y_stage, yb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(s));
}

moe_status moe_rms_normalize(const void* x, int32_t T, int32_t d, void* out, void* stream) {
    if (T < 0 || d <= 0 || d % 8) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_rms_normalize(x, T, d, out, kNormEps, static_cast<cudaStream_t>(stream)));
}

moe_status moe_set_expert_range(moe_handle* h, int32_t begin, int32_t end, int32_t with_shared) {
    if (!h || begin < 0 || end < begin || end > h->cfg.n_experts || (with_shared != 0 && with_shared != 1))
        return MOE_ERR_INVALID_ARG;
    h->ep_begin = begin;
    h->ep_end = end;
    h->ep_shared = with_shared;
    return MOE_OK;
}

moe_status moe_destroy(moe_handle* h) {
    if (!h) return MOE_OK;
    cudaError_t e = cudaSuccess;
    if (h->arena) e = cudaFree(h->arena);
    for (cudaEvent_t ev : h->ev) cudaEventDestroy(ev);
    delete h;
    return cuda_status(e);
}

moe_status moe_debug_dequant(moe_handle* h, int32_t layer, int32_t expert, int32_t mat, float* out, void* stream) {
    moe_status st = check_layer(h, layer);
    if (st != MOE_OK) return st;
    const moe_config& c = h->cfg;
    if (expert < 0 || expert >= c.n_experts + c.n_shared || mat < 0 || mat > 2 || !out || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const moe_layer_state& L = h->layers[layer];
    const int64_t mc = (int64_t)c.f * c.d * c.bits / 8, ms = (int64_t)c.f * c.d / 32;
    const int64_t stride = (int64_t)c.f * c.d * (2 * c.bits + bits_down(c)) / 8;
    const int N = mat < 2 ? c.f : c.d, K = mat < 2 ? c.d : c.f;
    return cuda_status(moe::launch_dequant(L.codes + expert * stride + mat * mc, L.scales + (expert * 3 + mat) * ms,
                                           N, K, mat < 2 ? c.bits : bits_down(c), out,
                                           static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_bucket(moe_handle* h, const int32_t* ids, int32_t T, const float* w, int32_t* offsets,
                            int32_t* pairs, int32_t* inv, int32_t* active, float* wsorted, uint32_t flags,
                            void* stream) {
    if (!h || T < 0 || T > h->cfg.max_tokens || (flags & ~kAllFlags)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!ids || !offsets || !pairs || !inv || !active || !aligned16(ids) || !aligned16(offsets) ||
        !aligned16(pairs) || !aligned16(inv) || !aligned16(active) || (w && !aligned16(w)) ||
        (wsorted && !aligned16(wsorted)))
        return MOE_ERR_INVALID_ARG;
    const moe_config& c = h->cfg;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    moe::BucketArgs ba;
    ba.ids = ids;
    ba.T = T;
    ba.k = c.top_k;
    ba.E = c.n_experts;
    ba.offsets = offsets;
    ba.pairs = pairs;
    ba.inv = inv;
    ba.active = active;
    ba.meta = h->meta;
    ba.status = h->status;
    if (w && wsorted) {
        ba.w = w;
        ba.wsorted = wsorted;
    }
    ba.cnt = h->bucket_cnt;
    ba.skip_rank = skip_rank(c, flags);
    ba.e_begin = h->ep_begin;
    ba.e_end = h->ep_end;
    const cudaError_t e = run(h, MOE_K_BUCKET, s, [&] { return moe::launch_bucket(ba, s); });
    h->launches += moe::bucket_kernel_count(ba) - 1;
    return cuda_status(e);
}

moe_status moe_debug_last_routing(moe_handle* h, int32_t T, int32_t* ids, float* w, void* stream) {
    if (!h || T < 0 || T > h->cfg.max_tokens || (T > 0 && (!ids || !w))) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = (size_t)T * h->cfg.top_k;
    if (cudaMemcpyAsync(ids, h->ids, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cuda_status(cudaMemcpyAsync(w, h->w, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
}

moe_status moe_check_status(moe_handle* h) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, h->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(h->status, 0, sizeof(uint32_t)) != cudaSuccess) return MOE_ERR_CUDA;
    if (v) {
        // A launch that hit an anomaly may have left the fused kernels' counters
        // out of step: start them afresh (nothing is in flight).
        const size_t sync_bytes = sizeof(int) * moe::decode_sync_words(
                                                   std::min(h->cfg.max_tokens, moe::kDecodeMaxTokens),
                                                   h->cfg.n_experts, h->cfg.d);
        if (cudaMemset(h->sync, 0, sync_bytes) != cudaSuccess ||
            cudaMemset(h->ctr, 0, sizeof(unsigned long long) * moe::kPairCounters) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    if (v & moe::kStatusTimeout) return MOE_ERR_TIMEOUT;
    if (v & moe::kStatusBounds) return MOE_ERR_BOUNDS;
    if (v & moe::kStatusRange) return MOE_ERR_RANGE;
    return MOE_OK;
}

moe_status moe_debug_wait_limit(moe_handle* h, uint32_t spins, int32_t withhold_cta) {
    if (!h || spins == 0 || withhold_cta < -1) return MOE_ERR_INVALID_ARG;
    h->spin_limit = spins;
    h->withhold = withhold_cta;
    return MOE_OK;
}

moe_status moe_get_stats(moe_handle* h, moe_stats* out) {
    if (!h || !out) return MOE_ERR_INVALID_ARG;
    moe::Meta m;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(&m, h->meta, sizeof(m), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    out->fixup_tokens = m.n_fixup;
    out->active_experts = m.n_active;
    out->max_group = m.max_count;
    out->launches = h->launches;
    out->cuda_error = h->last_cuda_error;
    return MOE_OK;
}

moe_status moe_profile(moe_handle* h, int32_t enable) {
    if (!h) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    h->prof_on = enable != 0;
    h->ev_kernel.clear();
    for (int i = 0; i < MOE_KERNEL_COUNT; ++i) {
        h->prof_ms[i] = 0.0;
        h->prof_n[i] = 0;
    }
    return MOE_OK;
}

moe_status moe_profile_read(moe_handle* h, double* total_ms, int64_t* launches) {
    if (!h || !total_ms || !launches) return MOE_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    for (size_t j = 0; j < h->ev_kernel.size(); ++j) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, h->ev[2 * j], h->ev[2 * j + 1]) != cudaSuccess) return MOE_ERR_CUDA;
        h->prof_ms[h->ev_kernel[j]] += ms;
        h->prof_n[h->ev_kernel[j]] += 1;
    }
    h->ev_kernel.clear();
    for (int i = 0; i < MOE_KERNEL_COUNT; ++i) {
        total_ms[i] = h->prof_ms[i];
        launches[i] = h->prof_n[i];
    }
    return MOE_OK;
}

const char* moe_kernel_name(int32_t kernel) {
    return (kernel >= 0 && kernel < MOE_KERNEL_COUNT) ? kKernelNames[kernel] : "unknown";
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_OOM: return "out of device memory";
        case MOE_ERR_NOT_LOADED: return "layer weights not loaded";
        case MOE_ERR_TIMEOUT: return "a bounded device-side wait gave up";
        case MOE_ERR_BOUNDS: return "a device-side index was out of range";
        case MOE_ERR_RANGE: return "a value left the range of an internal fp16 operand";
        default: return "unknown status";
    }
}

}  // extern "C"

// kernels.h -- host-side launchers of the routed-MoE kernels (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

struct Meta;

struct RouteArgs {
    const void* x;      // bf16 [T x d]
    int T, d, E, k;
    const void* wr;     // bf16 [E x d]
    const float* bias;  // [E] or null
    const float* wnorm; // [E] ||W_r,e||_2, rounded up
    float* logits;      // scratch [T x E]; [logit_parts][T x E] raw chunk sums (split router GEMM)
    int logit_parts = 1;  // > 1: the reader adds the parts in order, then the bias
    int32_t* ids;       // [T x k]
    float* w;           // [T x k]
    Meta* meta;
    float depth = 0.f;  // logits error bound (see launch_topk); 0: the CUDA-core logits kernel's
};

// Bucketing of the T*k (token, slot) pairs by expert.
struct BucketArgs {
    const int32_t* ids;  // [T x k]
    int T, k, E;
    int32_t* offsets;    // [E + 1] start of each expert's group in `pairs`
    int32_t* pairs;      // [T*k] t*k + r, grouped by expert, ascending t within a group
    int32_t* inv;        // [T*k] position of pair t*k + r in `pairs`
    int32_t* active;     // [E] experts with >= 1 pair, ascending
    Meta* meta;
    uint32_t* status;
    const float* w = nullptr;  // [T x k] routing weights; with wsorted:
    float* wsorted = nullptr;  // [T*k] w of pairs[pos] at pos (or null: not written)
    int32_t* cnt = nullptr;    // scratch [2 x 128 x E] for the multi-CTA variant (large T), or null
    int skip_rank = 0;         // route-tail skip: drop experts whose best rank in the batch is >= this (0: off)
    int e_begin = 0, e_end = 1 << 30;  // experts outside [e_begin, e_end) are dropped (expert parallelism)
    // the expert GEMMs' tile list, built at the end of the single-CTA variant (desc_gu null: not built)
    int4* desc_gu = nullptr;
    int4* desc_dn = nullptr;
    int32_t* tile_counts = nullptr;
    int n_shared = 0, jt_gateup = 0, jt_down = 0;
};
size_t bucket_scratch_words(int E);
int bucket_kernel_count(const BucketArgs& a);  // kernels launch_bucket enqueues: 1, or 3 at large T
bool bucket_builds_tiles(const BucketArgs& a);  // the single-CTA variant, which can build the tile list

// Grouped GEMV/GEMM problem description shared by the expert kernels.
struct ExpertArgs {
    int T, d, f, E, k, n_shared, bits;
    int bits_down = 0;        // code width of the down matrices (0: bits)
    int64_t code_stride = 0;  // code bytes per expert: f*d*(2*bits + bits_down)/8 (0: 3*f*d*bits/8)
    const uint8_t* codes;   // layer codes, expert-major (gate, up, down)
    const uint16_t* scales; // layer scales, same order
    const void* x;          // bf16 [T x d]
    const int32_t* offsets; // [E + 1]
    const int32_t* pairs;   // [T*k]
    const int32_t* active;  // [E]
    const Meta* meta;
    void* h;                // fp16 [(T*k + T*n_shared) x f]
    float* obuf;            // fp32 [(T*k + T*n_shared) x d]
    uint32_t* status;
};

struct CombineArgs {
    int T, d, k, n_shared;
    const float* obuf;
    const int32_t* inv;
    const float* w;         // [T x k]
    void* y;                // bf16 or fp32 [T x d]
    bool out_fp32, accumulate;
};

// Whole layer for up to kDecodeMaxTokens tokens in one persistent kernel.
constexpr int kDecodeMaxTokens = 64;
// Automatic dispatch of moe_forward: the fused kernel up to this many tokens,
// the tensor-core path above (measured crossover on the full-shape layer:
// equal at 16 tokens, the tensor-core path 2.6x faster at 64).
constexpr int kFusedMaxTokens = 16;
struct DecodeLaunch {
    int T, d, f, E, k, n_shared, bits;
    const void* x;
    void* y;
    int out_fp32, accumulate;
    const uint8_t* codes;
    const uint16_t* scales;
    const void* wr;
    const float* bias;
    const float* wnorm;
    float* logits;
    double* logits64;
    int32_t* ids;
    float* w;
    int32_t* offsets;
    int32_t* pairs;
    int32_t* inv;
    int32_t* active;
    Meta* meta;
    uint32_t* status;
    void* h;
    float* obuf;
    int* sync;  // zeroed once; the kernel leaves it zeroed
    int skip_rank = 0;  // route-tail skip: drop experts whose best rank in the batch is >= this (0: off)
    int e_begin = 0, e_end = 1 << 30;  // experts outside [e_begin, e_end) are dropped (expert parallelism)
    // the clustered kernel (launch_decode_pair)
    int bits_down = 0;                // code width of the down matrices (0: bits)
    float* part = nullptr;            // [T x (k + n_shared) x f/128 x d] partial sums (pair_part_floats)
    unsigned long long* ctr = nullptr;  // [kPairCounters] monotonic counters, zero once
    uint32_t spin_limit = 1u << 21;   // polls before a bounded wait gives up
    int withhold = -1;                // test only: this CTA never announces its router rows
    int norm_input = 0;               // the layer reads rmsnorm(x) (bit-identical to launch_rms_normalize)
    const CUtensorMap* down_codes_map = nullptr;   // make_pair_down_maps of the layer
    const CUtensorMap* down_scales_map = nullptr;
};
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t s);
size_t decode_sync_words(int max_tokens, int E, int d);
// Whole layer for up to kPairMaxTokens tokens: 74 clusters of two CTAs, one
// grid-wide hand-off (decode_pair.cu).  Any code widths.
constexpr int kPairMaxTokens = 16;
constexpr int kPairCounters = 8;
bool pair_decode_supported(const DecodeLaunch& L);
size_t pair_part_floats(int max_tokens, int k, int n_shared, int d, int f);
cudaError_t make_pair_down_maps(CUtensorMap* codes_map, CUtensorMap* scales_map, const void* codes,
                                const void* scales, int n_experts_total, int d, int f, int bits, int bits_down);
cudaError_t launch_decode_pair(const DecodeLaunch& L, cudaStream_t s);

cudaError_t launch_router_norms(const void* wr, int E, int d, float* out, cudaStream_t s);
cudaError_t launch_router_logits(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_topk(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_bucket(const BucketArgs& a, cudaStream_t s);
cudaError_t launch_gemv_gateup(const ExpertArgs& a, cudaStream_t s);
cudaError_t launch_gemv_down(const ExpertArgs& a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);
// tcgen05 path (T > kDecodeMaxTokens)
cudaError_t launch_router_gemm(const RouteArgs& a, uint32_t* status, cudaStream_t s);
bool router_gemm_split(int T);
int router_gemm_chunks(int T, int d);
cudaError_t launch_router_reduce(const float* parts, int chunks, int T, int E, const float* bias, float* logits,
                                 cudaStream_t s);
float router_gemm_depth(int d, int chunks);
size_t tile_desc_count(int T, int k, int E, int n_shared, int jt);
cudaError_t launch_build_tiles(const ExpertArgs& a, int4* desc_gu, int4* desc_dn, int32_t* counts, cudaStream_t s);
// TMA descriptors of one expert GEMM: its activation rows (two box heights)
// and the layer's packed codes and scales.
struct GemmMaps {
    CUtensorMap b_small, b_big, codes, scales;
};
cudaError_t make_row_maps(GemmMaps* m, const void* base, int64_t rows, int cols);
cudaError_t make_weight_maps(GemmMaps* m, const void* codes, const void* scales, int n_experts_total, int d, int f,
                             int bits, int bits_down, bool gateup);
cudaError_t launch_gather_f16(const void* x, int T, int d, int k, int n_shared, const int32_t* pairs,
                              const int32_t* n_pairs, void* xg, uint32_t* status, cudaStream_t s);
cudaError_t launch_gemm_gateup(const ExpertArgs& a, const GemmMaps& maps, const int4* desc, const int32_t* counts,
                               cudaStream_t s);
cudaError_t launch_gemm_down(const ExpertArgs& a, const GemmMaps& maps, const float* wsorted, void* o,
                             const int4* desc, const int32_t* counts, cudaStream_t s);
cudaError_t launch_combine_f16(const CombineArgs& a, const void* o, cudaStream_t s);
cudaError_t launch_rms_normalize(const void* x, int T, int d, void* out, float eps, cudaStream_t s);
cudaError_t launch_dequant(const uint8_t* codes, const uint16_t* scales, int N, int K, int bits, float* out,
                           cudaStream_t s);

}  // namespace moe

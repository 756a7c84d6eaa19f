// Prefill (many tokens per expert) path of the MoE layer: tcgen05 tensor-core
// tiles over sign-expanded fp16 weights.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"

namespace gale {

struct PrefillWs {
    int32_t* status;
    int32_t* counts;        // [E]
    int32_t* offsets;       // [E+1]
    int32_t* perm;          // [B*K]
    int32_t* pos_of_pair;   // [B*K]
    void* route_scratch;    // range counts of the many-CTA routing permute
    void* jobs;             // [max_jobs] (expert, first slot, tokens), chunks of 128 slots
    int32_t* n_jobs;        // [1]
    int max_jobs;
    __half* x16;            // [B*K][d_model] rotated x of each pair, permuted order, scaled
    float* x_unscale;       // [B*K] factor that undoes each slot's x16 scale
    float* h_unscale;       // [B*K] the same for h16
    float* h;               // [B*K][d_ff]
    __half* h16;            // [B*K][d_ff] rotated h, scaled per slot
    float* o;               // [B*K][d_model]
    float* scratch;         // [B][d_model]
    size_t bytes;
};

PrefillWs carve_prefill_ws(void* ws, const gale_layer& L, int B, int K);
bool prefill_supported(const gale_layer& L, int B, int K);
int launch_moe_prefill(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                       void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st);

// Gate-weighted combine in fixed k order (+ residual and RMSNorm): o holds one
// row per pair in permuted order, pos_of_pair maps (t, k) to that row.
int launch_moe_combine(const float* o, const int32_t* pos_of_pair, const float* gates, const uint16_t* x, int B,
                       int K, int d_model, void* out, int out_dtype, bool fuse_norm, float eps, float* scratch,
                       cudaStream_t st);

}  // namespace gale

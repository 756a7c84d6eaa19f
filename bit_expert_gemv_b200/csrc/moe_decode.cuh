// Decode path of the MoE layer (small token batches): workspace layout and
// host entry.
#pragma once
#include "common.cuh"

namespace gale {

constexpr int kDecodeMaxPairs = 384;     // B * K handled by the decode kernels
constexpr int kDecodeMaxDModel = 4096;   // shared-memory budget of the stages
constexpr int kDecodeMaxDff = 4096;

struct DecodeWs {
    int32_t* status;
    int32_t* gbar;         // grid-barrier arrivals (in the status block)
    int32_t* comb_cnt;     // [B][d_model/64] experts finished per (token, 64-row block)
    int32_t* tok_cnt;      // [B]            row blocks finished per token (RMSNorm)
    float* ssq;            // [B][d_model/64] partial sums of squares (RMSNorm)
    float* h;              // [pairs][d_ff]   SwiGLU output, permuted slot order
    float* o;              // [pairs][d_model] expert outputs, permuted slot order
    float* v;              // [B][d_model]    x + y before the norm
    size_t bytes;
};

DecodeWs carve_decode_ws(void* ws, const gale_layer& L, int B, int K);
bool decode_supported(const gale_layer& L, int B, int K);
int launch_moe_decode(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                      void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st);

}  // namespace gale

// Decode path of the MoE layer (batches of up to 384 (token, expert) pairs):
// one persistent streaming kernel; workspace layout and host entry.
#pragma once
#include "common.cuh"

namespace gale {

constexpr int kDecodeMaxPairsStream = 384;   // B * K handled by the streaming kernel

struct StreamWs {
    int32_t* status;      // device status word
    int32_t* hcnt;        // [segments][d_ff/1024] finished 16-row tiles of h per 1024-block
    int32_t* comb;        // [B][d_model/64] experts finished per (token, 64-row block)
    int32_t* tokcnt;      // [B] row blocks combined per token (RMSNorm)
    int64_t layer_ints;   // int32 between the hcnt / comb / tokcnt blocks of consecutive layers
    int32_t* xready;      // [layers] tokens whose output of that layer is written
    size_t counter_bytes; // status .. xready, cleared by one memset per call
    float* ssq;           // [B][d_model/64] sums of squares of v per block
    float* h;             // [B*K][d_ff] SwiGLU output of every pair (pair index t*K + k)
    float* o;             // [B*K][d_model] expert output of every pair
    float* v;             // [B][d_model] x + y before the norm
    uint16_t* xbuf;       // [2][B][d_model] bf16 hidden states between layers (chains only)
    size_t bytes;
};

StreamWs carve_stream_ws(void* ws, const gale_layer& L, int B, int K, int n_layers = 1);
bool stream_supported(const gale_layer& L, int B, int K);
// n_layers > 1: a chain of layers (x_{l+1} = bf16 RMSNorm(x_l + MoE_l(x_l))),
// layer l's experts at indices l * layer_experts + e of the expert records
// that start at L.base.
int launch_moe_stream(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                      void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st,
                      int n_layers = 1, int64_t layer_experts = 0, const float* xf = nullptr, int fixed_e = -1);

}  // namespace gale

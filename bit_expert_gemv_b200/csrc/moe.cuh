// Internal structures of the MoE layer (workspace carving and kernel arguments).
#pragma once
#include "common.cuh"

namespace gale {

struct MoeWs {
    int32_t* status;       // device status word (first bytes of the workspace)
    int32_t* counts;       // [E]
    int32_t* offsets;      // [E+1]
    int32_t* perm;         // [B*K] pair indices by (expert, pair)
    int32_t* pos_of_pair;  // [B*K] position of each pair in perm (-1 if dropped)
    int32_t* active;       // [E] experts with pairs, increasing id
    int32_t* n_active;     // [1]
    float* x_rot;          // [B][d_model]
    float* h;              // [B*K][d_ff], permuted pair order
    float* o;              // [B*K][d_model], permuted pair order
    size_t bytes;
};

MoeWs carve_ws(void* ws, const gale_layer& L, int B, int K);

struct GroupArgs {
    const void* base;
    int64_t expert_stride;
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* perm;
    const int32_t* active;
    const int32_t* n_active;
    int K;
    int rows, cols;
    int64_t mat_off_a, mat_off_b;   // byte offsets of the matrices inside a record
    const float* x;
    float* out;
    int chunk;
};

struct CombineArgs {
    const float* o;
    const int32_t* pos_of_pair;
    const float* gates;
    const uint16_t* x;
    int K, d_model;
    void* out;
    int out_dtype;
    int fuse_norm;
    float eps;
    float* scratch;
};

int validate_layer(const gale_layer* L);
bool small_batch(const gale_layer& L, int B, int K);

}  // namespace gale

// Routing permute kernel arguments (shared by gale_route_permute and the MoE layer).
#pragma once
#include "common.cuh"

namespace gale {

struct RouteArgs {
    const int32_t* ids;     // [B][K]
    int B, K, E;
    int32_t* counts;        // [E] or null
    int32_t* offsets;       // [E+1] or null
    int32_t* perm;          // [B*K]
    int32_t* pos_of_pair;   // [B*K] or null: position of pair p in perm
    int32_t* active;        // [E] or null: experts with pairs, increasing id
    int32_t* n_active;      // [1] or null
    int32_t* status;
};

int launch_route_permute(const RouteArgs& a, cudaStream_t st);

// Many-CTA form (three launches); `scratch` holds route_grid_scratch_bytes().
size_t route_grid_scratch_bytes(int B, int K, int E);
int launch_route_permute_grid(const RouteArgs& a, void* scratch, cudaStream_t st);

}  // namespace gale

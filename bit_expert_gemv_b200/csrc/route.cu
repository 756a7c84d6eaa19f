// Routing permute: stable counting sort of the (token, slot) pairs by expert.
//
// One CTA of 1024 threads.  Warp w owns the contiguous pair range
// [w * chunk, (w + 1) * chunk) and walks it 32 pairs at a time, in order:
// pass 1 counts each expert's pairs per warp (match_any groups, the group's
// leader adds); a scan in (expert, warp) order gives every warp the first
// position of each of its experts; pass 2 walks the range again and places
// each pair at that base + its running rank.  The order is the stable one
// (pair order within an expert), independent of scheduling.
#include "common.cuh"
#include "route.cuh"

namespace gale {

namespace {
// Experts of the 32 pairs base .. base + 31 of a warp step (lane = pair), or
// -1 past the range end, out of range, or repeated earlier in the token.  The
// earlier pairs of a token (K <= 16) are in this step or the previous one:
// `prev` holds the previous step's ids (its lane l = pair base - 32 + l).
__device__ __forceinline__ int step_experts(const RouteArgs& a, int base, int end, int id, int prev) {
    const int lane = threadIdx.x & 31, p = base + lane;
    int e = (p < end && id >= 0 && id < a.E) ? id : -1;
    const int t0 = p - p % a.K;
    for (int j = 1; j < a.K; ++j) {   // uniform trip count: every lane shuffles
        const int q = p - j, src = q - base;
        const int vc = __shfl_sync(0xffffffffu, id, src & 31), vp = __shfl_sync(0xffffffffu, prev, src & 31);
        const int v = src >= 0 ? vc : vp;
        if (q >= t0 && v == e) e = -1;
    }
    return e;
}

// Steps a warp walks per batch of id loads.
constexpr int kBlockSteps = 8;

// The ids of the kBlockSteps steps from base0 (lane = pair), -1 past `end`.
__device__ __forceinline__ void load_block(const RouteArgs& a, int base0, int end, int (&idb)[kBlockSteps]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < kBlockSteps; ++j) {
        const int p = base0 + 32 * j + lane;
        idb[j] = p < end ? __ldg(a.ids + p) : -1;
    }
}
}  // namespace

__global__ void __launch_bounds__(1024) route_permute_kernel(RouteArgs a) {
    extern __shared__ int smem[];
    const int E = a.E;
    int* wcnt = smem;                // [32][E]: pairs of expert e in warp w's range, then w's base
    int* scan = wcnt + 32 * E;       // [2 * 1024] scan scratch
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BK = a.B * a.K;
    const int chunk = (BK + 31) / 32;
    const int p0 = warp * chunk, p1 = min(BK, p0 + chunk);

    for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    // pass 1: per-warp counts (and validation); the ids of kBlockSteps steps
    // are loaded at once, so that their latencies overlap
    int prev;
    {
        // the token of the range's first pair may start in the previous range
        const int q = p0 - 32 + lane;
        prev = (q >= 0 && q < BK && p0 < p1) ? a.ids[q] : -1;
    }
    const int prev0 = prev;
    for (int base0 = p0; base0 < p1; base0 += 32 * kBlockSteps) {
        int idb[kBlockSteps];
        load_block(a, base0, p1, idb);
#pragma unroll
        for (int j = 0; j < kBlockSteps; ++j) {
            const int base = base0 + 32 * j;
            if (base >= p1) break;
            const int p = base + lane;
            const int e = step_experts(a, base, p1, idb[j], prev);
            if (p < p1 && e < 0) set_status(a.status, GALE_ERR_ARG);
            prev = idb[j];
            const unsigned grp = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(grp) - 1) wcnt[warp * E + e] += __popc(grp);
            __syncwarp();
        }
    }
    __syncthreads();
    // totals per expert (thread e sums its column in warp order), exclusive
    // scans of the totals and of the non-empty flags
    const int c = tid < E ? [&] {
        int t = 0;
        for (int w = 0; w < 32; ++w) t += wcnt[w * E + tid];
        return t;
    }() : 0;
    const int nz = c > 0;
    int* s1 = scan;
    int* s2 = scan + 1024;
    s1[tid] = c;
    s2[tid] = nz;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int v1 = tid >= off ? s1[tid - off] : 0;
        const int v2 = tid >= off ? s2[tid - off] : 0;
        __syncthreads();
        s1[tid] += v1;
        s2[tid] += v2;
        __syncthreads();
    }
    if (tid < E) {
        const int excl = s1[tid] - c;
        if (a.counts) a.counts[tid] = c;
        if (a.offsets) a.offsets[tid] = excl;
        if (tid == E - 1 && a.offsets) a.offsets[E] = s1[tid];
        if (nz && a.active) a.active[s2[tid] - 1] = tid;
        if (tid == E - 1 && a.n_active) *a.n_active = s2[tid];
        // first position of expert tid in each warp's range
        int run = excl;
        for (int w = 0; w < 32; ++w) {
            const int n = wcnt[w * E + tid];
            wcnt[w * E + tid] = run;
            run += n;
        }
    }
    __syncthreads();
    // pass 2: placement in pair order
    prev = prev0;
    for (int base0 = p0; base0 < p1; base0 += 32 * kBlockSteps) {
        int idb[kBlockSteps];
        load_block(a, base0, p1, idb);
#pragma unroll
        for (int j = 0; j < kBlockSteps; ++j) {
            const int base = base0 + 32 * j;
            if (base >= p1) break;
            const int p = base + lane;
            const int e = step_experts(a, base, p1, idb[j], prev);
            prev = idb[j];
            const unsigned grp = __match_any_sync(0xffffffffu, e);
            if (e >= 0) {
                const int pos = wcnt[warp * E + e] + __popc(grp & ((1u << lane) - 1u));
                a.perm[pos] = p;
                if (a.pos_of_pair) a.pos_of_pair[p] = pos;
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(grp) - 1) wcnt[warp * E + e] += __popc(grp);
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------------------
// Many-CTA form for large batches (the one-CTA kernel above runs on one SM).
// Warp range r holds the kGridWarpPairs pairs from r * kGridWarpPairs, walked
// in kBlockSteps steps with one batch of id loads.  route_count_kernel writes
// every range's per-expert counts [rows][E]; route_scan_kernel turns them, in
// (expert, range) order, into each range's first position per expert
// relative to the expert's offset, and writes counts and offsets;
// route_place_kernel places every pair at its range's base + its running
// rank.  The order is the same stable one.
constexpr int kGridWarps = 8;                    // warps (ranges) per block
constexpr int kGridWarpPairs = 32 * kBlockSteps;

namespace {
__host__ __device__ inline int64_t grid_rows(int64_t BK) { return (BK + kGridWarpPairs - 1) / kGridWarpPairs; }
}  // namespace

size_t route_grid_scratch_bytes(int B, int K, int E) {
    return size_t(grid_rows(int64_t(B) * K)) * size_t(E) * 4;
}

// The validated experts of one warp range, handed to `f(p, e, grp)` step by
// step (e < 0: dropped or past the end; grp: the lanes of the step with the
// same e).
template <typename F>
__device__ __forceinline__ void walk_range(const RouteArgs& a, int p0, int p1, F f) {
    const int lane = threadIdx.x & 31, BK = a.B * a.K;
    int prev;
    {
        const int q = p0 - 32 + lane;
        prev = (q >= 0 && q < BK) ? __ldg(a.ids + q) : -1;
    }
    int idb[kBlockSteps];
    load_block(a, p0, p1, idb);
#pragma unroll
    for (int j = 0; j < kBlockSteps; ++j) {
        const int base = p0 + 32 * j;
        if (base >= p1) break;
        const int e = step_experts(a, base, p1, idb[j], prev);
        prev = idb[j];
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        f(base + lane, e, grp);
    }
}

__global__ void __launch_bounds__(kGridWarps * 32) route_count_kernel(RouteArgs a, int32_t* __restrict__ cnt) {
    extern __shared__ int wc[];   // [kGridWarps][E]
    const int E = a.E, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int BK = a.B * a.K;
    const int64_t rows = grid_rows(BK);
    for (int i = threadIdx.x; i < kGridWarps * E; i += blockDim.x) wc[i] = 0;
    __syncthreads();
    const int64_t r = int64_t(blockIdx.x) * kGridWarps + warp;
    if (r < rows) {
        const int p0 = int(r) * kGridWarpPairs, p1 = min(BK, p0 + kGridWarpPairs);
        walk_range(a, p0, p1, [&](int p, int e, unsigned grp) {
            if (p < p1 && e < 0) set_status(a.status, GALE_ERR_ARG);
            if (e >= 0 && lane == __ffs(grp) - 1) wc[warp * E + e] += __popc(grp);
            __syncwarp();
        });
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kGridWarps * E; i += blockDim.x) {
        const int w = i / E;
        const int64_t rw = int64_t(blockIdx.x) * kGridWarps + w;
        if (rw < rows) cnt[rw * E + (i - w * E)] = wc[i];
    }
}

// One CTA: thread e runs down expert e's column of range counts.
__global__ void __launch_bounds__(1024) route_scan_kernel(RouteArgs a, int32_t* __restrict__ cnt) {
    __shared__ int s1[1024];
    const int E = a.E, tid = threadIdx.x;
    const int64_t rows = grid_rows(int64_t(a.B) * a.K);
    int run = 0;
    if (tid < E) {
#pragma unroll 8
        for (int64_t r = 0; r < rows; ++r) {
            const int v = cnt[r * E + tid];
            cnt[r * E + tid] = run;
            run += v;
        }
    }
    s1[tid] = tid < E ? run : 0;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int v = tid >= off ? s1[tid - off] : 0;
        __syncthreads();
        s1[tid] += v;
        __syncthreads();
    }
    if (tid < E) {
        if (a.counts) a.counts[tid] = run;
        a.offsets[tid] = s1[tid] - run;
        if (tid == E - 1) a.offsets[E] = s1[tid];
    }
}

__global__ void __launch_bounds__(kGridWarps * 32) route_place_kernel(RouteArgs a, const int32_t* __restrict__ base) {
    extern __shared__ int wb[];   // [kGridWarps][E]: next position of each expert in each range
    const int E = a.E, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int BK = a.B * a.K;
    const int64_t rows = grid_rows(BK);
    for (int i = threadIdx.x; i < kGridWarps * E; i += blockDim.x) {
        const int w = i / E, e = i - w * E;
        const int64_t rw = int64_t(blockIdx.x) * kGridWarps + w;
        wb[i] = rw < rows ? base[rw * E + e] + a.offsets[e] : 0;
    }
    __syncthreads();
    const int64_t r = int64_t(blockIdx.x) * kGridWarps + warp;
    if (r >= rows) return;
    const int p0 = int(r) * kGridWarpPairs, p1 = min(BK, p0 + kGridWarpPairs);
    walk_range(a, p0, p1, [&](int p, int e, unsigned grp) {
        if (e >= 0) {
            const int pos = wb[warp * E + e] + __popc(grp & ((1u << lane) - 1u));
            a.perm[pos] = p;
            if (a.pos_of_pair) a.pos_of_pair[p] = pos;
        }
        __syncwarp();
        if (e >= 0 && lane == __ffs(grp) - 1) wb[warp * E + e] += __popc(grp);
        __syncwarp();
    });
}

int launch_route_permute_grid(const RouteArgs& a, void* scratch, cudaStream_t st) {
    const int64_t BK = int64_t(a.B) * a.K;
    if (BK == 0) return launch_route_permute(a, st);
    if (!a.offsets) return GALE_ERR_ARG;
    int32_t* cnt = static_cast<int32_t*>(scratch);
    const unsigned blocks = unsigned((grid_rows(BK) + kGridWarps - 1) / kGridWarps);
    const size_t smem = size_t(kGridWarps) * a.E * sizeof(int);
    route_count_kernel<<<blocks, kGridWarps * 32, smem, st>>>(a, cnt);
    GALE_LAUNCH_CHECK();
    route_scan_kernel<<<1, 1024, 0, st>>>(a, cnt);
    GALE_LAUNCH_CHECK();
    route_place_kernel<<<blocks, kGridWarps * 32, smem, st>>>(a, cnt);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

int launch_route_permute(const RouteArgs& a, cudaStream_t st) {
    const size_t smem = (size_t(32) * a.E + 2048) * sizeof(int);
    if (smem > 48 * 1024)
        GALE_CUDA_TRY(cudaFuncSetAttribute(route_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem)));
    route_permute_kernel<<<1, 1024, smem, st>>>(a);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

}  // namespace gale

extern "C" int gale_route_permute(const int32_t* ids, int B, int K, int E, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* status, void* stream) {
    if (B < 0 || K < 1 || K > 16 || E < 1 || E > 1024 || !counts || !offsets || !status)
        return GALE_ERR_ARG;
    if (B > 0 && (!ids || !perm)) return GALE_ERR_ARG;
    if (!gale::aligned(ids, 4) || !gale::aligned(counts, 4) || !gale::aligned(offsets, 4) ||
        !gale::aligned(perm, 4) || !gale::aligned(status, 4))
        return GALE_ERR_ALIGN;
    if (int64_t(B) * K > (1 << 30)) return GALE_ERR_UNSUPPORTED;
    cudaStream_t st = gale::as_stream(stream);
    GALE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    gale::RouteArgs a{};
    a.ids = ids;
    a.B = B;
    a.K = K;
    a.E = E;
    a.counts = counts;
    a.offsets = offsets;
    a.perm = perm;
    a.status = status;
    return gale::launch_route_permute(a, st);
}

extern "C" size_t gale_route_permute_scratch_bytes(int B, int K, int E) {
    if (B < 0 || K < 1 || K > 16 || E < 1 || E > 1024) return 0;
    return gale::route_grid_scratch_bytes(B, K, E);
}

extern "C" int gale_route_permute_grid(const int32_t* ids, int B, int K, int E, int32_t* counts,
                                       int32_t* offsets, int32_t* perm, int32_t* status, void* scratch,
                                       size_t scratch_bytes, void* stream) {
    if (B < 0 || K < 1 || K > 16 || E < 1 || E > 1024 || !counts || !offsets || !status)
        return GALE_ERR_ARG;
    if (B > 0 && (!ids || !perm || !scratch)) return GALE_ERR_ARG;
    if (!gale::aligned(ids, 4) || !gale::aligned(counts, 4) || !gale::aligned(offsets, 4) ||
        !gale::aligned(perm, 4) || !gale::aligned(status, 4) || !gale::aligned(scratch, 4))
        return GALE_ERR_ALIGN;
    if (int64_t(B) * K > (1 << 30)) return GALE_ERR_UNSUPPORTED;
    if (scratch_bytes < gale::route_grid_scratch_bytes(B, K, E)) return GALE_ERR_WORKSPACE;
    cudaStream_t st = gale::as_stream(stream);
    GALE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    gale::RouteArgs a{};
    a.ids = ids;
    a.B = B;
    a.K = K;
    a.E = E;
    a.counts = counts;
    a.offsets = offsets;
    a.perm = perm;
    a.status = status;
    return gale::launch_route_permute_grid(a, scratch, st);
}

// ----------------------------------------------------------------------------
// router: top-K experts by logit and their softmax gates
// ----------------------------------------------------------------------------

namespace gale {
namespace {

// One warp per token.  Lane l holds the logits of experts l, l + 32, ...;
// each of the K rounds takes the warp-wide (largest logit, lowest index) not
// yet taken, and lane k keeps round k's pick.  NaN logits count as -inf.
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int B, int E, int K,
                                                         int32_t* __restrict__ ids, float* __restrict__ gates) {
    const int lane = threadIdx.x & 31;
    const int t = int((blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5);
    if (t >= B) return;
    const float* l = logits + int64_t(t) * E;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int e = lane + 32 * j;
        const float x = e < E ? __ldg(l + e) : -INFINITY;
        v[j] = x == x ? x : -INFINITY;
    }
    uint32_t taken = 0u;
    float mine = -INFINITY;
    int mine_id = -1;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int e = lane + 32 * j;
            if (e < E && !((taken >> j) & 1u) && (v[j] > bv || (v[j] == bv && e < bi))) {
                bv = v[j];
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == k) {
            mine = bv;
            mine_id = bi;
        }
    }
    // softmax over the K picks (lane 0 holds the largest)
    const float m = __shfl_sync(0xffffffffu, mine, 0);
    const float ex = lane < K ? expf(mine - m) : 0.f;
    const float sum = warp_sum(ex);
    if (lane < K) {
        ids[int64_t(t) * K + lane] = mine_id;
        gates[int64_t(t) * K + lane] = ex / sum;
    }
}

}  // namespace
}  // namespace gale

extern "C" int gale_route_topk(const float* logits, int B, int E, int K, int32_t* ids, float* gates, void* stream) {
    if (B < 0 || E < 1 || E > 1024 || K < 1 || K > 16 || K > E) return GALE_ERR_ARG;
    if (B == 0) return GALE_OK;
    if (!logits || !ids || !gates) return GALE_ERR_ARG;
    if (!gale::aligned(logits, 4) || !gale::aligned(ids, 4) || !gale::aligned(gates, 4)) return GALE_ERR_ALIGN;
    const int64_t threads = int64_t(B) * 32;
    gale::route_topk_kernel<<<unsigned((threads + 255) / 256), 256, 0, gale::as_stream(stream)>>>(logits, B, E, K, ids,
                                                                                                 gates);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

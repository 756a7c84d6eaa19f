// Routing permute: stable counting sort of the (token, slot) pairs by expert.
//
// One CTA of 1024 threads.  Pairs are placed in rounds of 1024 in pair order;
// within a round a pair's rank among equal experts is its rank inside its
// warp (match_any) plus the counts of that expert in the earlier warps, so the
// result is the stable order, independent of scheduling.
#include "common.cuh"
#include "route.cuh"

namespace gale {

__global__ void __launch_bounds__(1024) route_permute_kernel(RouteArgs a) {
    extern __shared__ int smem[];
    const int E = a.E;
    int* cnt = smem;                 // [E]
    int* cur = cnt + E;              // [E]
    int* wcnt = cur + E;             // [32][E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BK = a.B * a.K;

    for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    // histogram + validation (out-of-range or repeated within a token)
    for (int p = tid; p < BK; p += blockDim.x) {
        int e = a.ids[p];
        bool ok = e >= 0 && e < E;
        if (ok) {
            int t0 = p - p % a.K;
            for (int j = t0; j < p; ++j)
                if (a.ids[j] == e) ok = false;
        }
        if (ok) atomicAdd(&cnt[e], 1);
        else set_status(a.status, GALE_ERR_ARG);
    }
    __syncthreads();
    // exclusive scan of counts (E <= 1024: one element per thread), plus the
    // list of experts with at least one pair, in increasing id order
    {
        int c = tid < E ? cnt[tid] : 0;
        int nz = c > 0;
        // block-wide inclusive scans through shared memory (two arrays in wcnt)
        int* s1 = wcnt;
        int* s2 = wcnt + 1024;
        s1[tid] = c;
        s2[tid] = nz;
        __syncthreads();
        for (int off = 1; off < 1024; off <<= 1) {
            int v1 = tid >= off ? s1[tid - off] : 0;
            int v2 = tid >= off ? s2[tid - off] : 0;
            __syncthreads();
            s1[tid] += v1;
            s2[tid] += v2;
            __syncthreads();
        }
        if (tid < E) {
            int excl = s1[tid] - c;
            cur[tid] = excl;
            if (a.counts) a.counts[tid] = c;
            if (a.offsets) a.offsets[tid] = excl;
            if (tid == E - 1 && a.offsets) a.offsets[E] = s1[tid];
            if (nz && a.active) a.active[s2[tid] - 1] = tid;
            if (tid == E - 1 && a.n_active) *a.n_active = s2[tid];
        }
        __syncthreads();
    }
    // stable placement, 1024 pairs per round
    for (int base = 0; base < BK; base += blockDim.x) {
        for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
        __syncthreads();
        const int p = base + tid;
        int e = -1;
        if (p < BK) {
            e = a.ids[p];
            bool ok = e >= 0 && e < E;
            if (ok) {
                int t0 = p - p % a.K;
                for (int j = t0; j < p; ++j)
                    if (a.ids[j] == e) ok = false;
            }
            if (!ok) e = -1;
        }
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(grp & ((1u << lane) - 1u));
        if (e >= 0 && rank == 0) wcnt[warp * E + e] = __popc(grp);
        __syncthreads();
        if (e >= 0) {
            int pos = cur[e] + rank;
            for (int w = 0; w < warp; ++w) pos += wcnt[w * E + e];
            a.perm[pos] = p;
            if (a.pos_of_pair) a.pos_of_pair[p] = pos;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += blockDim.x) {
            int s = 0;
            for (int w = 0; w < 32; ++w) s += wcnt[w * E + ee];
            cur[ee] += s;
        }
        __syncthreads();
    }
}

int launch_route_permute(const RouteArgs& a, cudaStream_t st) {
    size_t smem = size_t(34) * a.E * sizeof(int);
    if (smem < 2048 * sizeof(int) + 2 * a.E * sizeof(int)) smem = 2048 * sizeof(int) + 2 * a.E * sizeof(int);
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

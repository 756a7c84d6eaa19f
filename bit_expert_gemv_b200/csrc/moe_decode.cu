// Decode path of gale_moe_forward: two streaming kernels chained by
// programmatic dependent launch.
//
//   w13 : jobs (expert, token pair, row block) of w1 and w3.  Each CTA rotates
//         (FWHT-1024, warp shuffles) the tokens its jobs need and keeps their
//         fixed-point int8 digits in shared memory; a producer warp streams the packed
//         tiles with TMA while 8 consumer warps run the tensor-core tile
//         routine split by (matrix, 1024-column chunk); SwiGLU; h to global.
//   w2  : jobs (expert, token pair, row block) of w2.  After waiting for w13,
//         each CTA rotates the h rows its jobs need; expert outputs go to
//         global, and the last expert to finish a (token, row block) sums the
//         K contributions in fixed k order with the gates (deterministic, no
//         float atomics), optionally adds the residual; the last row block of
//         a token applies RMSNorm.
// Both kernels compute the routing themselves from the ids, and w2's producer
// starts streaming weights before waiting for w13.
#include "common.cuh"
#include "fwht.cuh"
#include "moe.cuh"
#include "moe_decode.cuh"
#include "mma_tile.cuh"

namespace gale {

namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;

struct DecArgs {
    const char* base;
    int64_t stride;
    int E, d_model, d_ff, B, K;
    int64_t off_w1, off_w3, off_w2;
    const uint16_t* x;
    const int32_t* ids;
    const float* gates;
    void* out;
    int out_dtype, fuse_norm;
    float eps;
    DecodeWs ws;
};

// ----------------------------------------------------------------------------
// routing inside a CTA (B*K <= kDecodeMaxPairs, E <= 1024)
// ----------------------------------------------------------------------------

struct RouteSmem {
    int cnt[1024];                    // per expert: valid pairs
    int off[1024];                    // per expert: first slot
    int aidx[1024];                   // per expert: index among the active experts
    int pe[kDecodeMaxPairs];          // expert of each pair, -1 if dropped
    int active[kDecodeMaxPairs];      // active expert ids, increasing
    int first_slot[kDecodeMaxPairs];
    int n_tok[kDecodeMaxPairs];
    int job_start[kDecodeMaxPairs + 1];
    int grp_base[kDecodeMaxPairs + 1];
    int slot_tok[kDecodeMaxPairs];    // token of each slot
    int pos_of_pair[kDecodeMaxPairs]; // slot of each pair (-1: dropped)
    int tok_valid[kDecodeMaxPairs];   // valid pairs per token
    int scan_tmp[32];
    int n_active, n_jobs, n_groups, bad;
};

// Block-wide exclusive scan of a[0..n) (n <= 4 * blockDim.x) in place; returns the total.
__device__ int block_exclusive_scan(int* a, int n, int* tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int i0 = tid * per;
    int loc[4] = {0, 0, 0, 0};
    int s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < per && i0 + j < n) loc[j] = a[i0 + j];
        s += loc[j];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) {
            const int v = tmp[w];
            tmp[w] = run;
            run += v;
        }
        tmp[31] = run;
    }
    __syncthreads();
    int excl = tmp[warp] + incl - s;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j < per && i0 + j < n) a[i0 + j] = excl;
        excl += loc[j];
    }
    const int total = tmp[31];
    __syncthreads();
    return total;
}

// Small batches (B*K <= 32): one warp computes the same tables with
// shuffles, lane p handling pair p.
__device__ void build_route_small(const DecArgs& A, RouteSmem& R, int tiles) {
    const int lane = threadIdx.x & 31;
    const int BK = A.B * A.K, E = A.E;
    const bool in = lane < BK;
    int e = in ? A.ids[lane] : -1;
    bool ok = in && e >= 0 && e < E;
    if (in) {
        const int t0 = lane - lane % A.K;
        for (int j = t0; ok && j < lane; ++j) ok = A.ids[j] != e;
    }
    if (!ok) e = -1;
    const unsigned bad = __ballot_sync(0xffffffffu, in && !ok);
    // slot = rank of (e, p) among the valid pairs; first pair of each expert
    int rank = 0, same = 0, first_before = 0;
    bool first = ok;
    for (int q = 0; q < 32; ++q) {
        const int eq = __shfl_sync(0xffffffffu, e, q);
        if (eq < 0) continue;
        rank += (eq < e) || (eq == e && q < lane);
        same += (eq == e);
        if (eq == e && q < lane) first = false;
    }
    // active index: number of distinct valid experts below e
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    for (int q = 0; q < 32; ++q) {
        const int eq = __shfl_sync(0xffffffffu, e, q);
        if ((firsts >> q) & 1) first_before += (eq < e);
    }
    const int n_active = __popc(firsts);
    if (in) R.pos_of_pair[lane] = ok ? rank : -1;
    if (ok) R.slot_tok[rank] = lane / A.K;
    int groups = 0;
    if (first) {
        R.active[first_before] = e;
        R.first_slot[first_before] = rank;
        R.n_tok[first_before] = same;
        groups = (same + 1) / 2;
    }
    // prefix sums of groups and jobs over the active experts (indexed by first_before)
    int g_a = 0;
    for (int q = 0; q < 32; ++q) {
        const int gq = __shfl_sync(0xffffffffu, groups, q);
        const int aq = __shfl_sync(0xffffffffu, first_before, q);
        if (((firsts >> q) & 1) && aq < first_before) g_a += gq;
    }
    if (first) {
        R.grp_base[first_before] = g_a;
        R.job_start[first_before] = g_a * tiles;
    }
    int n_groups = groups;
    for (int o = 16; o > 0; o >>= 1) n_groups += __shfl_xor_sync(0xffffffffu, n_groups, o);
    {
        int v = 0;   // valid pairs of token `lane`
        for (int k = 0; k < A.K; ++k) {
            const int src = lane * A.K + k;
            const int okq = __shfl_sync(0xffffffffu, ok ? 1 : 0, src & 31);
            if (src < BK) v += okq;
        }
        if (lane < A.B) R.tok_valid[lane] = v;
    }
    if (lane == 0) {
        R.n_active = n_active;
        R.n_groups = n_groups;
        R.n_jobs = n_groups * tiles;
        R.job_start[n_active] = n_groups * tiles;
        R.grp_base[n_active] = n_groups;
        R.bad = bad != 0u;
    }
}

// Stable grouping of the (token, slot) pairs by expert, and the job table:
// every active expert has ceil(n_tok / 2) token groups of at most two tokens,
// and every group has `tiles` row-tile jobs.
__device__ void build_route(const DecArgs& A, RouteSmem& R, int tiles) {
    const int tid = threadIdx.x;
    const int BK = A.B * A.K, E = A.E;
    if (BK <= 32) {
        if (tid < 32) build_route_small(A, R, tiles);
        __syncthreads();
        return;
    }
    for (int e = tid; e < E; e += blockDim.x) R.cnt[e] = 0;
    for (int t = tid; t < A.B; t += blockDim.x) R.tok_valid[t] = 0;
    if (tid == 0) R.bad = 0;
    __syncthreads();
    for (int p = tid; p < BK; p += blockDim.x) {
        const int e = A.ids[p];
        bool ok = e >= 0 && e < E;
        const int t0 = p - p % A.K;
        for (int j = t0; ok && j < p; ++j) ok = A.ids[j] != e;
        R.pe[p] = ok ? e : -1;
        if (ok) {
            atomicAdd(&R.cnt[e], 1);
            atomicAdd(&R.tok_valid[p / A.K], 1);
        } else {
            R.bad = 1;
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        R.off[e] = R.cnt[e];
        R.aidx[e] = R.cnt[e] > 0;
    }
    __syncthreads();
    block_exclusive_scan(R.off, E, R.scan_tmp);
    const int n_active = block_exclusive_scan(R.aidx, E, R.scan_tmp);
    for (int e = tid; e < E; e += blockDim.x) {
        if (R.cnt[e] > 0) {
            const int a = R.aidx[e];
            R.active[a] = e;
            R.first_slot[a] = R.off[e];
            R.n_tok[a] = R.cnt[e];
            const int groups = (R.cnt[e] + 1) / 2;
            R.grp_base[a] = groups;
            R.job_start[a] = groups * tiles;
        }
    }
    for (int p = tid; p < BK; p += blockDim.x) {
        const int e = R.pe[p];
        int slot = -1;
        if (e >= 0) {
            int rank = 0;
            for (int q = 0; q < p; ++q) rank += (R.pe[q] == e);
            slot = R.off[e] + rank;
            R.slot_tok[slot] = p / A.K;
        }
        R.pos_of_pair[p] = slot;
    }
    __syncthreads();
    const int n_groups = block_exclusive_scan(R.grp_base, n_active, R.scan_tmp);
    const int n_jobs = block_exclusive_scan(R.job_start, n_active, R.scan_tmp);
    if (tid == 0) {
        R.n_active = n_active;
        R.n_jobs = n_jobs;
        R.n_groups = n_groups;
        R.job_start[n_active] = n_jobs;
        R.grp_base[n_active] = n_groups;
    }
    __syncthreads();
}

struct Job {
    int e, a, group, tile, slot0, slot1;
};

__device__ __forceinline__ Job decode_job(const RouteSmem& R, int j, int tiles) {
    int lo = 0, hi = R.n_active - 1;   // last a with job_start[a] <= j
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (R.job_start[mid] <= j) lo = mid;
        else hi = mid - 1;
    }
    Job J;
    J.a = lo;
    J.e = R.active[lo];
    const int rem = j - R.job_start[lo];
    const int gi = rem / tiles;
    J.tile = rem - gi * tiles;
    J.group = R.grp_base[lo] + gi;
    J.slot0 = R.first_slot[lo] + 2 * gi;
    J.slot1 = (2 * gi + 1 < R.n_tok[lo]) ? J.slot0 + 1 : -1;
    return J;
}

// ----------------------------------------------------------------------------
// streaming kernels: one producer warp (TMA ring) + 8 consumer warps that
// split every job by (row tile, matrix, 1024-column chunk)
// ----------------------------------------------------------------------------

constexpr int kCapMax = 8;

struct Shape {
    int rows, cols;      // rows and columns of the streamed matrices
    int n_mat;           // 2 (w1, w3) or 1 (w2)
    int n_chunk;         // cols / 1024
    int r_tiles;         // 16-row tiles per job: 8 / (n_mat * n_chunk)
    int job_rows;        // 16 * r_tiles
    int row_blocks;      // jobs per token group: ceil(rows / job_rows)
    int tile_bytes;      // stage_layout(cols).bytes
    int stage_bytes;     // r_tiles * n_mat * tile_bytes
    int n_stages;        // ring depth
    int tok_cap;         // rotated vectors cached in shared memory
    int tok_bytes;       // pieces + 128-block sums of one cached vector
};

__host__ __device__ inline Shape make_shape(int rows, int cols, int n_mat) {
    Shape s{};
    s.rows = rows;
    s.cols = cols;
    s.n_mat = n_mat;
    s.n_chunk = cols / 1024;
    s.r_tiles = kDecWarps / (n_mat * s.n_chunk);
    s.job_rows = 16 * s.r_tiles;
    s.row_blocks = (rows + s.job_rows - 1) / s.job_rows;
    s.tile_bytes = stage_layout(cols).bytes;
    s.stage_bytes = s.r_tiles * n_mat * s.tile_bytes;
    s.tok_bytes = int(align_up(cols * kPieces + (cols / 128) * 4 + cols * 2, 16));
    return s;
}

struct CacheSmem {
    int key[kCapMax];
    float sigma[kCapMax];
    int stamp[kCapMax];
    int plan_slot[2], plan_key[2], n_plan, clock;
    float red[kDecWarps];
    int cres[2];       // cache indices of the current job's vectors
    int flag[8];       // combine / RMSNorm last-arriver flags
    float wsum[kDecWarps];
    float inv;
};

struct StreamSmem {
    int stages, cache, route, partials, scratch, bars, misc, bytes;
};

__host__ __device__ inline StreamSmem stream_smem(const Shape& sh) {
    StreamSmem s;
    int o = 0;
    s.stages = o;
    o += sh.n_stages * sh.stage_bytes;
    s.cache = o;
    o += sh.tok_cap * sh.tok_bytes;
    s.route = o;
    o += int(align_up(sizeof(RouteSmem), 16));
    s.partials = o;
    o += 2 * kDecWarps * 16 * 2 * 4;
    s.scratch = o;
    o += kDecWarps * kWarpScratchFloats * 4;
    s.bars = o;
    o += 2 * sh.n_stages * 8;
    s.misc = o;
    o += int(align_up(sizeof(CacheSmem), 16));
    s.bytes = int(align_up(o, 1024)) + 1024;
    return s;
}

// the 8 consumer warps must split a job evenly
__host__ __device__ inline bool shape_ok(int cols, int n_mat) {
    const int units = n_mat * (cols / 1024);
    return cols % 1024 == 0 && units >= 1 && units <= kDecWarps && kDecWarps % units == 0;
}

// Make sure the rotated vectors `key0`, `key1` (tokens for w13, slots for w2;
// -1 = none) are in the shared-memory cache; returns their cache indices.
// All 256 consumer threads call it.  A missing vector is loaded (bf16 x or
// fp32 h), rotated by FWHT-1024 (one warp per 1024-block), and turned into
// pieces and 128-block sums; the least recently used entry is replaced.
template <bool W13>
__device__ void ensure_cached(const DecArgs& A, const Shape& sh, uint8_t* cache, CacheSmem& M, int key0, int key1,
                              int& c0, int& c1) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = sh.cols, nblk = C / 1024;
    if (tid == 0) {
        const int keys[2] = {key0, key1};
        int found[2] = {-1, -1};
        M.n_plan = 0;
        for (int e = 0; e < 2; ++e) {
            if (keys[e] < 0) continue;
            for (int q = 0; q < sh.tok_cap; ++q)
                if (M.key[q] == keys[e]) found[e] = q;
        }
        for (int e = 0; e < 2; ++e) {
            if (keys[e] < 0 || found[e] >= 0) continue;
            int victim = -1, best = 0x7fffffff;
            for (int q = 0; q < sh.tok_cap; ++q) {
                if (q == found[0] || q == found[1]) continue;
                if (M.stamp[q] < best) {
                    best = M.stamp[q];
                    victim = q;
                }
            }
            found[e] = victim;
            M.key[victim] = keys[e];
            M.plan_slot[M.n_plan] = victim;
            M.plan_key[M.n_plan] = keys[e];
            ++M.n_plan;
        }
        for (int e = 0; e < 2; ++e)
            if (found[e] >= 0) M.stamp[found[e]] = ++M.clock;
        M.cres[0] = found[0];
        M.cres[1] = found[1];
    }
    named_bar_sync(1, kDecThreads);
    c0 = M.cres[0];
    c1 = M.cres[1];
    const int n_plan = M.n_plan;
    if (n_plan == 0) return;
    // warps [e * nblk, (e + 1) * nblk) rotate entry e, one 1024-block each
    const int e = warp / nblk, blk = warp % nblk;
    float v[32];
    const bool act = e < n_plan;
    if (act) {
        const int key = M.plan_key[e];
        if (W13) {
            const uint16_t* src = A.x + int64_t(key) * C + blk * 1024;
#pragma unroll
            for (int r = 0; r < 32; ++r) v[r] = bf16_to_f32(src[piece_elem(lane, r)]);
        } else {
            const float* src = A.ws.h + int64_t(key) * C + blk * 1024;
#pragma unroll
            for (int r = 0; r < 32; ++r) v[r] = __ldcg(src + piece_elem(lane, r));
        }
        fwht1024_warp(v, lane);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= (1.0f / 32.0f);
        const float m = block_absmax(v);
        if (lane == 0) M.red[warp] = m;
    }
    named_bar_sync(1, kDecThreads);
    if (act) {
        float m = 0.f;
        for (int w = e * nblk; w < (e + 1) * nblk; ++w) m = fmaxf(m, M.red[w]);
        const float S = fixed_scale(m);
        uint8_t* dst = cache + M.plan_slot[e] * sh.tok_bytes;
        pieces_from_regs(v, S, dst + blk * 8 * kPieceBlockBytes,
                         reinterpret_cast<float*>(dst + C * kPieces) + blk * 8,
                         reinterpret_cast<__half*>(dst + C * kPieces + (C / 128) * 4) + blk * 1024);
        if (blk == 0 && lane == 0) M.sigma[M.plan_slot[e]] = 1.0f / S;
    }
    named_bar_sync(1, kDecThreads);
}

template <bool W13>
__global__ void __launch_bounds__(kDecThreads + 32, 1) moe_stream_kernel(
    const __grid_constant__ CUtensorMap sa, const __grid_constant__ CUtensorMap ba,
    const __grid_constant__ CUtensorMap sb, const __grid_constant__ CUtensorMap bb, DecArgs A, Shape sh) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    const StreamSmem S = stream_smem(sh);
    RouteSmem& R = *reinterpret_cast<RouteSmem*>(smem + S.route);
    CacheSmem& M = *reinterpret_cast<CacheSmem*>(smem + S.misc);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* empty = full + sh.n_stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < sh.n_stages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, kDecWarps);
        }
        fence_mbar_init();
        for (int q = 0; q < kCapMax; ++q) {
            M.key[q] = -1;
            M.stamp[q] = 0;
        }
        M.clock = 0;
    }
    build_route(A, R, sh.row_blocks);   // contains __syncthreads
    // contiguous job range of this CTA
    const int J = R.n_jobs, G = gridDim.x;
    const int j0 = int((int64_t(J) * blockIdx.x) / G), j1 = int((int64_t(J) * (blockIdx.x + 1)) / G);
    const int n_my = j1 - j0;
    const int64_t off_a = W13 ? A.off_w1 : A.off_w2;
    const int64_t off_b = W13 ? A.off_w3 : A.off_w2;
    auto view = [&](int e, int mat) {
        return make_view(A.base + int64_t(e) * A.stride + (mat ? off_b : off_a), sh.rows, sh.cols);
    };

    if (warp == kDecWarps) {
        // ---------------- producer: weights only, no dependency on earlier kernels.
        // Lane 0 arms the stage's barrier with the job's byte count, then every
        // lane issues the copies of one (row tile, matrix) of the job.
        const int n_tiles = sh.r_tiles * sh.n_mat;
        for (int i = 0; i < n_my; ++i) {
            const int s = i % sh.n_stages;
            int ok_wait = 1;
            if (lane == 0 && i >= sh.n_stages) ok_wait = mbar_wait(empty + s, ((i / sh.n_stages) - 1) & 1);
            ok_wait = __shfl_sync(0xffffffffu, ok_wait, 0);
            if (!ok_wait) {
                if (lane == 0) set_status(A.ws.status, GALE_ERR_TIMEOUT);
                break;
            }
            const Job Jb = decode_job(R, j0 + i, sh.row_blocks);
            const int tr = lane / sh.n_mat, mt = lane % sh.n_mat;
            const int r0 = Jb.tile * sh.job_rows + tr * 16;
            const bool mine = lane < n_tiles && r0 < sh.rows;
            uint32_t tx = 0;
            MatView mv{};
            if (mine) {
                mv = view(Jb.e, mt);
                tx = tile_tx_bytes(mv, r0);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, o);
            if (lane == 0) mbar_arrive_expect_tx(full + s, tx);
            __syncwarp();
            if (mine)
                issue_tile_copies(smem + S.stages + s * sh.stage_bytes + (tr * sh.n_mat + mt) * sh.tile_bytes,
                                  full + s, mt ? &sb : &sa, mt ? &bb : &ba, mv, Jb.e, r0);
        }
        return;
    }

    // ---------------- consumers
    const int tid = threadIdx.x;   // 0..255
    const int d = A.d_model;
    const int comb_blocks = (d + 63) / 64;   // w2 row blocks (64 rows)
    if (W13) {
        // w2's counters start at zero; w2 touches them only after waiting for this grid
        if (blockIdx.x == 0) {
            for (int i = tid; i < A.B * comb_blocks; i += kDecThreads) A.ws.comb_cnt[i] = 0;
            for (int i = tid; i < A.B; i += kDecThreads) A.ws.tok_cnt[i] = 0;
            if (tid == 0 && R.bad) set_status(A.ws.status, GALE_ERR_ARG);
        }
        pdl_launch_dependents();
    } else {
        pdl_wait();   // h of every expert and the zeroed counters
    }
    uint8_t* cache = smem + S.cache;
    const int tr = warp / (sh.n_mat * sh.n_chunk);
    const int mat = (warp / sh.n_chunk) % sh.n_mat;
    const int ch = warp % sh.n_chunk;
    float* scratch = reinterpret_cast<float*>(smem + S.scratch) + warp * kWarpScratchFloats;
    float* partials = reinterpret_cast<float*>(smem + S.partials);
    const int C = sh.cols;
    bool ok = true;
    int pk0 = -2, pk1 = -2, c0 = -1, c1 = -1;

    for (int i = 0; i < n_my; ++i) {
        const Job Jb = decode_job(R, j0 + i, sh.row_blocks);
        const int key0 = Jb.slot0 < 0 ? -1 : (W13 ? R.slot_tok[Jb.slot0] : Jb.slot0);
        const int key1 = Jb.slot1 < 0 ? -1 : (W13 ? R.slot_tok[Jb.slot1] : Jb.slot1);
        if (key0 != pk0 || key1 != pk1) {   // uniform over the CTA
            ensure_cached<W13>(A, sh, cache, M, key0, key1, c0, c1);
            pk0 = key0;
            pk1 = key1;
        }
        TokRef tok[2];
        for (int e = 0; e < 2; ++e) {
            const int cs = e ? c1 : c0;
            if (cs < 0) {
                tok[e] = TokRef{nullptr, nullptr, nullptr, 1.f, nullptr};
                continue;
            }
            const uint8_t* base = cache + cs * sh.tok_bytes;
            tok[e] = TokRef{base, reinterpret_cast<const float*>(base + C * kPieces), nullptr, M.sigma[cs],
                            reinterpret_cast<const __half*>(base + C * kPieces + (C / 128) * 4)};
        }
        const int s = i % sh.n_stages;
        if (ok && !mbar_wait(full + s, (i / sh.n_stages) & 1)) {
            ok = false;
            if (lane == 0) set_status(A.ws.status, GALE_ERR_TIMEOUT);
        }
        const int r0 = Jb.tile * sh.job_rows + tr * 16;
        float part[2] = {0.f, 0.f};
        if (ok && r0 < sh.rows) {
            uint8_t* tile = smem + S.stages + s * sh.stage_bytes + (tr * sh.n_mat + mat) * sh.tile_bytes;
            chunk_compute(tile, view(Jb.e, mat), r0, ch, tok, scratch, part);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        float* pb = partials + (i & 1) * (kDecWarps * 32);
        if (lane < 16) {
            pb[warp * 32 + lane * 2] = part[0];
            pb[warp * 32 + lane * 2 + 1] = part[1];
        }
        named_bar_sync(1, kDecThreads);
        if (W13) {
            // h = silu(w1 x) * (w3 x) for the job's rows and tokens
            if (tid < sh.r_tiles * 32) {
                const int t_r = tid >> 5, row = tid & 15, t = (tid >> 4) & 1;
                const int slot = t ? Jb.slot1 : Jb.slot0;
                const int r = Jb.tile * sh.job_rows + t_r * 16 + row;
                float y1 = 0.f, y3 = 0.f;
                for (int c2 = 0; c2 < sh.n_chunk; ++c2) {
                    y1 += pb[((t_r * 2 + 0) * sh.n_chunk + c2) * 32 + row * 2 + t];
                    y3 += pb[((t_r * 2 + 1) * sh.n_chunk + c2) * 32 + row * 2 + t];
                }
                if (slot >= 0 && r < sh.rows) A.ws.h[int64_t(slot) * sh.rows + r] = silu(y1) * y3;
            }
            continue;
        }
        // ---- w2: expert outputs of the job's rows, then the (token, row block) combine
        if (tid < sh.r_tiles * 32) {
            const int t_r = tid >> 5, row = tid & 15, t = (tid >> 4) & 1;
            const int slot = t ? Jb.slot1 : Jb.slot0;
            const int r = Jb.tile * sh.job_rows + t_r * 16 + row;
            float y = 0.f;
            for (int c2 = 0; c2 < sh.n_chunk; ++c2) y += pb[(t_r * sh.n_chunk + c2) * 32 + row * 2 + t];
            if (slot >= 0 && r < d) A.ws.o[int64_t(slot) * d + r] = y;
            __threadfence();
        }
        named_bar_sync(1, kDecThreads);
        // combine granularity: 64-row blocks of d_model (a job covers job_rows >= 64 rows)
        const int nsub = sh.job_rows / 64;
        if (tid < 2 * nsub) {
            const int sl = tid & 1, sub = tid >> 1;
            const int slot = sl ? Jb.slot1 : Jb.slot0;
            int last = 0;
            const int rb = Jb.tile * nsub + sub;
            if (slot >= 0 && rb < comb_blocks) {
                const int t = R.slot_tok[slot];
                last = atomicAdd(A.ws.comb_cnt + t * comb_blocks + rb, 1) == R.tok_valid[t] - 1;
            }
            M.flag[tid] = last;   // flag index = 2 * sub + sl (nsub <= 2)
        }
        named_bar_sync(1, kDecThreads);
        for (int f = 0; f < 2 * nsub; ++f) {
            if (!M.flag[f]) continue;
            const int sl = f & 1, sub = f >> 1;
            const int slot = sl ? Jb.slot1 : Jb.slot0;
            const int t = R.slot_tok[slot];
            const int rb = Jb.tile * nsub + sub;
            __threadfence();
            float v = 0.f;
            const int r = rb * 64 + tid;
            const bool mine = tid < 64 && r < d;
            if (mine) {
                float y = 0.f;
                for (int k = 0; k < A.K; ++k) {
                    const int pos = R.pos_of_pair[t * A.K + k];
                    if (pos >= 0) y = fmaf(A.gates[t * A.K + k], __ldcg(A.ws.o + int64_t(pos) * d + r), y);
                }
                if (!A.fuse_norm) store_from_f32(A.out, A.out_dtype, int64_t(t) * d + r, y);
                else {
                    v = bf16_to_f32(A.x[int64_t(t) * d + r]) + y;
                    A.ws.v[int64_t(t) * d + r] = v;
                }
            }
            if (!A.fuse_norm) continue;
            // sum of squares of this 64-row block, fixed order
            const float ss = warp_sum(mine ? v * v : 0.f);
            if (lane == 0 && warp < 2) M.wsum[warp] = ss;
            if (mine) __threadfence();
            named_bar_sync(1, kDecThreads);
            if (tid == 0) {
                A.ws.ssq[t * comb_blocks + rb] = M.wsum[0] + M.wsum[1];
                __threadfence();
                M.flag[2 * nsub] = atomicAdd(A.ws.tok_cnt + t, 1) == comb_blocks - 1;
            }
            named_bar_sync(1, kDecThreads);
            if (!M.flag[2 * nsub]) continue;
            // every row block of token t is done: RMSNorm over d_model
            __threadfence();
            if (warp == 0) {
                float tot = 0.f;
                for (int q = lane; q < comb_blocks; q += 32) tot += __ldcg(A.ws.ssq + t * comb_blocks + q);
                tot = warp_sum(tot);
                if (lane == 0) M.inv = rsqrtf(tot / float(d) + A.eps);
            }
            named_bar_sync(1, kDecThreads);
            const float inv = M.inv;
            for (int c = tid; c < d; c += kDecThreads)
                store_from_f32(A.out, GALE_BF16, int64_t(t) * d + c, __ldcg(A.ws.v + int64_t(t) * d + c) * inv);
            named_bar_sync(1, kDecThreads);
        }
    }
}

template <typename Kern, typename... Args>
int launch_pdl(Kern kernel, int grid, int block, int smem, cudaStream_t st, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = size_t(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? GALE_OK : GALE_ERR_CUDA;
}

// Deepest ring (up to 6 stages) with at least `min_cap` cached vectors that
// fits the shared-memory budget.
Shape fit_shape(Shape sh, int min_cap, int max_cap) {
    constexpr int kBudget = 226 * 1024;
    for (int cap = max_cap; cap >= min_cap; --cap) {
        for (int st = 6; st >= 3; --st) {
            sh.n_stages = st;
            sh.tok_cap = cap;
            if (stream_smem(sh).bytes <= kBudget) return sh;
        }
    }
    sh.n_stages = 2;
    sh.tok_cap = min_cap;
    return sh;
}

}  // namespace

DecodeWs carve_decode_ws(void* ws, const gale_layer& L, int B, int K) {
    DecodeWs w{};
    char* p = static_cast<char*>(ws);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        char* q = p ? p + o : nullptr;
        o = align_up(o + bytes, 256);
        return q;
    };
    const int64_t P = int64_t(B) * K, dm = L.d_model, df = L.d_ff;
    const int64_t blocks = (dm + 63) / 64;
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.comb_cnt = reinterpret_cast<int32_t*>(take(4 * B * blocks));
    w.tok_cnt = reinterpret_cast<int32_t*>(take(4 * int64_t(B)));
    w.ssq = reinterpret_cast<float*>(take(4 * B * blocks));
    w.h = reinterpret_cast<float*>(take(4 * P * df));
    w.o = reinterpret_cast<float*>(take(4 * P * dm));
    w.v = reinterpret_cast<float*>(take(4 * B * dm));
    w.bytes = size_t(o);
    return w;
}

bool decode_supported(const gale_layer& L, int B, int K) {
    if (B < 1 || int64_t(B) * K > kDecodeMaxPairs || L.d_model > kDecodeMaxDModel || L.d_ff > kDecodeMaxDff ||
        L.n_experts > 1024 || !shape_ok(L.d_model, 2) || !shape_ok(L.d_ff, 1))
        return false;
    // the w2 jobs must cover whole 64-row combine blocks
    return make_shape(L.d_model, L.d_ff, 1).job_rows % 64 == 0 && make_shape(L.d_model, L.d_ff, 1).job_rows <= 128;
}

int launch_moe_decode(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                      void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st) {
    DecArgs A{};
    A.base = static_cast<const char*>(L.base);
    A.stride = L.expert_stride;
    A.E = L.n_experts;
    A.d_model = L.d_model;
    A.d_ff = L.d_ff;
    A.B = B;
    A.K = K;
    const int64_t l1 = make_layout(L.d_ff, L.d_model).total;
    A.off_w1 = 0;
    A.off_w3 = l1;
    A.off_w2 = 2 * l1;
    A.x = x;
    A.ids = ids;
    A.gates = gates;
    A.out = out;
    A.out_dtype = out_dtype;
    A.fuse_norm = fuse_norm;
    A.eps = eps;
    A.ws = carve_decode_ws(ws, L, B, K);

    CUtensorMap s1, b1, s3, b3, s2, b2;
    const char* base = static_cast<const char*>(L.base);
    int rc = cached_map(&s1, false, base, L.d_ff, L.d_model, L.n_experts, L.expert_stride);
    if (rc == GALE_OK) rc = cached_map(&b1, true, base, L.d_ff, L.d_model, L.n_experts, L.expert_stride);
    if (rc == GALE_OK) rc = cached_map(&s3, false, base + l1, L.d_ff, L.d_model, L.n_experts, L.expert_stride);
    if (rc == GALE_OK) rc = cached_map(&b3, true, base + l1, L.d_ff, L.d_model, L.n_experts, L.expert_stride);
    if (rc == GALE_OK) rc = cached_map(&s2, false, base + 2 * l1, L.d_model, L.d_ff, L.n_experts, L.expert_stride);
    if (rc == GALE_OK) rc = cached_map(&b2, true, base + 2 * l1, L.d_model, L.d_ff, L.n_experts, L.expert_stride);
    if (rc != GALE_OK) return rc;

    const int grid = sm_count();
    // w1/w3: an ordinary launch, so that it follows all earlier work on the stream
    const Shape s13 = fit_shape(make_shape(L.d_ff, L.d_model, 2), 2, 4);
    StreamSmem S = stream_smem(s13);
    rc = ensure_smem(reinterpret_cast<const void*>(moe_stream_kernel<true>), S.bytes);
    if (rc != GALE_OK) return rc;
    rc = launch_pdl(moe_stream_kernel<true>, grid, kDecThreads + 32, S.bytes, st, false, s1, b1, s3, b3, A, s13);
    if (rc != GALE_OK) return rc;
    // w2: programmatic dependent launch after w1/w3
    const Shape s2sh = fit_shape(make_shape(L.d_model, L.d_ff, 1), 2, 8);
    S = stream_smem(s2sh);
    rc = ensure_smem(reinterpret_cast<const void*>(moe_stream_kernel<false>), S.bytes);
    if (rc != GALE_OK) return rc;
    return launch_pdl(moe_stream_kernel<false>, grid, kDecThreads + 32, S.bytes, st, true, s2, b2, s2, b2, A, s2sh);
}

}  // namespace gale

// Decode path of gale_moe_forward: one persistent kernel, one CTA per SM,
// launched cooperatively (all CTAs resident).
//
//   routing : every CTA groups the (token, k) pairs by expert from the ids;
//             a job is (expert, group of <= 2 of its tokens, row block)
//   stream  : a producer warp copies the packed tiles of the CTA's w1/w3
//             jobs and then of its w2 jobs into a ring of stages (TMA), with
//             no dependency on any computation, so the w2 weights arrive
//             while w1/w3 is still being computed
//   w1/w3   : 8 consumer warps split each job by (matrix, 1024-column chunk)
//             on the int8 tensor cores; the outlier corrections of the job
//             are split by (matrix, row); the last warp to finish a job sums
//             the pieces and stores h = silu(w1 x) * (w3 x)
//   barrier : grid-wide (bounded wait): h of every expert is complete
//   w2      : the same with the rotated h rows; the last warp of a job
//             stores the expert outputs, and the last expert to finish a
//             (token, 64-row block) sums the K contributions in fixed k order
//             with the gates (deterministic, no float atomics), optionally
//             adding the residual; the last row block of a token applies
//             RMSNorm.
#include <cuda_bf16.h>

#include "common.cuh"
#include "fwht.cuh"
#include "moe.cuh"
#include "moe_decode.cuh"
#include "mma_tile.cuh"
#include "tma.cuh"

namespace gale {

namespace {

constexpr int kDecWarps = 8;                   // consumer warps
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecBlock = kDecThreads + 64;    // + the producer warp and the epilogue warp
constexpr int kPhaseBar = kDecThreads + 32;     // consumers and the epilogue warp
constexpr int kCapMax = 8;                     // rotated vectors cached per CTA
constexpr int kMaxStages = 16;

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

struct RouteTables {
    int active[kDecodeMaxPairs];       // active expert ids, increasing
    int first_slot[kDecodeMaxPairs];   // first slot of each active expert
    int n_tok[kDecodeMaxPairs];        // valid pairs of each active expert
    int grp_base[kDecodeMaxPairs + 1]; // first token group of each active expert
    int slot_tok[kDecodeMaxPairs];     // token of each slot
    int pos_of_pair[kDecodeMaxPairs];  // slot of each pair (-1: dropped)
    int tok_valid[kDecodeMaxPairs];    // valid pairs per token
    int n_active, n_groups, bad;
};

// Scratch of the block-wide routing; it lives in the ring before any copy starts.
struct RouteScratch {
    int cnt[1024];   // per expert: valid pairs
    int off[1024];   // per expert: first slot
    int aidx[1024];  // per expert: index among the active experts
    int pe[kDecodeMaxPairs];
    int scan_tmp[32];
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

// Small batches (B*K <= 32): one warp builds the tables.  Lane p holds pair
// p; a bitonic sort of the keys (expert << 5 | p) leaves the i-th valid pair
// of the stable expert order in lane i, which is its slot.
__device__ void build_route_small(const DecArgs& A, RouteTables& R) {
    const int lane = threadIdx.x & 31;
    const int BK = A.B * A.K, E = A.E, K = A.K;
    const bool in = lane < BK;
    const int e = in ? __ldg(A.ids + lane) : -1;
    bool ok = in && e >= 0 && e < E;
    {
        // an id repeated within a token drops the later pair
        const int t0 = lane - lane % K;
#pragma unroll 1
        for (int j = 0; j < K; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e, (t0 + j) & 31);
            if (t0 + j < lane && ej == e) ok = false;
        }
    }
    const unsigned okb = __ballot_sync(0xffffffffu, ok);
    const unsigned bad = __ballot_sync(0xffffffffu, in && !ok);
    uint32_t key = ok ? (uint32_t(e) << 5) | uint32_t(lane) : 0xFFFFFFFFu;
#pragma unroll
    for (int k2 = 2; k2 <= 32; k2 <<= 1) {
#pragma unroll
        for (int j = k2 >> 1; j > 0; j >>= 1) {
            const uint32_t other = __shfl_xor_sync(0xffffffffu, key, j);
            const bool keep_min = ((lane & j) == 0) == ((lane & k2) == 0);
            key = keep_min ? min(key, other) : max(key, other);
        }
    }
    const bool v = key != 0xFFFFFFFFu;
    const int se = v ? int(key >> 5) : -1, sp = int(key & 31u);
    const int nvalid = __popc(okb);
    if (v) {
        R.slot_tok[lane] = sp / K;
        R.pos_of_pair[sp] = lane;
    }
    if (in && !ok) R.pos_of_pair[lane] = -1;
    // runs of equal experts in slot order: the active experts
    const int prev = __shfl_up_sync(0xffffffffu, se, 1);
    const bool first = v && (lane == 0 || prev != se);
    const unsigned fb = __ballot_sync(0xffffffffu, first);
    const unsigned later = lane == 31 ? 0u : fb & (0xFFFFFFFFu << (lane + 1));
    const int run = (later ? __ffs(later) - 1 : nvalid) - lane;
    const int groups = first ? (run + 1) / 2 : 0;
    int incl = groups;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (first) {
        const int a = __popc(fb & ((1u << lane) - 1u));
        R.active[a] = se;
        R.first_slot[a] = lane;
        R.n_tok[a] = run;
        R.grp_base[a] = incl - groups;
    }
    if (lane < A.B) R.tok_valid[lane] = __popc(okb & (((1u << K) - 1u) << (lane * K)));
    const int n_groups = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
        const int n_active = __popc(fb);
        R.n_active = n_active;
        R.n_groups = n_groups;
        R.grp_base[n_active] = n_groups;
        R.bad = bad != 0u;
    }
}

// Stable grouping of the (token, k) pairs by expert: every active expert has
// ceil(n_tok / 2) token groups of at most two tokens.  All threads call it.
__device__ void build_route(const DecArgs& A, RouteTables& R, RouteScratch& T) {
    const int tid = threadIdx.x;
    const int BK = A.B * A.K, E = A.E;
    if (BK <= 32) {
        if (tid < 32) build_route_small(A, R);
        __syncthreads();
        return;
    }
#pragma unroll 1
    for (int e = tid; e < E; e += blockDim.x) T.cnt[e] = 0;
#pragma unroll 1
    for (int t = tid; t < A.B; t += blockDim.x) R.tok_valid[t] = 0;
    if (tid == 0) R.bad = 0;
    __syncthreads();
#pragma unroll 1
    for (int p = tid; p < BK; p += blockDim.x) {
        const int e = A.ids[p];
        bool ok = e >= 0 && e < E;
        const int t0 = p - p % A.K;
#pragma unroll 1
        for (int j = t0; ok && j < p; ++j) ok = A.ids[j] != e;
        T.pe[p] = ok ? e : -1;
        if (ok) {
            atomicAdd(&T.cnt[e], 1);
            atomicAdd(&R.tok_valid[p / A.K], 1);
        } else {
            R.bad = 1;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int e = tid; e < E; e += blockDim.x) {
        T.off[e] = T.cnt[e];
        T.aidx[e] = T.cnt[e] > 0;
    }
    __syncthreads();
    block_exclusive_scan(T.off, E, T.scan_tmp);
    const int n_active = block_exclusive_scan(T.aidx, E, T.scan_tmp);
#pragma unroll 1
    for (int e = tid; e < E; e += blockDim.x) {
        if (T.cnt[e] > 0) {
            const int a = T.aidx[e];
            R.active[a] = e;
            R.first_slot[a] = T.off[e];
            R.n_tok[a] = T.cnt[e];
            R.grp_base[a] = (T.cnt[e] + 1) / 2;
        }
    }
#pragma unroll 1
    for (int p = tid; p < BK; p += blockDim.x) {
        const int e = T.pe[p];
        int slot = -1;
        if (e >= 0) {
            int rank = 0;
#pragma unroll 1
            for (int q = 0; q < p; ++q) rank += (T.pe[q] == e);
            slot = T.off[e] + rank;
            R.slot_tok[slot] = p / A.K;
        }
        R.pos_of_pair[p] = slot;
    }
    __syncthreads();
    const int n_groups = block_exclusive_scan(R.grp_base, n_active, T.scan_tmp);
    if (tid == 0) {
        R.n_active = n_active;
        R.n_groups = n_groups;
        R.grp_base[n_active] = n_groups;
    }
    __syncthreads();
}

struct Job {
    int e, tile, slot0, slot1;
};

// Job j of a phase with `tiles` row blocks per token group.
__device__ __forceinline__ Job decode_job(const RouteTables& R, int j, int tiles) {
    const int gi = j / tiles;
    int lo = 0, hi = R.n_active - 1;   // last a with grp_base[a] <= gi
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (R.grp_base[mid] <= gi) lo = mid;
        else hi = mid - 1;
    }
    Job J;
    J.e = R.active[lo];
    J.tile = j - gi * tiles;
    const int g = gi - R.grp_base[lo];
    J.slot0 = R.first_slot[lo] + 2 * g;
    J.slot1 = (2 * g + 1 < R.n_tok[lo]) ? J.slot0 + 1 : -1;
    return J;
}

// A job packed in 8 bytes: (expert, row block) and the two slots (0xFFFF: none).
__device__ __forceinline__ uint2 pack_job(const Job& J) {
    return make_uint2(uint32_t(J.e) | (uint32_t(J.tile) << 16), uint32_t(J.slot0 & 0xFFFF) | (uint32_t(J.slot1 & 0xFFFF) << 16));
}
__device__ __forceinline__ Job unpack_job(uint2 v) {
    Job J;
    J.e = int(v.x & 0xFFFFu);
    J.tile = int(v.x >> 16);
    J.slot0 = int(v.y & 0xFFFFu);
    J.slot1 = (v.y >> 16) == 0xFFFFu ? -1 : int(v.y >> 16);
    return J;
}

// ----------------------------------------------------------------------------
// shapes and shared memory
// ----------------------------------------------------------------------------

// One matrix's part of a staged job of R consecutive rows.  In a packed record
// the R rows of every section are contiguous, so each section arrives in one
// bulk copy (large copies keep the copy engines near full bandwidth; 16-row
// boxes of 2 KB reached about a third of it).  Signs stay in record order:
// row r at r * C / 8 bytes.
struct JobTile {
    int signs, scales, idx, q, srow, bytes;
};

__host__ __device__ inline JobTile job_tile(int C, int R) {
    const int k = outliers_per_row(C);
    JobTile t;
    int o = 0;
    t.signs = o;
    o += R * (C / 8);
    t.scales = o;
    o += R * (C / 64);
    t.idx = o;
    o += (R * k * 2 + 15) & ~15;
    t.q = o;
    o += ((R * k + 1) / 2 + 31) & ~15;   // plus the source's offset from a 16-byte boundary
    t.srow = o;
    o += (R * 2 + 15) & ~15;
    t.bytes = (o + 1023) & ~1023;   // the signs of every tile start on a 1024-byte swizzle atom
    return t;
}

// ----------------------------------------------------------------------------
// ----------------------------------------------------------------------------

struct Shape {
    int rows, cols;      // rows and columns of the streamed matrices
    int n_mat;           // 2 (w1, w3) or 1 (w2)
    int n_chunk;         // cols / 1024
    int r_tiles;         // 16-row tiles per job: 8 / (n_mat * n_chunk)
    int job_rows;        // 16 * r_tiles
    int row_blocks;      // jobs per token group: ceil(rows / job_rows)
    int mat_bytes;       // job_tile(cols, job_rows).bytes
    int stage_bytes;     // n_mat * mat_bytes
    int tok_bytes;       // digits + 128-block sums + fp16 copy of one rotated vector
    int pairs;           // (matrix, row) pairs of a job: n_mat * job_rows
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
    s.mat_bytes = job_tile(cols, s.job_rows).bytes;
    s.stage_bytes = n_mat * s.mat_bytes;
    s.tok_bytes = int(align_up(cols * kPieces + (cols / 128) * 4 + cols * 2, 16));
    s.pairs = n_mat * s.job_rows;
    return s;
}

// the 8 consumer warps must split a job evenly
__host__ __device__ inline bool shape_ok(int cols, int n_mat) {
    const int units = n_mat * (cols / 1024);
    return cols % 1024 == 0 && units >= 1 && units <= kDecWarps && kDecWarps % units == 0;
}

struct Plan {
    Shape s13, s2;
    int n_stages, stage_bytes, cache_bytes, cap13, cap2;
    int max_jobs;   // jobs of both phases one CTA may get
};

struct CacheSmem {
    int key[kCapMax];
    float sigma[kCapMax];
    int stamp[kCapMax];
    int plan_slot[2], plan_key[2], n_plan, clock;
    float red[kDecWarps];
    int cres[2];                  // cache indices of the current job's vectors
    int gate_ok;
};

constexpr int kPartFloats = kDecWarps * 32 + 2 * 128;   // per stage: MMA pieces + outlier sums

struct DecSmem {
    int ring, cache, route, jobs, part, scratch, bars, misc, bytes;
};

__host__ __device__ inline DecSmem dec_smem(const Plan& P) {
    DecSmem s;
    int o = 0;
    s.ring = o;
    o += P.n_stages * P.stage_bytes;
    s.cache = o;
    o += P.cache_bytes;
    s.route = o;
    o += int(align_up(sizeof(RouteTables), 16));
    s.jobs = o;
    o += int(align_up(8 * P.max_jobs, 16));
    s.part = o;
    o += P.n_stages * kPartFloats * 4;
    s.scratch = o;
    o += kDecWarps * kWarpScratchFloats * 4;
    s.bars = o;
    o += 3 * P.n_stages * 8;
    s.misc = o;
    o += int(align_up(sizeof(CacheSmem), 16));
    s.bytes = int(align_up(o, 1024)) + 1024;
    return s;
}

// ----------------------------------------------------------------------------
// rotated-vector cache
// ----------------------------------------------------------------------------

// Make sure the rotated vectors `key0`, `key1` (tokens for w1/w3, slots for
// w2; -1 = none) are in the shared-memory cache; returns their cache
// indices.  All consumer threads call it (named barrier 1).  A missing vector
// is loaded (bf16 x or fp32 h), rotated by FWHT-1024 (one warp per
// 1024-block), and turned into digits, 128-block sums and an fp16 copy; the
// least recently used entry is replaced.
__device__ __forceinline__ void ensure_cached(const DecArgs& A, const Shape& sh, int cap, uint8_t* cache, CacheSmem& M,
                                          bool W13, int key0, int key1, int& c0, int& c1) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C = sh.cols, nblk = C / 1024;
    if (warp == 0) {
        // lane q < cap looks after cache entry q; hits by ballot, victims by a
        // warp-wide argmin of (stamp, entry)
        const int kq = lane < cap ? M.key[lane] : -2;
        int stq = lane < cap ? M.stamp[lane] : 0x7fffffff;
        const unsigned m0 = __ballot_sync(0xffffffffu, key0 >= 0 && kq == key0);
        const unsigned m1 = __ballot_sync(0xffffffffu, key1 >= 0 && kq == key1);
        int f0 = m0 ? __ffs(m0) - 1 : -1, f1 = m1 ? __ffs(m1) - 1 : -1;
        int nk = kq, n_plan = 0;
        auto victim = [&](int other) {
            int best = (lane < cap && lane != other) ? stq : 0x7fffffff, bl = lane;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const int ob = __shfl_xor_sync(0xffffffffu, best, o), ol = __shfl_xor_sync(0xffffffffu, bl, o);
                if (ob < best || (ob == best && ol < bl)) {
                    best = ob;
                    bl = ol;
                }
            }
            return bl;
        };
        if (key0 >= 0 && f0 < 0) {
            f0 = victim(f1);
            if (lane == f0) nk = key0;
            if (lane == 0) {
                M.plan_slot[n_plan] = f0;
                M.plan_key[n_plan] = key0;
            }
            ++n_plan;
        }
        if (key1 >= 0 && f1 < 0) {
            f1 = victim(f0);
            if (lane == f1) nk = key1;
            if (lane == 0) {
                M.plan_slot[n_plan] = f1;
                M.plan_key[n_plan] = key1;
            }
            ++n_plan;
        }
        int clk = M.clock;
        if (f0 >= 0 && lane == f0) stq = clk + 1;
        if (f0 >= 0) ++clk;
        if (f1 >= 0 && lane == f1) stq = clk + 1;
        if (f1 >= 0) ++clk;
        __syncwarp();
        if (lane < cap) {
            M.key[lane] = nk;
            M.stamp[lane] = stq;
        }
        if (lane == 0) {
            M.clock = clk;
            M.n_plan = n_plan;
            M.cres[0] = f0;
            M.cres[1] = f1;
        }
    }
    named_bar_sync(1, kDecThreads);
    c0 = M.cres[0];
    c1 = M.cres[1];
    const int n_plan = M.n_plan;
    if (n_plan == 0) return;
    // warps [e * nblk, (e + 1) * nblk) rotate entry e, one 1024-block each.
    // Lane l loads elements 32 i + l; butterflies over the register index
    // (element bits 5..9); a transpose through the entry's own (not yet
    // written) bytes gives lane l the elements 32 l + i; butterflies over the
    // register index again (bits 0..4).  Lane l = 4 b + tig then holds the
    // 32 consecutive columns 128 b + 32 tig + i, which are exactly the four
    // elements (i = q + 8 i') of each of its digit words (b, tig, q).
    const int e = warp / nblk, blk = warp % nblk;
    const bool act = e < n_plan;
    float v[32];
    uint8_t* dst = act ? cache + M.plan_slot[e] * sh.tok_bytes : cache;
    if (act) {
        const int key = M.plan_key[e];
        if (W13) {
            const uint16_t* src = A.x + int64_t(key) * C + blk * 1024;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = bf16_to_f32(src[32 * i + lane]);
        } else {
            const float* src = A.ws.h + int64_t(key) * C + blk * 1024;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __ldcg(src + 32 * i + lane);
        }
        fwht32_cg(v);
        float* tb = reinterpret_cast<float*>(dst) + blk * 33 * 32;   // 33-float rows: no bank conflicts
#pragma unroll
        for (int i = 0; i < 32; ++i) tb[i * 33 + lane] = v[i];
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = tb[lane * 33 + i] * (1.0f / 32.0f);
        fwht32_cg(v);
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) M.red[warp] = m;
    }
    named_bar_sync(1, kDecThreads);   // every transpose has been read back; block maxima known
    if (act) {
        float m = 0.f;
        for (int w = e * nblk; w < (e + 1) * nblk; ++w) m = fmaxf(m, M.red[w]);
        const float S = fixed_scale(m);
        const int b = blk * 8 + (lane >> 2), tig = lane & 3;
        // fp16 copy of v S / 64 (|v S| <= 2^20, so it cannot overflow whatever
        // the size of the vector; the outlier sums are scaled back by 64 / S)
        // and the 128-block sums
        uint4* x16 = reinterpret_cast<uint4*>(dst + C * kPieces + (C / 128) * 4) + blk * 128 + lane * 4;
        const float s64 = S * 0.015625f;
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t hw[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half2 h2 = __floats2half2_rn(v[8 * i + 2 * j] * s64, v[8 * i + 2 * j + 1] * s64);
                hw[j] = *reinterpret_cast<const uint32_t*>(&h2);
                sum += v[8 * i + 2 * j] + v[8 * i + 2 * j + 1];
            }
            x16[i] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (tig == 0) reinterpret_cast<float*>(dst + C * kPieces)[b] = sum;
        // digit word q takes registers q, q + 8, q + 16, q + 24: a rolled loop
        // over q that shifts the registers down by one each time (small code
        // for a step that runs once per vector)
        uint32_t* pieces = reinterpret_cast<uint32_t*>(dst + b * kPieceBlockBytes + tig * 32);
#pragma unroll 1
        for (int q = 0; q < 8; ++q) {
            const float sc = S * inv_a(q);
            uint32_t word[kPieces] = {0u, 0u, 0u};
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                uint32_t d1, d2, d3;
                fixed_digits(v[8 * i4] * sc, d1, d2, d3);
                word[0] |= d1 << (8 * i4);
                word[1] |= d2 << (8 * i4);
                word[2] |= d3 << (8 * i4);
            }
#pragma unroll
            for (int j = 0; j < kPieces; ++j) pieces[j * 32 + q] = word[j];
#pragma unroll
            for (int i = 0; i < 31; ++i) v[i] = v[i + 1];
        }
        if (blk == 0 && lane == 0) M.sigma[M.plan_slot[e]] = 1.0f / S;
    }
    named_bar_sync(1, kDecThreads);
}

// ----------------------------------------------------------------------------
// per-warp pieces of a job
// ----------------------------------------------------------------------------

// Tensor-core part of one 1024-column chunk `ch` of 16 staged rows (signs in
// record order from `signs16`, block scales from `sblk`) for
// up to two tokens: lanes 0..15 return, for row r0 + lane and tokens 0 and 1,
//   sum_{b in chunk} s_blk[row, b] (X_b - 2 P_b).
// The chunk's eight 128-column blocks run in two halves of four blocks with
// one accumulator each, so that consecutive MMAs are independent.
__device__ __forceinline__ void chunk_mma(const uint8_t* signs, const __half* sblk, int C, int ch,
                                          const TokRef (&tok)[2], float* scratch, float (&part)[2]) {
    // signs: this chunk's 128-byte piece of the tile's first row, swizzled
    // (16-byte chunk bb of row r at position bb ^ (r & 7)); rows 128 bytes apart
    const int lane = threadIdx.x & 31;
    const int nb = C / 128;
    const int row = lane & 15, half = lane >> 4;
    const bool has0 = tok[0].pieces != nullptr, has1 = tok[1].pieces != nullptr;

    // block-scale-weighted 128-block sums of x over the chunk (4 blocks per half)
    float xt0 = 0.f, xt1 = 0.f;
    {
        const int b0 = ch * 8 + half * 4;
        const uint2 sv = *reinterpret_cast<const uint2*>(sblk + row * nb + b0);
        const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sv.x));
        const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sv.y));
        if (has0) {
            const float4 x = *reinterpret_cast<const float4*>(tok[0].xsum + b0);
            xt0 = s01.x * x.x + s01.y * x.y + s23.x * x.z + s23.y * x.w;
        }
        if (has1) {
            const float4 x = *reinterpret_cast<const float4*>(tok[1].xsum + b0);
            xt1 = s01.x * x.x + s01.y * x.y + s23.x * x.z + s23.y * x.w;
        }
    }

    const int g = lane >> 2, tig = lane & 3;
    const bool bsrc = g < 6 && (g < 3 ? has0 : has1);
    const uint8_t* pieces = (g < 3 ? tok[0].pieces : tok[1].pieces);
    const uint8_t* bsrc_p = bsrc ? pieces + (g % 3) * 128 + tig * 32 + ch * 8 * kPieceBlockBytes : nullptr;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
        uint32_t wg[4], wg8[4];
        uint4 q0[4], q1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int bb = 4 * hb + j;
            const uint8_t* wa = signs + g * 128 + ((bb ^ g) << 4) + tig * 4;   // rows g and g + 8 share g & 7
            wg[j] = *reinterpret_cast<const uint32_t*>(wa);
            wg8[j] = *reinterpret_cast<const uint32_t*>(wa + 8 * 128);
            if (bsrc) {
                q0[j] = *reinterpret_cast<const uint4*>(bsrc_p + bb * kPieceBlockBytes);
                q1[j] = *reinterpret_cast<const uint4*>(bsrc_p + bb * kPieceBlockBytes + 16);
            } else {
                q0[j] = make_uint4(0u, 0u, 0u, 0u);
                q1[j] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        int c[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0;
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t a0, a1, a2, a3;
                a_regs(wg[j], wg8[j], mm, a0, a1, a2, a3);
                const uint32_t b0 = mm == 0 ? q0[j].x : mm == 1 ? q0[j].z : mm == 2 ? q1[j].x : q1[j].z;
                const uint32_t b1 = mm == 0 ? q0[j].y : mm == 1 ? q0[j].w : mm == 2 ? q1[j].y : q1[j].w;
                mma_s8(c[j], a0, a1, a2, a3, b0, b1);
            }
        }
        const uint2 sg = *reinterpret_cast<const uint2*>(sblk + g * nb + ch * 8 + 4 * hb);
        const uint2 sg8 = *reinterpret_cast<const uint2*>(sblk + (g + 8) * nb + ch * 8 + 4 * hb);
        const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&sg.x));
        const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&sg.y));
        const float2 h01 = __half22float2(*reinterpret_cast<const __half2*>(&sg8.x));
        const float2 h23 = __half22float2(*reinterpret_cast<const __half2*>(&sg8.y));
        const float sgv[4] = {g01.x, g01.y, g23.x, g23.y}, s8v[4] = {h01.x, h01.y, h23.x, h23.y};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[0] = fmaf(sgv[j], float(c[j][0]), acc[0]);
            acc[1] = fmaf(sgv[j], float(c[j][1]), acc[1]);
            acc[2] = fmaf(s8v[j], float(c[j][2]), acc[2]);
            acc[3] = fmaf(s8v[j], float(c[j][3]), acc[3]);
        }
    }
    // gather the 8 MMA columns of every row through shared memory
    scratch[g * 8 + 2 * tig] = acc[0];
    scratch[g * 8 + 2 * tig + 1] = acc[1];
    scratch[(g + 8) * 8 + 2 * tig] = acc[2];
    scratch[(g + 8) * 8 + 2 * tig + 1] = acc[3];
    __syncwarp();
    xt0 += __shfl_xor_sync(0xffffffffu, xt0, 16);
    xt1 += __shfl_xor_sync(0xffffffffu, xt1, 16);
    const float* col = scratch + row * 8;
    part[0] = has0 ? xt0 - 2.0f * tok[0].sigma * (col[0] * 16384.0f + col[1] * 128.0f + col[2]) : 0.f;
    part[1] = has1 ? xt1 - 2.0f * tok[1].sigma * (col[3] * 16384.0f + col[4] * 128.0f + col[5]) : 0.f;
    __syncwarp();
}

// Outlier corrections  sum_j (q s_row - sign s_blk) x_c  of one row of a
// staged tile over the outliers j = sub, sub + step, ... (a fixed lane set
// of the row sums them afterwards in a fixed order); six at a time so that
// their loads overlap.
__device__ __forceinline__ void row_outliers(const uint8_t* tile, const JobTile& L, int C, int job_rows, int k,
                                             int q_delta, int row, int sub, int step, const TokRef (&tok)[2],
                                             float& corr0, float& corr1) {
    const int nb = C / 128;
    const uint16_t* ri = reinterpret_cast<const uint16_t*>(tile + L.idx) + row * k;
    const uint8_t* qn = tile + L.q + q_delta;
    const __half* sblk = reinterpret_cast<const __half*>(tile + L.scales) + row * nb;
    // the row in the swizzled sign layout: [piece][row][128 bytes]
    const uint8_t* signs = tile + L.signs + row * 128;
    const int piece_bytes = job_rows * 128, sw = row & 7;
    const float srow = __half2float(reinterpret_cast<const __half*>(tile + L.srow)[row]);
    const bool has0 = tok[0].pieces != nullptr, has1 = tok[1].pieces != nullptr;
    const __half* x0 = tok[0].x16;
    const __half* x1 = tok[1].x16;
    float c0 = 0.f, c1 = 0.f;   // in units of the fp16 copies (v S / 64)
    for (int jb = sub; jb < k; jb += 6 * step) {
        int c[6];
        bool use[6];
#pragma unroll
        for (int u = 0; u < 6; ++u) {
            const int j = jb + u * step;
            c[u] = j < k ? int(ri[j]) : C;
            use[u] = c[u] < C;   // past the row's outliers, or a record that failed validation
            if (!use[u]) c[u] = 0;
        }
#pragma unroll
        for (int u = 0; u < 6; ++u) {
            const int n = row * k + (use[u] ? jb + u * step : 0);
            const int qb = int(qn[n >> 1]) >> ((n & 1) * 4);
            const int qv = (qb & 15) - ((qb & 8) << 1);
            const int wd = (c[u] >> 5) & 31;   // word within the 1024-column piece
            const uint32_t word = *reinterpret_cast<const uint32_t*>(signs + (c[u] >> 10) * piece_bytes +
                                                                     (((wd >> 2) ^ sw) << 4) + (wd & 3) * 4);
            const float sb = __half2float(sblk[c[u] >> 7]);
            float wq = fmaf(float(qv), srow, ((word >> (c[u] & 31)) & 1u) ? sb : -sb);
            wq = use[u] ? wq : 0.f;
            if (has0) c0 = fmaf(wq, __half2float(x0[c[u]]), c0);
            if (has1) c1 = fmaf(wq, __half2float(x1[c[u]]), c1);
        }
    }
    if (has0) corr0 = fmaf(c0, 64.0f * tok[0].sigma, corr0);
    if (has1) corr1 = fmaf(c1, 64.0f * tok[1].sigma, corr1);
}

// ----------------------------------------------------------------------------
// the kernel
// ----------------------------------------------------------------------------

// The epilogue of a job, run by the epilogue warp, in two parts.  epi_rows
// sums the job's partial sums (shared memory of the job's stage) row tile by
// row tile and stores the rows: h = silu(w1 x) * (w3 x) for w1/w3, the expert
// outputs o for w2; after it the stage can be refilled.  epi_combine (w2
// only) runs the (token, 64-row block) combine and the RMSNorm of finished
// tokens.  Lane l covers row l & 15 of every row tile and token slot l >> 4.
__device__ __forceinline__ void epi_rows(const DecArgs& A, const Shape& sh, bool W13, const Job& Jb,
                                         const float* pb, int lane) {
    const float* pc = pb + kDecWarps * 32;
    const int row = lane & 15, t = lane >> 4;
    const int m1 = W13 ? 2 : 1;
    const int slot = t ? Jb.slot1 : Jb.slot0;
    const int d = A.d_model;
#pragma unroll 1
    for (int i = 0; i < sh.r_tiles; ++i) {
        // outlier sums first, then the MMA pieces in chunk order
        float y1 = pc[(i * 16 + row) * 2 + t];
        float y3 = W13 ? pc[(sh.job_rows + i * 16 + row) * 2 + t] : 0.f;
        const float* p1 = pb + i * m1 * sh.n_chunk * 32 + row * 2 + t;
        const float* p3 = p1 + sh.n_chunk * 32;
#pragma unroll 4
        for (int c2 = 0; c2 < sh.n_chunk; ++c2) {
            y1 += p1[c2 * 32];
            if (W13) y3 += p3[c2 * 32];
        }
        const int r = Jb.tile * sh.job_rows + i * 16 + row;
        if (slot < 0 || r >= sh.rows) continue;
        if (W13) A.ws.h[int64_t(slot) * sh.rows + r] = __fdividef(y1, 1.0f + __expf(-y1)) * y3;
        else A.ws.o[int64_t(slot) * d + r] = y1;
    }
}

__device__ __forceinline__ void epi_combine(const DecArgs& A, const RouteTables& R, const Shape& sh, const Job& Jb,
                                            int lane) {
    const int d = A.d_model;
    const int comb_blocks = (d + 63) / 64;
    __threadfence();
    __syncwarp();
    // the (token, 64-row block) combine: the last expert to finish sums the K outputs
    const int nsub = sh.job_rows / 64;
    int flags = 0;
    if (lane < 2 * nsub) {
        const int sl = lane & 1, sb = lane >> 1;
        const int slot = sl ? Jb.slot1 : Jb.slot0;
        const int rb = Jb.tile * nsub + sb;
        if (slot >= 0 && rb < comb_blocks) {
            const int t = R.slot_tok[slot];
            flags = atomicAdd(A.ws.comb_cnt + t * comb_blocks + rb, 1) == R.tok_valid[t] - 1;
        }
    }
    const unsigned fl = __ballot_sync(0xffffffffu, flags);
#pragma unroll 1
    for (int f = 0; f < 2 * nsub; ++f) {
        if (!((fl >> f) & 1)) continue;
        __threadfence();
        const int sl = f & 1, sb = f >> 1;
        const int t = R.slot_tok[sl ? Jb.slot1 : Jb.slot0];
        const int rb = Jb.tile * nsub + sb;
        // lane k holds the token's (k0 + k)-th (slot, gate); eight experts'
        // loads in flight at a time; the sum runs in fixed k order
        const int r0 = rb * 64 + lane, r1 = r0 + 32;
        // the residual rows are loaded first, alongside the expert outputs
        float x0 = 0.f, x1 = 0.f;
        if (A.fuse_norm) {
            if (r0 < d) x0 = bf16_to_f32(A.x[int64_t(t) * d + r0]);
            if (r1 < d) x1 = bf16_to_f32(A.x[int64_t(t) * d + r1]);
        }
        float y0 = 0.f, y1 = 0.f;
#pragma unroll 1
        for (int k0 = 0; k0 < A.K; k0 += 32) {
            int pos_l = -1;
            float g_l = 0.f;
            if (k0 + lane < A.K) {
                pos_l = R.pos_of_pair[t * A.K + k0 + lane];
                g_l = A.gates[t * A.K + k0 + lane];
            }
            const int kn = A.K - k0 < 32 ? A.K - k0 : 32;
#pragma unroll 1
            for (int k8 = 0; k8 < kn; k8 += 8) {
                float o0[8], o1[8], gg[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int pos = __shfl_sync(0xffffffffu, pos_l, (k8 + j) & 31);
                    gg[j] = __shfl_sync(0xffffffffu, g_l, (k8 + j) & 31);
                    o0[j] = o1[j] = 0.f;
                    if (k8 + j < kn && pos >= 0) {
                        const float* orow = A.ws.o + int64_t(pos) * d;
                        if (r0 < d) o0[j] = __ldcg(orow + r0);
                        if (r1 < d) o1[j] = __ldcg(orow + r1);
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    y0 = fmaf(gg[j], o0[j], y0);
                    y1 = fmaf(gg[j], o1[j], y1);
                }
            }
        }
        if (!A.fuse_norm) {
            if (r0 < d) store_from_f32(A.out, A.out_dtype, int64_t(t) * d + r0, y0);
            if (r1 < d) store_from_f32(A.out, A.out_dtype, int64_t(t) * d + r1, y1);
            continue;
        }
        float ss = 0.f;
        if (r0 < d) {
            const float v = x0 + y0;
            A.ws.v[int64_t(t) * d + r0] = v;
            ss = v * v;
        }
        if (r1 < d) {
            const float v = x1 + y1;
            A.ws.v[int64_t(t) * d + r1] = v;
            ss = fmaf(v, v, ss);
        }
        // sum of squares of this 64-row block (fixed order), then the last
        // block of the token normalises the whole row
        ss = warp_sum(ss);
        int lastblk = 0;
        if (lane == 0) {
            A.ws.ssq[t * comb_blocks + rb] = ss;
            __threadfence();
            lastblk = atomicAdd(A.ws.tok_cnt + t, 1) == comb_blocks - 1;
        }
        __syncwarp();
        lastblk = __shfl_sync(0xffffffffu, lastblk, 0);
        if (!lastblk) continue;
        __threadfence();
        // sixteen 16-byte loads of the row in flight per lane (the first
        // batch together with the block sums of squares), then bf16 pairs out
        const float4* vrow = reinterpret_cast<const float4*>(A.ws.v + int64_t(t) * d);
        __nv_bfloat162* orow = reinterpret_cast<__nv_bfloat162*>(static_cast<uint16_t*>(A.out) + int64_t(t) * d);
        const int n4 = d / 4;
        float inv = 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < n4; c0 += 32 * 16) {
            float4 vv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int c = c0 + 32 * j + lane;
                vv[j] = c < n4 ? __ldcg(vrow + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (c0 == 0) {
                float tot = 0.f;
                for (int q = lane; q < comb_blocks; q += 32) tot += __ldcg(A.ws.ssq + t * comb_blocks + q);
                tot = warp_sum(tot);
                inv = rsqrtf(tot / float(d) + A.eps);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < n4) {
                    orow[2 * c] = __floats2bfloat162_rn(vv[j].x * inv, vv[j].y * inv);
                    orow[2 * c + 1] = __floats2bfloat162_rn(vv[j].z * inv, vv[j].w * inv);
                }
            }
        }
    }
}


__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of the cooperative launch, one thread per CTA (whose
// threads have fenced their writes before the CTA barrier that precedes it);
// the counter starts at zero every call.  Every CTA adds one and polls the
// counter itself until all G have arrived: the release is the last arrival,
// with no separate flag.  False if the wait ran out (2 s).
__device__ bool grid_barrier(int32_t* cnt, int G) {
    __threadfence();
    atomicAdd(cnt, 1);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(cnt) < G)
        if (globaltimer_ns() - t0 > 2000000000ull) return false;
    __threadfence();
    return true;
}


__global__ void __launch_bounds__(kDecBlock, 1) moe_decode_kernel(const __grid_constant__ CUtensorMap map13,
                                                                   const __grid_constant__ CUtensorMap map2, DecArgs A,
                                                                   Plan P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const DecSmem S = dec_smem(P);
    RouteTables& R = *reinterpret_cast<RouteTables*>(smem + S.route);
    CacheSmem& M = *reinterpret_cast<CacheSmem*>(smem + S.misc);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* empty = full + P.n_stages;
    uint64_t* done = empty + P.n_stages;   // the 8 pieces of the stage's job are in its partial sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;

    if (warp == kDecWarps && lane == 0) {   // the producer's descriptors, before the routing is known
        prefetch_tensormap(&map13);
        prefetch_tensormap(&map2);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < P.n_stages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);           // the epilogue warp, once it has gathered the job
            mbar_init(done + s, kDecWarps);
        }
        fence_mbar_init();
        for (int q = 0; q < kCapMax; ++q) {
            M.key[q] = -1;
            M.stamp[q] = 0;
        }
        M.clock = 0;
    }
    {
        // the first tokens' rows of x head for L2 while the routing is built
        const int64_t xb = int64_t(A.B < 8 ? A.B : 8) * A.d_model * 2;
        for (int64_t o = int64_t(threadIdx.x) * 128; o < xb; o += int64_t(blockDim.x) * 128)
            prefetch_l2(reinterpret_cast<const char*>(A.x) + o);
    }
    const bool small = A.B * A.K <= 32;
    if (small) {
        // small batches: the epilogue warp routes the pairs and releases the
        // producer at once; meanwhile, for one or two tokens, the consumers
        // rotate x (its tokens are known without the routing) into cache
        // entries that the jobs then find
        __syncthreads();   // the cache bookkeeping is initialised
        if (warp == kDecWarps + 1) {
            build_route_small(A, R);
            __syncwarp();
            named_bar_arrive(3, 64);          // with the producer
            named_bar_arrive(4, kPhaseBar);   // with the consumers
        } else if (warp == kDecWarps) {
            named_bar_sync(3, 64);
        } else {
            if (A.B <= 2) {
                int c0, c1;
                ensure_cached(A, P.s13, P.cap13, smem + S.cache, M, true, 0, A.B > 1 ? 1 : -1, c0, c1);
            }
            named_bar_sync(4, kPhaseBar);
        }
    } else {
        build_route(A, R, *reinterpret_cast<RouteScratch*>(smem + S.ring));   // contains __syncthreads
    }
    // contiguous job ranges of this CTA in both phases; the producer decodes
    // its jobs as it goes, the other warps read them from a table
    const int J13 = R.n_groups * P.s13.row_blocks, J2 = R.n_groups * P.s2.row_blocks;
    // (J * G < 2^32: at most 384 groups x 256 row blocks x the SM count; 32-bit divisions)
    const unsigned g = unsigned(G), bx = blockIdx.x;
    const int a0 = int(unsigned(J13) * bx / g), n13 = int(unsigned(J13) * (bx + 1) / g) - a0;
    const int b0 = int(unsigned(J2) * bx / g), n2 = int(unsigned(J2) * (bx + 1) / g) - b0;
    uint2* jobs = reinterpret_cast<uint2*>(smem + S.jobs);
    if (warp < kDecWarps)
        for (int i = threadIdx.x; i < n13 + n2; i += kDecThreads)
            jobs[i] = pack_job(i < n13 ? decode_job(R, a0 + i, P.s13.row_blocks)
                                       : decode_job(R, b0 + (i - n13), P.s2.row_blocks));
    if (small) {
        if (warp != kDecWarps) named_bar_sync(2, kPhaseBar);   // the table is written
    } else {
        __syncthreads();
    }

    if (warp == kDecWarps) {
        // ---------------- producer: weights only.  Lane mt copies matrix mt of
        // the job: the signs of all the job's rows as one swizzled tensor box,
        // then four bulk copies (block scales, outlier columns, outlier values,
        // row scales); lane 0 arms the stage's barrier with the job's byte
        // count first (a tensor box always delivers its full size).
        int s = 0, ph = 0;
        for (int i = 0; i < n13 + n2; ++i) {
            int ok_wait = 1;
            if (lane == 0 && i >= P.n_stages) ok_wait = mbar_wait(empty + s, uint32_t(ph ^ 1));
            ok_wait = __shfl_sync(0xffffffffu, ok_wait, 0);
            if (!ok_wait) {
                if (lane == 0) set_status(A.ws.status, GALE_ERR_TIMEOUT);
                break;
            }
            const bool w13 = i < n13;
            const Shape& sh = w13 ? P.s13 : P.s2;
            const Job Jb = w13 ? decode_job(R, a0 + i, P.s13.row_blocks) : decode_job(R, b0 + (i - n13), P.s2.row_blocks);
            const int C = sh.cols, nb = C / 128, k = outliers_per_row(C);
            const int r0 = Jb.tile * sh.job_rows;
            const int R = min(sh.job_rows, sh.rows - r0);
            const bool mine = lane < sh.n_mat;
            const JobTile L = job_tile(C, sh.job_rows);
            uint32_t sz[5] = {0u, 0u, 0u, 0u, 0u};
            const char* src[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
            if (mine) {
                const int64_t off = w13 ? (lane ? A.off_w3 : A.off_w1) : A.off_w2;
                const MatView mv = make_view(A.base + int64_t(Jb.e) * A.stride + off, sh.rows, C);
                const char* qs = reinterpret_cast<const char*>(mv.q) + int64_t(r0) * k / 2;   // r0 is even
                const int qd = int(reinterpret_cast<uintptr_t>(qs) & 15);
                sz[0] = uint32_t(sh.job_rows * (C / 8));
                src[1] = reinterpret_cast<const char*>(mv.s_blk + int64_t(r0) * nb);
                sz[1] = uint32_t(R * (C / 64));
                src[2] = reinterpret_cast<const char*>(mv.idx + int64_t(r0) * k);
                sz[2] = k ? uint32_t(R * k * 2) : 0u;
                src[3] = qs - qd;
                sz[3] = k ? uint32_t((qd + (R * k + 1) / 2 + 15) & ~15) : 0u;
                src[4] = reinterpret_cast<const char*>(mv.s_row + r0);
                sz[4] = uint32_t(R * 2);
            }
            uint32_t tx = sz[0] + sz[1] + sz[2] + sz[3] + sz[4];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tx += __shfl_xor_sync(0xffffffffu, tx, o);
            if (lane == 0) mbar_arrive_expect_tx(full + s, tx);
            __syncwarp();
            if (mine) {
                uint8_t* dst = smem + S.ring + s * P.stage_bytes + lane * sh.mat_bytes;
                tma_load_5d(dst + L.signs, w13 ? &map13 : &map2, full + s, 0, r0, 0, w13 ? lane : 0, Jb.e);
                const int dsto[5] = {L.signs, L.scales, L.idx, L.q, L.srow};
#pragma unroll
                for (int c = 1; c < 5; ++c)
                    if (sz[c]) bulk_load(dst + dsto[c], src[c], sz[c], full + s);
            }
            if (++s == P.n_stages) {
                s = 0;
                ph ^= 1;
            }
        }
        return;
    }

    if (warp == kDecWarps + 1) {
        // ---------------- epilogue warp: once the 8 pieces of a job are in its
        // stage's partial sums, gather them, release the stage and finish the
        // job (h rows in phase 1; o rows and the combine in phase 2), so that
        // the consumers go straight on to the next job
        bool eok = true;
        int s = 0, ph = 0;
#pragma unroll 1
        for (int phase = 0; phase < 2; ++phase) {
            const bool W13 = phase == 0;
            const Shape& sh = W13 ? P.s13 : P.s2;
            const int n_my = W13 ? n13 : n2, ibase = W13 ? 0 : n13;
#pragma unroll 1
            for (int i = 0; i < n_my; ++i) {
                const Job Jb = unpack_job(jobs[ibase + i]);
                if (eok && !mbar_wait(done + s, uint32_t(ph))) {
                    eok = false;
                    if (lane == 0) set_status(A.ws.status, GALE_ERR_TIMEOUT);
                }
                const float* pb = reinterpret_cast<const float*>(smem + S.part) + s * kPartFloats;
                if (eok) epi_rows(A, sh, W13, Jb, pb, lane);
                // the consumers only read the stage, so the barrier alone orders
                // their reads (and these sums) before the next copy into it
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + s);
                if (eok && !W13) epi_combine(A, R, sh, Jb, lane);
                if (++s == P.n_stages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (phase == 0) {
                __threadfence();
                named_bar_sync(2, kPhaseBar);   // this CTA's h rows are written
                named_bar_sync(2, kPhaseBar);   // the grid barrier has been passed
                if (!M.gate_ok) eok = false;
            }
        }
        return;
    }

    // ---------------- consumers
    const int tid = threadIdx.x;   // 0..255
    const int d = A.d_model;
    const int comb_blocks = (d + 63) / 64;
    if (blockIdx.x == 0) {
        // the combine counters start at zero; they are used only after the grid barrier
        for (int i = tid; i < A.B * comb_blocks; i += kDecThreads) A.ws.comb_cnt[i] = 0;
        for (int i = tid; i < A.B; i += kDecThreads) A.ws.tok_cnt[i] = 0;
        if (tid == 0 && R.bad) set_status(A.ws.status, GALE_ERR_ARG);
    }
    uint8_t* cache = smem + S.cache;
    float* scratch = reinterpret_cast<float*>(smem + S.scratch) + warp * kWarpScratchFloats;
    bool ok = true;
    int st = 0, ph = 0;   // ring position of the next job

#pragma unroll 1
    for (int phase = 0; phase < 2; ++phase) {
        const bool W13 = phase == 0;
        const Shape& sh = W13 ? P.s13 : P.s2;
        const int cap = W13 ? P.cap13 : P.cap2;
        const int n_my = W13 ? n13 : n2, ibase = W13 ? 0 : n13;
        const int C = sh.cols, k = outliers_per_row(C);
        // this warp's MMA piece of every job ...
        const int tr = warp / (sh.n_mat * sh.n_chunk);
        const int mat = (warp / sh.n_chunk) % sh.n_mat;
        const int ch = warp % sh.n_chunk;
        // ... and its (matrix, row) pairs of outlier corrections
        const int ppw = sh.pairs / kDecWarps, lpp = 32 / ppw;
        const int pair = warp * ppw + lane / lpp, sub = lane % lpp;
        const int o_mat = pair / sh.job_rows, o_tr = (pair % sh.job_rows) / 16, o_row = pair % 16;
        int pk0 = -2, pk1 = -2, c0 = -1, c1 = -1;

        for (int i = 0; i < n_my; ++i) {
            const Job Jb = unpack_job(jobs[ibase + i]);
            const int key0 = Jb.slot0 < 0 ? -1 : (W13 ? R.slot_tok[Jb.slot0] : Jb.slot0);
            const int key1 = Jb.slot1 < 0 ? -1 : (W13 ? R.slot_tok[Jb.slot1] : Jb.slot1);
            if (key0 != pk0 || key1 != pk1) {   // uniform over the consumers
                ensure_cached(A, sh, cap, cache, M, W13, key0, key1, c0, c1);
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
            const int s = st;
            if (ok && !mbar_wait(full + s, uint32_t(ph))) {
                ok = false;
                if (lane == 0) set_status(A.ws.status, GALE_ERR_TIMEOUT);
            }
            uint8_t* stage = smem + S.ring + s * P.stage_bytes;
            float* pb = reinterpret_cast<float*>(smem + S.part) + s * kPartFloats;
            float part[2] = {0.f, 0.f};
            float corr0 = 0.f, corr1 = 0.f;
            const int r0 = Jb.tile * sh.job_rows + tr * 16;
            const int or0 = Jb.tile * sh.job_rows + o_tr * 16;
            const bool do_mma = ok && r0 < sh.rows, do_out = ok && or0 + o_row < sh.rows && k;
            const JobTile L = job_tile(C, sh.job_rows);
            if (do_mma) {
                const uint8_t* mt_tile = stage + mat * sh.mat_bytes;
                chunk_mma(mt_tile + L.signs + ch * sh.job_rows * 128 + tr * 16 * 128,
                          reinterpret_cast<const __half*>(mt_tile + L.scales) + tr * 16 * (C / 128), C, ch, tok,
                          scratch, part);
            }
            if (do_out) {
                const MatView ov = make_view(A.base + int64_t(Jb.e) * A.stride +
                                                 (W13 ? (o_mat ? A.off_w3 : A.off_w1) : A.off_w2),
                                             sh.rows, C);
                const int q_delta = int(
                    reinterpret_cast<uintptr_t>(reinterpret_cast<const char*>(ov.q) + int64_t(Jb.tile * sh.job_rows) * k / 2) &
                    15);
                row_outliers(stage + o_mat * sh.mat_bytes, L, C, sh.job_rows, k, q_delta, o_tr * 16 + o_row, sub, lpp,
                             tok, corr0, corr1);
            }
            for (int o = 1; o < lpp; o <<= 1) {
                corr0 += __shfl_xor_sync(0xffffffffu, corr0, o);
                corr1 += __shfl_xor_sync(0xffffffffu, corr1, o);
            }
            if (lane < 16) {
                pb[warp * 32 + lane * 2] = part[0];
                pb[warp * 32 + lane * 2 + 1] = part[1];
            }
            if (sub == 0) {
                pb[kDecWarps * 32 + pair * 2] = corr0;
                pb[kDecWarps * 32 + pair * 2 + 1] = corr1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(done + s);
            if (++st == P.n_stages) {
                st = 0;
                ph ^= 1;
            }
        }

        if (phase == 0) {
            // ---------------- grid barrier: h of every expert is in global memory
            __threadfence();
            named_bar_sync(2, kPhaseBar);   // with the epilogue warp: this CTA's phase-1 work is done
            if (tid == 0) {
                M.gate_ok = grid_barrier(A.ws.gbar, G);
                if (!M.gate_ok) set_status(A.ws.status, GALE_ERR_TIMEOUT);
                for (int q = 0; q < kCapMax; ++q) {   // the cache now holds slots of h
                    M.key[q] = -1;
                    M.stamp[q] = 0;
                }
            }
            named_bar_sync(2, kPhaseBar);
            if (!M.gate_ok) ok = false;
        }
    }
}

// Deepest ring that fits the shared-memory budget with at least two cached
// vectors per phase; what is left over goes to the cache.
bool make_plan(const gale_layer& L, int B, int K, Plan& P) {
    constexpr int kBudget = 226 * 1024;
    P.s13 = make_shape(L.d_ff, L.d_model, 2);
    P.s2 = make_shape(L.d_model, L.d_ff, 1);
    // at most B*K token groups; a CTA gets its share of both phases' jobs, rounded up
    const int64_t groups = int64_t(B) * K, G = sm_count();
    P.max_jobs = int((groups * P.s13.row_blocks + G - 1) / G + (groups * P.s2.row_blocks + G - 1) / G);
    P.stage_bytes = P.s13.stage_bytes > P.s2.stage_bytes ? P.s13.stage_bytes : P.s2.stage_bytes;
    const int min_cache = 2 * (P.s13.tok_bytes > P.s2.tok_bytes ? P.s13.tok_bytes : P.s2.tok_bytes);
    for (int st = kMaxStages; st >= 3; --st) {
        P.n_stages = st;
        P.cache_bytes = min_cache;
        const int room = kBudget - dec_smem(P).bytes;
        if (room < 0) continue;
        // the space left grows the cache, up to kCapMax entries of the larger phase
        const int big = P.s13.tok_bytes > P.s2.tok_bytes ? P.s13.tok_bytes : P.s2.tok_bytes;
        const int cap_big = 2 + room / big > kCapMax ? kCapMax : 2 + room / big;
        P.cache_bytes = cap_big * big;
        P.cap13 = P.cache_bytes / P.s13.tok_bytes > kCapMax ? kCapMax : P.cache_bytes / P.s13.tok_bytes;
        P.cap2 = P.cache_bytes / P.s2.tok_bytes > kCapMax ? kCapMax : P.cache_bytes / P.s2.tok_bytes;
        if (dec_smem(P).bytes <= kBudget) return true;
    }
    return false;
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
    w.gbar = w.status + 4;   // a counter inside the status block, zeroed every call
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
    const Shape s2 = make_shape(L.d_model, L.d_ff, 1);
    if (s2.job_rows % 64 != 0 || s2.job_rows > 128) return false;
    Plan P;
    return make_plan(L, B, K, P);
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
    Plan P;
    if (!make_plan(L, B, K, P)) return GALE_ERR_UNSUPPORTED;

    int rc = GALE_OK;
    CUtensorMap map13, map2;
    rc = cached_sign_map5(&map13, A.base + A.off_w1, L.d_ff, L.d_model, 2, A.off_w3 - A.off_w1, L.n_experts,
                          L.expert_stride, P.s13.job_rows);
    if (rc == GALE_OK)
        rc = cached_sign_map5(&map2, A.base + A.off_w2, L.d_model, L.d_ff, 1, A.off_w3 - A.off_w1, L.n_experts,
                              L.expert_stride, P.s2.job_rows);
    if (rc != GALE_OK) return rc;
    const DecSmem S = dec_smem(P);
    rc = ensure_smem(reinterpret_cast<const void*>(moe_decode_kernel), S.bytes);
    if (rc != GALE_OK) return rc;
    // all CTAs resident at once (the grid barrier), one per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(sm_count()));
    cfg.blockDim = dim3(kDecBlock);
    cfg.dynamicSmemBytes = size_t(S.bytes);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_decode_kernel, map13, map2, A, P) == cudaSuccess ? GALE_OK : GALE_ERR_CUDA;
}

}  // namespace gale

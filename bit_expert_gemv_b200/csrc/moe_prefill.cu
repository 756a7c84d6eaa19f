// Prefill path of gale_moe_forward (many tokens per expert): the expert
// products are real dense contractions, run on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM).
//
//   route   : stable counting sort of the (token, slot) pairs by expert
//   jobs    : every expert's slots cut into chunks of 128 tokens
//   gather  : x of every pair, in permuted order, rotated (FWHT-1024) to fp16
//   w1/w3   : per (128-row tile, chunk): the packed signs are expanded in
//             registers to fp16 +-s_blk (exact), the outliers patched in
//             (q * s_row rounded to fp16), and the A operand is written
//             straight into TMEM; the tokens come in by TMA as the B operand;
//             both products accumulate in TMEM; SwiGLU epilogue
//   rotate  : h -> fp16 FWHT-1024
//   w2      : the same tile kernel over pairs of 128-row tiles of w2
//   combine : gate-weighted sum in fixed k order (+ residual, RMSNorm)
//
// A in TMEM keeps the shared-memory traffic to the B operand alone: the
// expansion is paid in instruction issue, the contraction on the tensor pipe.
#include "common.cuh"
#include "fwht.cuh"
#include "moe.cuh"
#include "moe_prefill.cuh"
#include "route.cuh"
#include "tc_prefill.cuh"
#include "tma.cuh"

namespace gale {

namespace {

constexpr int kTcM = 128;           // weight rows per tile (TMEM lanes)
constexpr int kTcK = 64;            // K per stage: one 128-byte row of fp16 tokens
constexpr int kTcStages = 4;
constexpr int kTcExpWarps = 16;     // expander warps: two groups of 8, 2 per TMEM lane quarter each
constexpr int kTcAuxWarps = 4;      // outlier lists of the next job, epilogue of the last one
constexpr int kTcThreads = (2 + kTcExpWarps + kTcAuxWarps) * 32;
constexpr int kMaxOutliers = 82;    // per row: round(0.01 * 8192)
constexpr uint32_t kSentinel = 0xFFFF0000u;

// Every job multiplies two A operands by one token chunk: w1 and w3 over the
// same 128 rows (SwiGLU epilogue), or two consecutive 128-row tiles of w2.
constexpr int kTcChunk = 128;                  // tokens per job (MMA N)
constexpr int kTcAccCols = 2 * kTcChunk;       // fp32 accumulator columns, one block per operand
constexpr int kTcACols = 2 * 32;               // TMEM columns of one A stage (both operands)
static_assert(kTcAccCols + kTcStages * kTcACols <= 512, "TMEM budget");

struct TcJob {
    int e, n0, n;   // expert, first slot of the chunk, tokens in the chunk
};

struct TcArgs {
    const char* base;
    int64_t stride;
    int64_t off_a, off_b;      // byte offsets of the matrices inside a record
    int rows, cols;            // of the streamed matrices
    const TcJob* jobs;
    const int32_t* n_jobs;
    float* out;                // [slots][rows] fp32
    const float* unscale;      // [slots] factor of each slot's fp16 activation tile
    int32_t* status;
};

struct TcSmem {
    int b, idx[2], q[2], srow[2], ent[2][2], start1[2], patch, bars, misc, bytes;
};

// Barriers of the tile kernel, in their shared-memory order.
enum TcBar {
    kBarBFull = 0,                        // [kTcStages] token tile landed
    kBarAFull = kTcStages,                // [kTcStages] A stage expanded (16 warps)
    kBarMmaDone = 2 * kTcStages,          // [kTcStages] the stage's MMAs completed
    kBarAccFull = 3 * kTcStages,          // the job's accumulators are final
    kBarAccEmpty,                         // the epilogue has read them (aux threads)
    kBarSideFull,                         // the job's outlier sections landed
    kBarSideFree,                         // the lists have been built from them (aux threads)
    kBarListReady,                        // [2] lists of a job in buffer b (aux threads)
    kBarListFree = kBarListReady + 2,     // [2] the expanders are done with buffer b
    kTcBars = kBarListFree + 2
};

__host__ __device__ inline int align16(int n) { return (n + 15) & ~15; }

// Shared memory: the token ring; per operand the job's outlier sections (bulk
// copies, one buffer); two buffers of outlier lists (per operand and row: the
// columns of the first and of the second 32-column half of every K-step, each
// list closed by two sentinels, and where the second list starts); the
// expanders' patch areas; barriers.
__host__ __device__ inline TcSmem tc_smem(int k) {
    TcSmem s;
    s.b = 0;
    int o = kTcStages * kTcChunk * 128;
    for (int mt = 0; mt < 2; ++mt) {
        s.idx[mt] = o;
        o += align16(kTcM * k * 2);
        s.q[mt] = o;
        o += align16(kTcM * k / 2 + 1);
        s.srow[mt] = o;
        o += kTcM * 2;
    }
    for (int b = 0; b < 2; ++b) {
        for (int mt = 0; mt < 2; ++mt) {
            s.ent[b][mt] = o;
            o += kTcM * (k + 4) * 4;
        }
        s.start1[b] = o;
        o += 2 * kTcM * 4;
    }
    // per expander warp, 16 words x 32 lanes of patched (outlier) words
    s.patch = o;
    o += kTcExpWarps * 16 * 32 * 4;
    s.bars = (o + 7) & ~7;
    s.misc = s.bars + 8 * kTcBars;
    s.bytes = s.misc + 16 + 1024;   // + slack to align the base to 1024 bytes
    return s;
}

// Tensor-map encoding of the permuted fp16 activations: boxes of 64 columns
// x `box_rows` slots, 128-byte swizzle (the K-major SW128 operand layout).
int act_map(CUtensorMap* m, const void* base, int cols, int64_t rows, int box_rows) {
    return make_map_3d(m, true, base, uint64_t(cols), uint64_t(rows), 1, uint64_t(cols) * 2,
                       uint64_t(cols) * 2 * uint64_t(rows), 64, uint32_t(box_rows), true);
}

// The job list: every expert's slots in chunks of kTcChunk, one thread per expert.
__global__ void __launch_bounds__(1024) prefill_jobs_kernel(const int32_t* counts, const int32_t* offsets, int E,
                                                            TcJob* jobs, int32_t* n_jobs) {
    __shared__ int tmp[32];
    const int e = threadIdx.x;
    const int lane = e & 31, warp = e >> 5;
    const int n_e = e < E ? counts[e] : 0;
    const int c = (n_e + kTcChunk - 1) / kTcChunk;
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (e == 0) {
        int run = 0;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) {
            const int v = tmp[w];
            tmp[w] = run;
            run += v;
        }
        *n_jobs = run;
    }
    __syncthreads();
    const int first = tmp[warp] + incl - c;
    for (int i = 0; i < c; ++i)
        jobs[first + i] = TcJob{e, offsets[e] + i * kTcChunk, min(kTcChunk, n_e - i * kTcChunk)};
}

// fp16 activation tiles carry a power-of-two scale per slot so that no value
// overflows (or falls below the normal range) whatever the size of the input:
// with m the row's largest |value| before the rotation, every rotated value
// is at most 32 m (1/32 times a sum of 1024 terms), so the stored value
// u * 2^k with 32 m 2^k in (2^13, 2^14] fits with room to spare; the tile
// epilogue multiplies its sums by 2^-k (exact).
__device__ __forceinline__ float slot_scale(float m) {
    if (!(m > 0.f) || !(m < 3.0e38f)) return 1.0f;   // zero (or non-finite) rows keep scale 1
    int e;
    frexpf(32.0f * m, &e);                           // 32 m = f 2^e, f in [0.5, 1)
    return ldexpf(1.0f, 14 - e);
}

// Largest |value| of row `src` (bf16 bits or fp32) of length d, all lanes of the warp.
__device__ __forceinline__ float row_absmax(const void* src, bool bf16, int d) {
    const int lane = threadIdx.x & 31;
    float m = 0.f;
    if (bf16) {
        const uint2* p = static_cast<const uint2*>(src);
#pragma unroll 4
        for (int i = lane; i < d / 4; i += 32) {
            const uint2 w = p[i];
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16_to_f32(uint16_t(w.x))), fabsf(bf16_to_f32(uint16_t(w.x >> 16)))),
                               fmaxf(fabsf(bf16_to_f32(uint16_t(w.y))), fabsf(bf16_to_f32(uint16_t(w.y >> 16))))));
        }
    } else {
        const float4* p = static_cast<const float4*>(src);
#pragma unroll 4
        for (int i = lane; i < d / 4; i += 32) {
            const float4 v = __ldcg(p + i);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// x of every pair in permuted order, rotated, as scaled fp16: one warp per
// (token, 1024-block) rotates the block once and writes it to the slot of
// each of the token's routed pairs (pairs with an invalid expert id have no
// slot); the warps of block 0 write the slots' unscaling factors.
__global__ void __launch_bounds__(256) gather_rotate_kernel(const uint16_t* __restrict__ x,
                                                            const int32_t* __restrict__ pos_of_pair, int B, int K,
                                                            int d, __half* __restrict__ y, float* __restrict__ unscale) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
    const int nb = d / 1024;
    if (wid >= int64_t(B) * nb) return;
    const int64_t t = wid / nb;
    const int blk = int(wid - t * nb);
    const float sc = slot_scale(row_absmax(x + t * d, true, d));
    const uint16_t* src = x + t * d + blk * 1024;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = bf16_to_f32(src[32 * i + lane]);
    fwht1024_warp(v, lane);
    __half hv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) hv[i] = __float2half_rn(v[i] * (sc * (1.0f / 32.0f)));
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        const int64_t s = pos_of_pair[t * K + k];
        if (s < 0) continue;
        __half* dst = y + s * d + blk * 1024;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[32 * i + lane] = hv[i];
        if (blk == 0 && lane == 0) unscale[s] = 1.0f / sc;
    }
}

// h of every slot rotated into scaled fp16 (the w2 operand), one warp per
// (slot, 1024-block); the warps of block 0 write the slots' unscaling factors.
__global__ void __launch_bounds__(256) rotate_h_kernel(const float* __restrict__ h, int64_t P, int d,
                                                       __half* __restrict__ y, float* __restrict__ unscale) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
    const int nb = d / 1024;
    if (wid >= P * nb) return;
    const int64_t s = wid / nb;
    const int blk = int(wid - s * nb);
    const float sc = slot_scale(row_absmax(h + s * d, false, d));
    const float* src = h + s * d + blk * 1024;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __ldcg(src + 32 * i + lane);
    fwht1024_warp(v, lane);
    __half* dst = y + s * d + blk * 1024;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[32 * i + lane] = __float2half_rn(v[i] * (sc * (1.0f / 32.0f)));
    if (blk == 0 && lane == 0) unscale[s] = 1.0f / sc;
}

// The 16 fp16 pairs of 32 weights: sign word w (bit c set = column c negative)
// and the block scale's fp16 bits sc.  Pair p holds columns 2p (low half) and
// 2p+1.  Multiplying a byte by 2^(15-2i) + 2^(30-2i) moves its bits 2i and
// 2i+1 to bit positions 15 and 31; the two shifted copies do not overlap, so
// no carry disturbs them.
__device__ __forceinline__ void expand_signs(uint32_t w, uint32_t sc, uint32_t (&v)[16]) {
    const uint32_t h2 = sc * 0x10001u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t b = __byte_perm(w, 0u, 0x4440u + j);
        v[4 * j + 0] = ((b * 0x40008000u) & 0x80008000u) ^ h2;
        v[4 * j + 1] = ((b * 0x10002000u) & 0x80008000u) ^ h2;
        v[4 * j + 2] = ((b * 0x04000800u) & 0x80008000u) ^ h2;
        v[4 * j + 3] = ((b * 0x01000200u) & 0x80008000u) ^ h2;
    }
}

// Persistent tile kernel: CTA c takes the (row tile, job) items c, c + grid,
// ... in order, where a row tile is 128 rows of w1 and w3 (SwiGLU epilogue,
// GLU) or two consecutive 128-row tiles of w2.  Warp 0 streams the outlier
// sections and the token tiles, warp 1 owns TMEM and issues the MMAs, warps
// 2..17 expand weights into TMEM, and warps 18..21 build the outlier lists of
// the next item and write out the accumulators of the last one, so that
// neither sits between two items' K loops.
template <bool GLU>
__global__ void __launch_bounds__(kTcThreads, 1) tc_tile_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs A) {
    constexpr int kRowsPerCta = GLU ? kTcM : 2 * kTcM;   // rows of the streamed matrix per item
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int n_mtiles = A.rows / kRowsPerCta;
    const int n_items = n_mtiles * *A.n_jobs;
    if (int(blockIdx.x) >= n_items) return;
    const int n_my = (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1;   // items of this CTA
    const int nk = A.cols / kTcK;
    const int kout = outliers_per_row(A.cols);
    const TcSmem S = tc_smem(kout);
    // offsets by operand / buffer as selects (an indexed TcSmem would live in local memory)
    auto off_idx = [&](int mt) { return mt ? S.idx[1] : S.idx[0]; };
    auto off_q = [&](int mt) { return mt ? S.q[1] : S.q[0]; };
    auto off_srow = [&](int mt) { return mt ? S.srow[1] : S.srow[0]; };
    auto off_ent = [&](int b, int mt) { return b ? (mt ? S.ent[1][1] : S.ent[1][0]) : (mt ? S.ent[0][1] : S.ent[0][0]); };
    auto off_start1 = [&](int b) { return b ? S.start1[1] : S.start1[0]; };
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S.misc);
    volatile int* fail = reinterpret_cast<volatile int*>(smem + S.misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // item i of this CTA: its row tile and job
    auto item = [&](int i, int& r0, TcJob& job) {
        const int w = int(blockIdx.x) + i * int(gridDim.x);
        const int jid = w / n_mtiles;
        r0 = (w - jid * n_mtiles) * kRowsPerCta;
        job = A.jobs[jid];
    };
    // a bounded wait that gives up at once after any earlier one ran out
    // (the flag is read only when the phase is not complete yet)
    auto wait = [&](int b, uint32_t parity) -> bool {
        if (mbar_try_wait(bar + b, parity)) return true;
        if (*fail) return false;
        if (mbar_wait(bar + b, parity)) return true;
        *fail = 1;
        return false;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(bar + kBarBFull + s, 1);
            mbar_init(bar + kBarAFull + s, kTcExpWarps * 32);
            mbar_init(bar + kBarMmaDone + s, 1);
        }
        mbar_init(bar + kBarAccFull, 1);
        mbar_init(bar + kBarAccEmpty, kTcAuxWarps * 32);
        mbar_init(bar + kBarSideFull, 1);
        mbar_init(bar + kBarSideFree, kTcAuxWarps * 32);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar + kBarListReady + b, kTcAuxWarps * 32);
            mbar_init(bar + kBarListFree + b, kTcExpWarps * 32);
        }
        *fail = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- producer: the outlier sections of item i + 1 once
        // the lists of item i are built, then the token tiles of item i
        if (lane == 0) {
            const uint32_t idx_bytes = uint32_t(kTcM * kout * 2), q_bytes = uint32_t(kTcM * kout / 2);
            auto load_side = [&](int i) {
                int r0;
                TcJob job;
                item(i, r0, job);
                const char* rec = A.base + int64_t(job.e) * A.stride;
                mbar_arrive_expect_tx(bar + kBarSideFull, 2u * (idx_bytes + q_bytes + kTcM * 2));
                for (int mt = 0; mt < 2; ++mt) {
                    const MatView mv = make_view(rec + (mt ? A.off_b : A.off_a), A.rows, A.cols);
                    const int rm = r0 + (GLU ? 0 : mt * kTcM);   // first row of operand mt
                    bulk_load(smem + off_idx(mt), mv.idx + int64_t(rm) * kout, idx_bytes, bar + kBarSideFull);
                    bulk_load(smem + off_q(mt), mv.q + int64_t(rm) * kout / 2, q_bytes, bar + kBarSideFull);
                    bulk_load(smem + off_srow(mt), mv.s_row + rm, kTcM * 2, bar + kBarSideFull);
                }
            };
            load_side(0);
            int sides = 1, gs = 0;
            for (int i = 0; i < n_my; ++i) {
                int r0;
                TcJob job;
                item(i, r0, job);
                if (i + 1 < n_my) {
                    if (!wait(kBarSideFree, uint32_t(i & 1))) break;
                    load_side(i + 1);
                    ++sides;
                }
                bool ok = true;
                for (int ks = 0; ks < nk; ++ks, ++gs) {
                    const int s = gs % kTcStages;
                    if (gs >= kTcStages && !wait(kBarMmaDone + s, uint32_t(((gs / kTcStages) - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar + kBarBFull + s, uint32_t(kTcChunk * 128));
                    tma_load_3d(smem + S.b + s * kTcChunk * 128, &xmap, bar + kBarBFull + s, ks * kTcK, job.n0, 0);
                }
                if (!ok) break;
            }
            // no copy may still be landing when the CTA exits (bounded waits,
            // also after a failure)
            mbar_wait(bar + kBarSideFull, uint32_t((sides - 1) & 1));
            for (int g = gs - kTcStages < 0 ? 0 : gs - kTcStages; g < gs; ++g)
                mbar_wait(bar + kBarBFull + g % kTcStages, uint32_t((g / kTcStages) & 1));
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: item i starts once the epilogue has read
        // the accumulators of item i - 1
        if (lane == 0) {
            int gs = 0;
            for (int i = 0; i < n_my; ++i) {
                int r0;
                TcJob job;
                item(i, r0, job);
                const uint32_t idesc = umma_idesc_f16(kTcM, (job.n + 15) & ~15);
                if (i > 0 && !wait(kBarAccEmpty, uint32_t((i - 1) & 1))) break;
                tc_fence_after();
                bool ok = true;
                for (int ks = 0; ks < nk; ++ks, ++gs) {
                    const int s = gs % kTcStages;
                    const uint32_t par = (gs / kTcStages) & 1;
                    if (!wait(kBarAFull + s, par) || !wait(kBarBFull + s, par)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bst = smem_u32(smem + S.b + s * kTcChunk * 128);
                    const uint32_t ast = tmem + uint32_t(kTcAccCols + s * kTcACols);
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
                        for (int kk = 0; kk < kTcK / 16; ++kk)
                            umma_f16_ts(tmem + uint32_t(mt * kTcChunk), ast + uint32_t(mt * 32 + kk * 8),
                                        umma_desc_sw128(bst + kk * 32), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(bar + kBarMmaDone + s);
                }
                if (!ok) break;
                umma_commit(bar + kBarAccFull);
            }
        }
    } else if (warp < 2 + kTcExpWarps) {
        // ---------------- expanders: two groups of 8 warps; group G expands
        // operand G (w1 / w3, or the first / second 128-row tile of w2) and
        // its thread (row t, half h) the 32 columns of half h of every K-step.
        const int ew = warp - 2;
        const int G = ew >> 3;
        const int quarter = warp & 3;   // TMEM lane quarter this warp may access
        const int h = (ew >> 2) & 1;
        const int t = 32 * quarter + lane;
        const int mt = G;
        const int nb = A.cols / 128;
        const int ng = nk / kTcStages;
        uint32_t* pw = reinterpret_cast<uint32_t*>(smem + S.patch) + ew * 512 + lane;   // this lane's column
        // Sign words and block scales arrive a group of kTcStages K-steps ahead:
        // two 16-byte loads hold the group's words of both halves, one 4-byte
        // load its two block scales; the next item's first group is requested
        // during the last group of the current one.
        auto row_src = [&](int r0, const TcJob& job, const uint4*& wsrc, const uint32_t*& ssrc) {
            const int row = r0 + (GLU ? 0 : mt * kTcM) + t;
            const MatView mv = make_view(A.base + int64_t(job.e) * A.stride + (mt ? A.off_b : A.off_a), A.rows, A.cols);
            wsrc = reinterpret_cast<const uint4*>(mv.signs + int64_t(row) * (A.cols / 32));
            ssrc = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(mv.s_blk) + int64_t(row) * nb);
        };
        const uint4* wsrc;
        const uint32_t* ssrc;
        {
            int r0;
            TcJob job;
            item(0, r0, job);
            row_src(r0, job, wsrc, ssrc);
        }
        uint4 wa = __ldg(wsrc), wb = __ldg(wsrc + 1);
        uint32_t sp = __ldg(ssrc);
        bool ok = true;
        int gg = 0;   // groups expanded so far (all items)
        for (int i = 0; i < n_my; ++i) {
            const int buf = i & 1;
            if (ok && !wait(kBarListReady + buf, uint32_t((i >> 1) & 1))) ok = false;
            // this thread's outliers in column order, as (column << 16 | fp16 value)
            const uint32_t* list = reinterpret_cast<const uint32_t*>(smem + off_ent(buf, mt)) + t * (kout + 4);
            int cur = h ? reinterpret_cast<const int*>(smem + off_start1(buf))[mt * kTcM + t] : 0;
            uint32_t ent = list[cur], nxt = list[cur + 1];
            // the next item's job is read now and used in the last group
            int r0n = 0;
            TcJob jn{};
            if (i + 1 < n_my) item(i + 1, r0n, jn);
            const uint4* wsrc_n = wsrc;
            const uint32_t* ssrc_n = ssrc;
            for (int g = 0; g < ng; ++g, ++gg) {
                const uint32_t wg[kTcStages] = {h ? wa.y : wa.x, h ? wa.w : wa.z, h ? wb.y : wb.x, h ? wb.w : wb.z};
                const uint32_t sg[2] = {sp & 0xFFFFu, sp >> 16};
                if (g + 1 < ng) {
                    wa = __ldg(wsrc + 2 * (g + 1));
                    wb = __ldg(wsrc + 2 * (g + 1) + 1);
                    sp = __ldg(ssrc + g + 1);
                } else if (i + 1 < n_my) {
                    row_src(r0n, jn, wsrc_n, ssrc_n);
                    wa = __ldg(wsrc_n);
                    wb = __ldg(wsrc_n + 1);
                    sp = __ldg(ssrc_n);
                }
#pragma unroll
                for (int s = 0; s < kTcStages; ++s) {
                    if (ok && gg > 0 && !wait(kBarMmaDone + s, uint32_t((gg - 1) & 1))) ok = false;
                    tc_fence_after();
                    const int lo = (g * kTcStages + s) * kTcK + 32 * h, hi = lo + 32;
                    const uint32_t w = wg[s], sc = sg[s >> 1];
                    uint32_t v[16];
                    expand_signs(w, sc, v);
                    // outliers of this range replace their weights: each lane
                    // walks its own entries (the next one already loaded),
                    // parks the patched words in its column of the warp's
                    // patch area and marks them; a predicated load per word
                    // then takes them in, with no per-outlier select over the
                    // sixteen words
                    uint32_t m = 0u;
                    int prev_p = -1;
                    uint32_t prev_a = 0u;
                    while (int(ent >> 16) < hi) {
                        const int u = int(ent >> 16) - lo;
                        const int P = u >> 1;
                        const uint32_t val = ent & 0xFFFFu;
                        uint32_t other = sc ^ (((w >> (u ^ 1)) & 1u) << 15);
                        if (P == prev_p) other = (u & 1) ? (prev_a & 0xFFFFu) : (prev_a >> 16);
                        const uint32_t a = (u & 1) ? (other | (val << 16)) : (val | (other << 16));
                        prev_p = P;
                        prev_a = a;
                        pw[P * 32] = a;
                        m |= 1u << P;
                        ent = nxt;
                        nxt = list[++cur + 1];
                    }
#pragma unroll
                    for (int p = 0; p < 16; ++p)
                        if ((m >> p) & 1u) v[p] = pw[p * 32];
                    __syncwarp();
                    tmem_st16(tmem + (uint32_t(32 * quarter) << 16) +
                                  uint32_t(kTcAccCols + s * kTcACols + mt * 32 + 16 * h),
                              v);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar + kBarAFull + s);
                }
            }
            mbar_arrive(bar + kBarListFree + buf);   // the lists of item i are no longer read
            wsrc = wsrc_n;
            ssrc = ssrc_n;
        }
    } else {
        // ---------------- aux warps: thread t owns row t of both operands.
        // Step i builds the outlier lists of item i, then writes out the
        // accumulators of item i - 1.
        const int quarter = warp & 3;   // TMEM lane quarter this warp may access
        const int t = 32 * quarter + lane;
        for (int i = 0; i <= n_my; ++i) {
            if (i < n_my) {
                const int buf = i & 1;
                bool ok = wait(kBarSideFull, uint32_t(i & 1));
                if (ok && i >= 2) ok = wait(kBarListFree + buf, uint32_t(((i >> 1) - 1) & 1));
                if (ok) {
                    for (int mt = 0; mt < 2; ++mt) {
                        // the columns of the first 32-column half of every K-step
                        // (bit 5 clear), then those of the second half
                        const uint16_t* sidx = reinterpret_cast<const uint16_t*>(smem + off_idx(mt)) + t * kout;
                        const uint8_t* sqv = smem + off_q(mt);
                        const float srow = __half2float(reinterpret_cast<const __half*>(smem + off_srow(mt))[t]);
                        uint32_t* list = reinterpret_cast<uint32_t*>(smem + off_ent(buf, mt)) + t * (kout + 4);
                        int n0 = 0;
                        for (int j = 0; j < kout; ++j) n0 += ((sidx[j] >> 5) & 1) == 0;
                        int o0 = 0, o1 = n0 + 2;
                        for (int j = 0; j < kout; ++j) {
                            const int c = sidx[j];
                            const int n = t * kout + j;
                            const int byte = sqv[n >> 1];
                            int qv = (n & 1) ? (byte >> 4) : (byte & 0xF);
                            qv = qv >= 8 ? qv - 16 : qv;
                            const uint32_t e = (uint32_t(c) << 16) | __half_as_ushort(__float2half_rn(float(qv) * srow));
                            if ((c >> 5) & 1) list[o1++] = e;
                            else list[o0++] = e;
                        }
                        list[n0] = kSentinel;
                        list[n0 + 1] = kSentinel;
                        list[kout + 2] = kSentinel;
                        list[kout + 3] = kSentinel;
                        reinterpret_cast<int*>(smem + off_start1(buf))[mt * kTcM + t] = n0 + 2;
                    }
                }
                mbar_arrive(bar + kBarSideFree);
                mbar_arrive(bar + kBarListReady + buf);
            }
            if (i >= 1) {
                int r0;
                TcJob job;
                item(i - 1, r0, job);
                const int n_mma = (job.n + 15) & ~15;
                const bool ok = __all_sync(0xffffffffu, wait(kBarAccFull, uint32_t((i - 1) & 1)));
                tc_fence_after();
                if (ok) {
                    const int ra = r0 + t, rb = r0 + kTcM + t;   // rows of the two accumulators (two w2 tiles)
                    for (int col = 0; col < n_mma; col += 16) {
                        float v1[16], v3[16];
                        tmem_ld16(tmem + (uint32_t(32 * quarter) << 16) + uint32_t(col), v1);
                        tmem_ld16(tmem + (uint32_t(32 * quarter) << 16) + uint32_t(kTcChunk + col), v3);
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int j = col + k;
                            if (j < job.n) {
                                float* o = A.out + int64_t(job.n0 + j) * A.rows;
                                const float u = __ldg(A.unscale + job.n0 + j);
                                const float a1 = v1[k] * u, a3 = v3[k] * u;
                                if (GLU) {
                                    o[ra] = __fdividef(a1, 1.0f + __expf(-a1)) * a3;
                                } else {
                                    o[ra] = a1;
                                    o[rb] = a3;
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(bar + kBarAccEmpty);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *fail) set_status(A.status, GALE_ERR_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <bool GLU>
int launch_tc(const CUtensorMap& map, const TcArgs& a, int max_jobs, cudaStream_t st) {
    const TcSmem S = tc_smem(outliers_per_row(a.cols));
    int rc = ensure_smem(reinterpret_cast<const void*>(tc_tile_kernel<GLU>), S.bytes);
    if (rc != GALE_OK) return rc;
    const int64_t items = int64_t(a.rows / (GLU ? kTcM : 2 * kTcM)) * max_jobs;   // at most
    const int grid = int(items < sm_count() ? items : sm_count());
    if (grid == 0) return GALE_OK;
    tc_tile_kernel<GLU><<<grid, kTcThreads, S.bytes, st>>>(map, a);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

}  // namespace

PrefillWs carve_prefill_ws(void* ws, const gale_layer& L, int B, int K) {
    PrefillWs w{};
    char* p = static_cast<char*>(ws);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        char* q = p ? p + o : nullptr;
        o = align_up(o + bytes, 256);
        return q;
    };
    const int64_t P = int64_t(B) * K, dm = L.d_model, df = L.d_ff;
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.counts = reinterpret_cast<int32_t*>(take(4 * int64_t(L.n_experts)));
    w.offsets = reinterpret_cast<int32_t*>(take(4 * (int64_t(L.n_experts) + 1)));
    w.perm = reinterpret_cast<int32_t*>(take(4 * P));
    w.pos_of_pair = reinterpret_cast<int32_t*>(take(4 * P));
    w.route_scratch = take(int64_t(route_grid_scratch_bytes(B, K, L.n_experts)));
    w.max_jobs = int(L.n_experts + P / kTcChunk + 1);
    w.jobs = take(int64_t(sizeof(TcJob)) * w.max_jobs);
    w.n_jobs = reinterpret_cast<int32_t*>(take(8));
    w.x16 = reinterpret_cast<__half*>(take(2 * P * dm));
    w.x_unscale = reinterpret_cast<float*>(take(4 * P));
    w.h_unscale = reinterpret_cast<float*>(take(4 * P));
    w.h = reinterpret_cast<float*>(take(4 * P * df));
    w.h16 = reinterpret_cast<__half*>(take(2 * P * df));
    w.o = reinterpret_cast<float*>(take(4 * P * dm));
    w.scratch = reinterpret_cast<float*>(take(4 * int64_t(B) * dm));
    w.bytes = size_t(o);
    return w;
}

bool prefill_supported(const gale_layer& L, int B, int K) {
    if (int64_t(B) * K > (int64_t(1) << 24) || L.n_experts > 1024) return false;
    // the expanders walk K in groups of one pass over the stage ring
    if (L.d_model % (kTcK * kTcStages) != 0 || L.d_ff % (kTcK * kTcStages) != 0) return false;
    // a tile's outlier lists stay in shared memory
    const int k1 = outliers_per_row(L.d_model), k2 = outliers_per_row(L.d_ff);
    // w2 goes by pairs of 128-row tiles
    return k1 <= kMaxOutliers && k2 <= kMaxOutliers && tc_smem(k1).bytes <= 227 * 1024 &&
           tc_smem(k2).bytes <= 227 * 1024 && L.d_model % (2 * kTcM) == 0;
}

int launch_moe_prefill(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                       void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st) {
    PrefillWs w = carve_prefill_ws(ws, L, B, K);
    const int64_t P = int64_t(B) * K;
    GALE_CUDA_TRY(cudaMemsetAsync(w.pos_of_pair, 0xFF, size_t(P) * 4, st));
    RouteArgs ra{};
    ra.ids = ids;
    ra.B = B;
    ra.K = K;
    ra.E = L.n_experts;
    ra.counts = w.counts;
    ra.offsets = w.offsets;
    ra.perm = w.perm;
    ra.pos_of_pair = w.pos_of_pair;
    ra.status = w.status;
    int rc = launch_route_permute_grid(ra, w.route_scratch, st);
    if (rc != GALE_OK) return rc;
    prefill_jobs_kernel<<<1, 1024, 0, st>>>(w.counts, w.offsets, L.n_experts, static_cast<TcJob*>(w.jobs), w.n_jobs);
    GALE_LAUNCH_CHECK();
    {
        const int64_t warps = int64_t(B) * (L.d_model / 1024);
        gather_rotate_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, st>>>(x, w.pos_of_pair, B, K, L.d_model,
                                                                                  w.x16, w.x_unscale);
        GALE_LAUNCH_CHECK();
    }
    const int64_t l1 = make_layout(L.d_ff, L.d_model).total;
    CUtensorMap xm;
    rc = act_map(&xm, w.x16, L.d_model, P, kTcChunk);
    if (rc != GALE_OK) return rc;
    TcArgs a{};
    a.base = static_cast<const char*>(L.base);
    a.stride = L.expert_stride;
    a.status = w.status;
    // w1 / w3 + SwiGLU
    a.jobs = static_cast<const TcJob*>(w.jobs);
    a.n_jobs = w.n_jobs;
    a.off_a = 0;
    a.off_b = l1;
    a.rows = L.d_ff;
    a.cols = L.d_model;
    a.out = w.h;
    a.unscale = w.x_unscale;
    rc = launch_tc<true>(xm, a, w.max_jobs, st);
    if (rc != GALE_OK) return rc;
    // rotate h into scaled fp16
    {
        const int64_t warps = P * (L.d_ff / 1024);
        rotate_h_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, st>>>(w.h, P, L.d_ff, w.h16, w.h_unscale);
        GALE_LAUNCH_CHECK();
    }
    CUtensorMap hm;
    rc = act_map(&hm, w.h16, L.d_ff, P, kTcChunk);
    if (rc != GALE_OK) return rc;
    // w2: two 128-row tiles per CTA, the same 128-slot chunks as w1/w3
    a.off_a = 2 * l1;
    a.off_b = 2 * l1;
    a.rows = L.d_model;
    a.cols = L.d_ff;
    a.out = w.o;
    a.unscale = w.h_unscale;
    rc = launch_tc<false>(hm, a, w.max_jobs, st);
    if (rc != GALE_OK) return rc;
    return launch_moe_combine(w.o, w.pos_of_pair, gates, x, B, K, L.d_model, out, out_dtype, fuse_norm, eps,
                              w.scratch, st);
}

}  // namespace gale

// Decode path of gale_moe_forward: the routed-expert layer for batches of up
// to 384 (token, expert) pairs as one persistent kernel, one CTA per SM,
// launched cooperatively (all CTAs resident: CTAs wait on each other's h).
// The same kernel runs a stack of layers (gale_moe_chain): it loops over the
// layers, each with its own counters, and starts layer l + 1 once every
// token's output of layer l (its input) has been written.
//
// Work.  The (token, k) pairs are grouped by expert, stable in pair order,
// and every expert's pairs are cut into segments of at most two (one MMA
// column group).  A unit is
//   phase 1: (segment, 16 rows of w1 and the same 16 rows of w3), full width;
//   phase 2: (segment, 64 rows of w2), full width.
// Each phase's unit list is cut into one contiguous range per CTA.
//
// Roles inside a CTA (15 consumer warps and one producer warp):
//  - producer: streams the packed rows of the CTA's units, phase 1 then
//    phase 2, into a ring of stages: the sign rows as one TMA tensor box with
//    128-byte swizzle, block scales, row scales, outlier columns and values
//    as bulk copies.  It waits only for a stage to be released, so the w2 rows
//    arrive while w1/w3 are still being computed; at batch 1 the ring holds
//    nearly a CTA's whole share of the layer.
//  - consumers: take pieces from one queue in unit order.  A unit has one
//    piece per (1024-column chunk, 32 rows) on the int8 tensor cores and two
//    outlier pieces.  The warp that finishes a unit's last piece sums the
//    partial sums in a fixed order and writes the rows:
//      phase 1: h = silu(w1 x) * (w3 x) into the workspace, then counts the
//               tile into the readiness counter of its (segment, 1024-block);
//      phase 2: the expert outputs o, then counts the unit into the
//               (token, 64-row block) counter; the last of a token's experts
//               sums the K outputs in fixed k order with the gates, and with
//               the fused norm the last block of a token applies the residual
//               and RMSNorm.
//    Activations (x in phase 1, h in phase 2) are rotated by the blocked
//    FWHT-1024 into one of two slots by the consumer warps, one group of
//    segments at a time: consecutive phase-1 segments with the same tokens
//    share a slot (at batch 1 a CTA rotates x once).  A phase-2 slot waits
//    until the segment's h blocks are complete in every CTA.
//
// Arithmetic of a tile (mma.sync m16n8k32, s8 x u8, exact int32 sums).  For
// row r and a 128-column block b,  sum_c sign(r,c) x_c = X_b - 2 P_b  with
// P_b = sum_{c in b, bit(r,c)=1} x_c.  A sign word w of 32 columns gives the
// A operand of bit position s as w & (0x01010101 << s), whose bytes are
// bit * a(s), a(s) = 2^s for s < 7 and -128 for s = 7.  Each 1024-block of an
// activation is held in fixed point, X_c = round(u_c S / a(c mod 8)) with u
// the unnormalised transform and S a power of two such that |u S| <= 2^20;
// Y_c = X_c + 2^20 (0 <= Y_c <= 2^21) is stored as three unsigned bytes, one
// MMA column per byte and token, plus a column of ones that counts
// sum a(s) bit, so that the 2^20 offset cancels exactly in int32.  The block
// sums X_b are exact integers of the same values.  The outlier corrections
// (q s_row - sign s_blk) x_c read x_c from an fp16 copy of u S / 64
// (per-block scale, so it cannot overflow).
//
// Code size matters here: code run once per launch is fetched cold, so the
// helpers are single out-of-line copies with rolled loops.
#include <cuda_bf16.h>

#include "common.cuh"
#include "moe_stream.cuh"
#include "ptx.cuh"
#include "tma.cuh"

namespace gale {

namespace {

constexpr int kCW = 15;                       // consumer warps (16 warps in all: 128 registers each)
constexpr int kThreads = (kCW + 1) * 32;      // + the producer warp
constexpr int kSegTok = 2;                    // pairs per segment
constexpr int kMaxStages = 12;
constexpr int kMaxLocalSeg = 64;
constexpr int kSmemBytes = 227 * 1024;
constexpr int kR1 = 16;                       // rows of w1 (and of w3) per phase-1 unit
constexpr int kR2 = 64;                       // rows of w2 per phase-2 unit
constexpr int kPartBytes = 192 * kSegTok * 4; // partial sums of a stage: 192 rows x 2 tokens
constexpr uint64_t kWaitNs = 2000000000ull;   // default bound of every wait

// Division by a run-time constant d >= 2 as a multiply-high: exact for
// n * d < 2^32 (n below 2^23 here, d at most a few hundred).
struct FastDiv {
    uint32_t d, m;
};
__host__ __device__ inline FastDiv make_div(uint32_t d) {
    return FastDiv{d, uint32_t((0x100000000ull + d - 1) / d)};
}
__device__ __forceinline__ int fdiv(int n, FastDiv f) { return int(__umulhi(uint32_t(n), f.m)); }

struct StreamArgs {
    const char* base;
    int64_t stride;
    int E, d_model, d_ff, B, K;
    int64_t off_w[3];       // w1, w3, w2 inside a record
    const uint16_t* x;
    const int32_t* ids;
    const float* gates;
    void* out;
    int out_dtype, fuse_norm;
    float eps;
    uint64_t wait_ns;       // bound of every wait
    int withhold_cta;       // failure-path testing: this CTA never counts its h tiles (-1: none)
    int n_layers;           // layers of a chain (1: one layer)
    int64_t layer_experts;  // expert records between consecutive layers
    int64_t e_off;          // first expert record of the current layer
    int32_t* xready;        // tokens of the current layer whose output is written
    const float* xf;        // fp32 activations in place of x (one expert's forward), or null
    int fixed_e;            // >= 0: every token's one pair is this expert with gate 1 (ids and gates unused)
    StreamWs ws;
};

// Byte offsets inside a stage for each phase (the rest of the stage after
// the data is the partial-sum area).
struct StageMap {
    int sb, sr, idx, q;     // block scales, row scales, outlier columns, values
    int sb_bytes;           // block scales of one matrix
    int idx_bytes;          // outlier columns of one matrix
    int q_bytes;            // room for the values of one matrix
};

// Activation layout of one token in a slot (bytes): digits [cols/128][3][4][32],
// int32 128-block sums, fp32 1024-block factors sigma = 1/(32 S), fp16 copy of
// u S / 64 in column order, fp32 factors 2 / S of that copy.
struct TokMap {
    int xsum, sig, x16, f16, bytes;
};

struct Plan {
    int C1, C2;                  // columns of w1/w3 (d_model) and of w2 (d_ff)
    int nch1, nch2;              // 1024-column chunks
    int k1, k2;                  // outliers per row
    int tiles1, tiles2;          // units per segment in each phase
    int pp1, pp2;                // pieces per unit
    TokMap t1, t2;
    StageMap m1, m2;
    int part;                    // partial area offset in a stage
    int stage_bytes;
    Layout L1, L2;
    FastDiv dt1, dt2, dpp1, dpp2;   // division by tiles1, tiles2, pp1, pp2
};

__host__ __device__ inline int align_i(int n, int a) { return (n + a - 1) / a * a; }


__host__ __device__ inline TokMap make_tokmap(int C) {
    TokMap t;
    t.xsum = 3 * C;
    t.sig = t.xsum + C / 32;
    t.x16 = align_i(t.sig + 4 * (C / 1024), 16);
    t.f16 = t.x16 + 2 * C;
    t.bytes = align_i(t.f16 + 4 * (C / 1024), 128);
    return t;
}

__host__ __device__ inline Plan make_stream_plan(int d_model, int d_ff) {
    Plan p{};
    p.C1 = d_model;
    p.C2 = d_ff;
    p.nch1 = d_model / 1024;
    p.nch2 = d_ff / 1024;
    p.k1 = outliers_per_row(d_model);
    p.k2 = outliers_per_row(d_ff);
    p.tiles1 = d_ff / kR1;
    p.tiles2 = d_model / kR2;
    p.pp1 = p.nch1 + 2;
    p.pp2 = 2 * p.nch2 + 2;
    p.t1 = make_tokmap(d_model);
    p.t2 = make_tokmap(d_ff);
    // phase 1: signs [mat 2][chunk][16 rows][128 B]
    p.m1.sb_bytes = kR1 * (p.C1 / 64);
    p.m1.idx_bytes = kR1 * p.k1 * 2;
    p.m1.q_bytes = align_i(kR1 * p.k1 / 2, 16) + 16;
    p.m1.sb = 2 * p.nch1 * 2048;
    p.m1.sr = p.m1.sb + 2 * p.m1.sb_bytes;
    p.m1.idx = p.m1.sr + 2 * 32;
    p.m1.q = p.m1.idx + 2 * align_i(p.m1.idx_bytes, 16);
    const int end1 = p.m1.q + 2 * p.m1.q_bytes;
    // phase 2: signs [chunk][64 rows][128 B]
    p.m2.sb_bytes = kR2 * (p.C2 / 64);
    p.m2.idx_bytes = kR2 * p.k2 * 2;
    p.m2.q_bytes = align_i(kR2 * p.k2 / 2, 16) + 16;
    p.m2.sb = p.nch2 * kR2 * 128;
    p.m2.sr = p.m2.sb + p.m2.sb_bytes;
    p.m2.idx = p.m2.sr + align_i(kR2 * 2, 16);
    p.m2.q = p.m2.idx + align_i(p.m2.idx_bytes, 16);
    const int end2 = p.m2.q + p.m2.q_bytes;
    p.part = align_i(end1 > end2 ? end1 : end2, 128);
    p.stage_bytes = align_i(p.part + kPartBytes, 1024);
    p.L1 = make_layout(d_ff, d_model);
    p.L2 = make_layout(d_model, d_ff);
    p.dt1 = make_div(uint32_t(p.tiles1));
    p.dt2 = make_div(uint32_t(p.tiles2));
    p.dpp1 = make_div(uint32_t(p.pp1));
    p.dpp2 = make_div(uint32_t(p.pp2));
    return p;
}

// Shared control block.
struct Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    int next_piece;
    int abort;
    int stage_done[kMaxStages];
    int slot_grp[2];       // group of segments held (or being built) by each slot
    int slot_claim[2];     // (group << 16) | activation pieces claimed for that group
    int slot_done[2];      // and finished
    int n_valid, n_seg, bad;
    int nmax;                    // most pairs in one segment (sizes the slots)
    int u1b, u1e, u2b, u2e;      // this CTA's unit ranges (global unit indices)
    int s1b, s2b, nl1, nl, ngrp; // first segment of each range, local segments of phase 1, in all; groups
    int stages, slot_bytes, ring;
    FastDiv dst;                 // division by stages
    int issued;                  // units whose copies the producer issued (all layers)
    int ubase;                   // units of this CTA in the layers before the current one
    uint64_t wait_ns;            // bound of every wait
    int grp_of[kMaxLocalSeg];    // group of each local segment
    int grp_seg[kMaxLocalSeg];   // the local segment whose pairs define each group
    int grp_left[kMaxLocalSeg];  // units of each group not finished yet
    int sorted[kDecodeMaxPairsStream];   // pair index at each sorted position
    int seg[kDecodeMaxPairsStream];      // packed (expert << 12) | (first << 3) | n
    uint32_t vmask[kDecodeMaxPairsStream];  // per token: bit k = pair (t, k) valid
    int wsum[32];
};

__device__ __forceinline__ int seg_e(int s) { return s >> 12; }
__device__ __forceinline__ int seg_first(int s) { return (s >> 3) & 511; }
__device__ __forceinline__ int seg_n(int s) { return s & 7; }

__device__ __forceinline__ float h2f(uint32_t bits) { return __half2float(__ushort_as_half(uint16_t(bits))); }

__device__ __forceinline__ float lds_f32(uint32_t addr) { return __uint_as_float(lds_u32(addr)); }
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) { sts_u32(addr, __float_as_uint(v)); }

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int vload(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Bounded waits that leave the issue slots to the warps doing work: a
// shared-memory counter of this CTA or a global counter of other CTAs is
// re-read after a short sleep; an mbarrier phase is awaited with the
// hardware's suspend hint.  Each returns false on abort or after `limit` ns.
__device__ __noinline__ bool wait_smem(const int* p, int v, bool eq, const int* abort, uint64_t limit) {
    unsigned ns = 64;
    uint64_t t0 = 0;
#pragma unroll 1
    for (int it = 0;; ++it) {
        const int x = vload(p);
        if (eq ? x == v : x >= v) return true;
        if (vload(abort)) return false;
        if (it == 0) t0 = globaltimer_ns();
        else if (globaltimer_ns() - t0 > limit) return false;
        __nanosleep(ns);
        if (ns < 512) ns <<= 1;
    }
}

__device__ __noinline__ bool wait_global(const int32_t* p, int v, const int* abort, uint64_t limit) {
    unsigned ns = 64;
    uint64_t t0 = 0;
#pragma unroll 1
    for (int it = 0;; ++it) {
        if (ld_acquire(p) >= v) return true;
        if (vload(abort)) return false;
        if (it == 0) t0 = globaltimer_ns();
        else if (globaltimer_ns() - t0 > limit) return false;
        __nanosleep(ns);
        if (ns < 512) ns <<= 1;
    }
}

__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, uint64_t limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity))
        if (globaltimer_ns() - t0 > limit) return false;
    return true;
}

// a(s) of bit position s inside a byte of a sign word
__device__ __forceinline__ int a_of(int s) { return s < 7 ? (1 << s) : -128; }

// ----------------------------------------------------------------------------
// routing and the CTA's plan (every thread of the CTA)
// ----------------------------------------------------------------------------

// Routing scratch (expert id and sort key of every pair) lives at the end of
// shared memory, which the ring reaches only after the plan is made.
struct RouteScratch {
    int ids[kDecodeMaxPairsStream];
    int key[kDecodeMaxPairsStream];
};
constexpr int kScratchOff = kSmemBytes - 1024 - int(sizeof(RouteScratch));

// Runs once per launch on the critical path before the first copy, so the
// code stays short and rolled (it is fetched cold).  Up to 32 pairs, one warp
// routes with shuffles alone; larger batches use the whole block.
__device__ void route_and_plan(const StreamArgs& A, const Plan& P, Ctl& c, RouteScratch& rs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BK = A.B * A.K, K = A.K;
    if (tid < kMaxLocalSeg) c.grp_left[tid] = 0;
    if (tid == 32) {
        c.wait_ns = A.wait_ns;
        c.next_piece = 0;
        c.slot_grp[0] = 0;
        c.slot_grp[1] = 1;
        c.slot_claim[0] = 0 << 16;
        c.slot_claim[1] = 1 << 16;
        c.slot_done[0] = c.slot_done[1] = 0;
        // slots for the tokens of the largest possible segment: the ring keeps
        // its number of stages across the layers of a chain
        c.nmax = A.B < kSegTok ? A.B : kSegTok;
    }
    if (BK <= 32) {
        if (warp == 0) {
            const int p = lane;
            const int e = p < BK ? (A.fixed_e >= 0 ? A.fixed_e : __ldg(A.ids + p)) : -1;
            if (lane < A.B) c.vmask[lane] = 0u;
            const int t = p / K, k = p - t * K;
            bool valid = p < BK && e >= 0 && e < A.E;
#pragma unroll 1
            for (int j = 1; j < K; ++j) {
                const int ej = __shfl_sync(0xffffffffu, e, (p - j) & 31);
                if (j <= k && ej == e) valid = false;   // a repeated id drops the later pair
            }
            const int key = valid ? (e << 9) | p : 0x7FFFFFFF;
            int r = 0;
#pragma unroll 1
            for (int q = 0; q < 32; ++q) r += __shfl_sync(0xffffffffu, key, q) < key;
            __syncwarp();
            if (valid) {
                atomicOr(&c.vmask[t], 1u << k);
                c.sorted[r] = p;
            }
            const unsigned vb = __ballot_sync(0xffffffffu, valid);
            const int nv = __popc(vb);
            const unsigned bad = __ballot_sync(0xffffffffu, p < BK && !valid);
            if (lane == 0) c.bad = bad != 0u;
            __syncwarp();
            // sorted position `lane`: its expert, run starts and segments of two
            const int sp = lane < nv ? c.sorted[lane] : 0;
            const int se = __shfl_sync(0xffffffffu, e, sp);
            const int prev = __shfl_up_sync(0xffffffffu, se, 1);
            const unsigned rsb = __ballot_sync(0xffffffffu, lane < nv && (lane == 0 || prev != se));
            const unsigned le = (2u << lane) - 1u;   // lanes <= this one
            const int rstart = 31 - __clz(rsb & le);
            const unsigned later = rsb & ~le;
            const int rend = later ? __ffs(later) - 1 : nv;
            const bool start = lane < nv && ((lane - rstart) % kSegTok) == 0;
            const unsigned sgb = __ballot_sync(0xffffffffu, start);
            const int sn = start ? min(kSegTok, rend - lane) : 0;
            if (start) c.seg[__popc(sgb & (le >> 1))] = (se << 12) | (lane << 3) | sn;
            if (lane == 0) {
                c.n_valid = nv;
                c.n_seg = __popc(sgb);
            }
        }
    } else {
        if (tid < A.B) c.vmask[tid] = 0u;
        if (tid < BK) rs.ids[tid] = A.fixed_e >= 0 ? A.fixed_e : __ldg(A.ids + tid);
        if (tid == 0) {
            c.n_valid = 0;
            c.bad = 0;
        }
        __syncthreads();
        bool valid = false;
        if (tid < BK) {
            const int e = rs.ids[tid];
            const int t = tid / K, k = tid - t * K;
            valid = e >= 0 && e < A.E;
#pragma unroll 1
            for (int j = tid - k; j < tid; ++j)
                if (rs.ids[j] == e) valid = false;   // a repeated id drops the later pair
            rs.key[tid] = valid ? (e << 9) | tid : 0x7FFFFFFF;
            if (valid) atomicOr(&c.vmask[t], 1u << k);
            else c.bad = 1;
        }
        const unsigned vb = __ballot_sync(0xffffffffu, valid);
        if (lane == 0 && vb) atomicAdd(&c.n_valid, __popc(vb));
        __syncthreads();
        if (valid) {
            const int k = rs.key[tid];
            int r = 0;
#pragma unroll 1
            for (int j = 0; j < BK; ++j) r += rs.key[j] < k;
            c.sorted[r] = tid;
        }
        __syncthreads();
        // segments: every kSegTok pairs of an expert's run; the run of the pair
        // at sorted position tid starts at lo and the segment ends before hi
        const int nv = c.n_valid;
        bool start = false;
        int packed = 0;
        if (tid < nv) {
            const int e = rs.ids[c.sorted[tid]];
            int lo = tid, hi = tid + 1;
#pragma unroll 1
            while (lo > 0 && rs.ids[c.sorted[lo - 1]] == e) --lo;
#pragma unroll 1
            while (hi < nv && rs.ids[c.sorted[hi]] == e && hi - tid < kSegTok) ++hi;
            start = (tid - lo) % kSegTok == 0;
            packed = (e << 12) | (tid << 3) | (hi - tid);
        }
        const unsigned sb = __ballot_sync(0xffffffffu, start);
        if (lane == 0) c.wsum[warp] = __popc(sb);
        __syncthreads();
        if (start) {
            int sid = __popc(sb & ((1u << lane) - 1u));
#pragma unroll 1
            for (int w = 0; w < warp; ++w) sid += c.wsum[w];
            c.seg[sid] = packed;
        }
        if (tid == 0) {
            int ns = 0;
#pragma unroll 1
            for (int w = 0; w < kThreads / 32; ++w) ns += c.wsum[w];
            c.n_seg = ns;
        }
    }
    __syncthreads();
    if (tid == 0) {
        // every unit costs the same (a segment is one MMA column group): the
        // CTA's ranges are equal shares of each phase's unit list
        const unsigned G = gridDim.x, i = blockIdx.x;
        const unsigned n1 = unsigned(c.n_seg * P.tiles1), n2 = unsigned(c.n_seg * P.tiles2);
        c.u1b = int(n1 * i / G);
        c.u1e = int(n1 * (i + 1) / G);
        c.u2b = int(n2 * i / G);
        c.u2e = int(n2 * (i + 1) / G);
        c.s1b = c.u1b / P.tiles1;
        c.s2b = c.u2b / P.tiles2;
        const int nl1 = c.u1e > c.u1b ? (c.u1e - 1) / P.tiles1 - c.s1b + 1 : 0;
        const int nl2 = c.u2e > c.u2b ? (c.u2e - 1) / P.tiles2 - c.s2b + 1 : 0;
        c.nl1 = nl1;
        c.nl = nl1 + nl2;
        if (c.nl > kMaxLocalSeg) {
            c.abort = 1;
            c.nl = kMaxLocalSeg;
        }
        // groups: consecutive phase-1 segments with the same tokens share one slot
        int g = -1, prev_t0 = -1, prev_t1 = -1;
#pragma unroll 1
        for (int q = 0; q < c.nl; ++q) {
            const bool p1 = q < nl1;
            const int s2 = p1 ? c.s1b + q : c.s2b + (q - nl1);
            const int sg = c.seg[s2];
            const int n = seg_n(sg), f = seg_first(sg);
            const int t0 = c.sorted[f] / K, t1 = n > 1 ? c.sorted[f + 1] / K : -1;
            if (!(p1 && q > 0 && t0 == prev_t0 && t1 == prev_t1)) {
                ++g;
                c.grp_seg[g] = q;
            }
            c.grp_of[q] = g;
            prev_t0 = p1 ? t0 : -1;
            prev_t1 = p1 ? t1 : -1;
            const int tiles = p1 ? P.tiles1 : P.tiles2;
            const int lo = max(s2 * tiles, p1 ? c.u1b : c.u2b), hi = min((s2 + 1) * tiles, p1 ? c.u1e : c.u2e);
            c.grp_left[g] += hi - lo;
        }
        c.ngrp = g + 1;
        // a slot holds the tokens of the largest segment, of either phase
        c.slot_bytes = c.nmax * (P.t1.bytes > P.t2.bytes ? P.t1.bytes : P.t2.bytes);
        c.ring = align_i(align_i(int(sizeof(Ctl)), 1024) + 2 * c.slot_bytes, 1024);
        const int st = (kSmemBytes - 1024 - c.ring) / P.stage_bytes;
        c.stages = st > kMaxStages ? kMaxStages : st;
        if (c.stages < 2) {
            c.abort = 1;
            c.stages = 2;
        }
        c.dst = make_div(uint32_t(c.stages));
        if (blockIdx.x == 0 && c.bad) set_status(A.ws.status, GALE_ERR_ARG);
        if (blockIdx.x == 0 && c.abort) set_status(A.ws.status, GALE_ERR_UNSUPPORTED);
    }
    __syncthreads();
}

// ----------------------------------------------------------------------------
// activations: rotate one 1024-block of a token and write its digits
// ----------------------------------------------------------------------------

// Register layout of a warp-held 1024-block: lane l, register r holds element
//   (l & 7) + 8 (r & 3) + 32 (l >> 3) + 128 (r >> 2),
// so that lane l = q + 8 tig holds, in registers 4 bb .. 4 bb + 3, the four
// elements 128 bb + 32 tig + 8 i + q (i = 0..3): byte i of digit word
// (bb, tig, q).  Digit storage per 128-column block b:
// [digit j (3: bits 16..23, 8..15, 0..7 of Y)][tig (4)][32 bytes], register q
// of lane-quad tig at bytes 4q..4q+3, which is the B fragment of the MMAs of
// bit positions q.
__device__ __forceinline__ int elem_of(int lane, int r) {
    return (lane & 7) + 8 * (r & 3) + 32 * (lane >> 3) + 128 * (r >> 2);
}

// Largest power of two S with m * S <= 2^20 (1 when m is 0).
__device__ __forceinline__ float fixed_scale_of(float m) {
    if (!(m > 0.f)) return 1.0f;
    int e;
    frexpf(1048576.0f / m, &e);
    return ldexpf(1.0f, e - 1);
}

// One 1024-block `blk` of a token's activation (bf16 x, or fp32 h) into the
// slot area `dst` of that token.  Runs a few times per launch and per SM, so
// the loops that do not need registers indexed at compile time stay rolled.
__device__ __noinline__ void build_block(const void* src, int bf16, int blk, uint32_t dst, TokMap tm) {
    const int lane = threadIdx.x & 31;
    float v[32];
    if (bf16) {
        const uint16_t* s = static_cast<const uint16_t*>(src) + 1024 * blk;
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = bf16_to_f32(__ldcg(s + elem_of(lane, r)));
    } else {
        const float* s = static_cast<const float*>(src) + 1024 * blk;
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = __ldcg(s + elem_of(lane, r));
    }
    // butterflies over the lane bits: lower lane v + o, upper lane o - v
#pragma unroll 1
    for (int st = 0; st < 5; ++st) {
        const float sg = ((lane >> st) & 1) ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = fmaf(v[i], sg, __shfl_xor_sync(0xffffffffu, v[i], 1 << st));
    }
    // butterflies over the register bits
#pragma unroll
    for (int st = 0; st < 5; ++st) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & (1 << st)) continue;
            const float a = v[i], b = v[i | (1 << st)];
            v[i] = a + b;
            v[i | (1 << st)] = a - b;
        }
    }
    float m = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) m = fmaxf(m, fabsf(v[r]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float S = fixed_scale_of(m);           // the unnormalised transform is 32x the rotation
    // fp16 copy of u S / 64 (|u S| <= 2^20) in column order, for the outliers
    const float s16 = S * 0.015625f;
#pragma unroll
    for (int r = 0; r < 32; ++r)
        sts_u16(dst + tm.x16 + 2 * (1024 * blk + elem_of(lane, r)), __half_as_ushort(__float2half_rn(v[r] * s16)));
    const int q = lane & 7, tig = lane >> 3;
    const float sc = S * (q < 7 ? __int_as_float((127 - q) << 23) : -0.0078125f);   // S / a(q)
    const int aq = a_of(q);
    const uint32_t a = dst + (blk * 8) * 384 + tig * 32 + q * 4;
    const uint32_t xs_a = dst + tm.xsum + 4 * (blk * 8);
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) {
        // fmaf(v, S / a, 2^23 + 2^20) rounds v S / a to an integer X (|X| <= 2^20)
        // and leaves Y = X + 2^20 in the low 24 bits: its bytes are the digits
        uint32_t y[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) y[i] = __float_as_uint(fmaf(v[4 * bb + i], sc, 9437184.0f));
        const uint32_t lo01 = __byte_perm(y[0], y[1], 0x5140), lo23 = __byte_perm(y[2], y[3], 0x5140);
        const uint32_t hi01 = __byte_perm(y[0], y[1], 0x0062), hi23 = __byte_perm(y[2], y[3], 0x0062);
        sts_u32(a + bb * 384, __byte_perm(hi01, hi23, 0x5410));         // bits 16..23
        sts_u32(a + bb * 384 + 128, __byte_perm(lo01, lo23, 0x7632));   // bits 8..15
        sts_u32(a + bb * 384 + 256, __byte_perm(lo01, lo23, 0x5410));   // bits 0..7
        // sum of the four X (each float word is 0x4B100000 + X)
        const int xs = int(y[0] + y[1] + y[2] + y[3] - 0x2C400000u);
        const int tot = __reduce_add_sync(0xffffffffu, xs * aq);
        if (lane == 0) sts_u32(xs_a + 4 * bb, uint32_t(tot));
    }
    // x_rot = u / 32 = X a / (32 S); the fp16 copy times 2 / S
    if (lane == 0) {
        sts_f32(dst + tm.sig + 4 * blk, 1.0f / (32.0f * S));
        sts_f32(dst + tm.f16 + 4 * blk, 2.0f / S);
    }
}

// ----------------------------------------------------------------------------
// pieces
// ----------------------------------------------------------------------------

// Two 16-row tiles (sign rows at sg0 / sg1, swizzled: 16-byte chunk bb of row
// r at chunk bb ^ (r & 7), rows 128 bytes apart; block scales at sb0 / sb1,
// row pitch sbp bytes) times the 1024-column chunk c of up to two tokens.
// Writes  sigma_c (sum_{b in c} s_blk (X_b - 2 P_b))  of row r of tile m,
// token t to part[(pr_m + r) * 2 + t].
//
// MMA column n = 4 t + j of token t: j = 0 the digit of bits 16..23 of
// Y = X + 2^20, j = 1 a column of ones, j = 2 and 3 the digits of bits 8..15
// and 0..7.  Per block a lane combines its two columns exactly in int32:
// lanes of even tig  D16 - 16 ONES  (the 2^20 offset times ONES, over 2^16),
// lanes of odd tig   256 D8 + D0,  so that P_b = 2^16 (even) + (odd).
// The eight blocks are unrolled; the sixteen block scales a lane needs (its
// two rows of each tile) come in four 16-byte loads before the loop.
__device__ __noinline__ void mma_piece(uint32_t sg0, uint32_t sg1, uint32_t sb0, uint32_t sb1, int sbp, int c,
                                       uint32_t slot, int tstride, TokMap tm, int ntok, uint32_t part, int pr0,
                                       int pr1) {
    const uint32_t sg[2] = {sg0, sg1}, sb[2] = {sb0, sb1};
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    const int j = g & 3;
    const bool ones = j == 1;
    const bool bl = !ones && (g < 4 || ntok > 1);
    const uint32_t bsrc = slot + (g >> 2) * tstride + (j == 0 ? 0 : j - 1) * 128 + tig * 32 + c * 8 * 384;
    const uint32_t bfill = ones ? 0x01010101u : 0u;
    const int mA = (tig & 1) ? 256 : 1, mB = (tig & 1) ? 1 : -16;
    uint4 sv[2][2];   // [tile][row g, row g + 8]: the chunk's eight fp16 block scales
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        sv[m][0] = lds_v4(sb[m] + g * sbp + 16 * c);
        sv[m][1] = lds_v4(sb[m] + (g + 8) * sbp + 16 * c);
    }
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const uint32_t woff = g * 128 + tig * 4;
    // two blocks per iteration (the scale pair of both is one 32-bit word of
    // sv, which moves down by one component per iteration)
#pragma unroll 1
    for (int bp = 0; bp < 4; ++bp) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int bb = 2 * bp + h;
            uint4 q0 = make_uint4(bfill, bfill, bfill, bfill), q1 = q0;
            if (bl) {
                q0 = lds_v4(bsrc + bb * 384);
                q1 = lds_v4(bsrc + bb * 384 + 16);
            }
            const uint32_t wo = woff + ((bb ^ g) << 4);
            uint32_t w[2][2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                w[m][0] = lds_u32(sg[m] + wo);
                w[m][1] = lds_u32(sg[m] + wo + 1024);
            }
            const uint32_t breg[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                // bit positions 0..3 and 4..7 as two independent MMA chains
                int ca[4] = {0, 0, 0, 0}, cb[4] = {0, 0, 0, 0};
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const uint32_t m0 = 0x01010101u << (2 * mm), m1 = m0 << 1;
                    const uint32_t n0 = m0 << 4, n1 = m1 << 4;
                    mma_s8u8(ca, w[m][0] & m0, w[m][1] & m0, w[m][0] & m1, w[m][1] & m1, breg[2 * mm],
                             breg[2 * mm + 1]);
                    mma_s8u8(cb, w[m][0] & n0, w[m][1] & n0, w[m][0] & n1, w[m][1] & n1, breg[2 * mm + 4],
                             breg[2 * mm + 5]);
                }
                const float s0 = h2f(h ? sv[m][0].x >> 16 : sv[m][0].x);
                const float s1 = h2f(h ? sv[m][1].x >> 16 : sv[m][1].x);
                acc[m][0] = fmaf(s0, float((ca[0] + cb[0]) * mA + (ca[1] + cb[1]) * mB), acc[m][0]);
                acc[m][1] = fmaf(s1, float((ca[2] + cb[2]) * mA + (ca[3] + cb[3]) * mB), acc[m][1]);
            }
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int r = 0; r < 2; ++r) sv[m][r] = make_uint4(sv[m][r].y, sv[m][r].z, sv[m][r].w, sv[m][r].x);
    }
    // P of rows g and g + 8 from the lane pair (tig even: high part, odd: low
    // part); the even lane then owns row g, the odd lane row g + 8, of token
    // tig >> 1.
    const int odd = tig & 1, tok = tig >> 1;
    const int orow = g + 8 * odd;
    const uint32_t tb = slot + tok * tstride;
    const uint4 x0 = lds_v4(tb + tm.xsum + 32 * c), x1 = lds_v4(tb + tm.xsum + 32 * c + 16);
    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    const float sig = lds_f32(tb + tm.sig + 4 * c);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const float o0 = __shfl_xor_sync(0xffffffffu, acc[m][0], 1);
        const float o1 = __shfl_xor_sync(0xffffffffu, acc[m][1], 1);
        const float P = odd ? fmaf(65536.0f, o1, acc[m][1]) : fmaf(65536.0f, acc[m][0], o0);
        if (tok < ntok) {
            const uint4 sc = odd ? sv[m][1] : sv[m][0];
            const uint32_t sw[4] = {sc.x, sc.y, sc.z, sc.w};
            float xt = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xt = fmaf(h2f(sw[i] & 0xFFFFu), float(int(xw[2 * i])), xt);
                xt = fmaf(h2f(sw[i] >> 16), float(int(xw[2 * i + 1])), xt);
            }
            sts_f32(part + (((m ? pr1 : pr0) + orow) * 2 + tok) * 4, sig * fmaf(-2.0f, P, xt));
        }
    }
}

// Where one row's outlier records, sign line and block scales sit in a stage.
struct RowRef {
    uint32_t idx;       // outlier columns of the row (uint16)
    uint32_t qb;        // byte holding nibble 0 of the values counted from n0
    int n0;             // nibble index of the row's value 0 relative to qb
    uint32_t sign;      // the row's 128-byte line in chunk 0 of the swizzled sign area
    int chunk_stride;   // bytes between chunks in the sign area
    int sw;             // row & 7
    uint32_t sblk;      // the row's block scales
    float srow;
};

// One outlier of the row: the value nibble q (offset binary q + 8 in `nib`)
// and column `col` (col >= C: a record that failed validation, counted as 0).
__device__ __forceinline__ void outlier_one(const RowRef& R, uint32_t col, uint32_t nib, int C, uint32_t x0,
                                            uint32_t f0, int tstride, int ntok, float& corr0, float& corr1) {
    const bool ok = col < uint32_t(C);
    const uint32_t cc = ok ? col : 0u;
    // value: float(q) through the exponent field of 2^23 (exact for small integers)
    const float q = __uint_as_float(nib ^ 0x4B000008u) - 8388616.0f;
    // the sign word holding column cc (swizzled 16-byte chunk of the row's line)
    const uint32_t word = lds_u32(R.sign + (cc >> 10) * uint32_t(R.chunk_stride) +
                                  (((cc >> 3) & 0x7Cu) ^ (uint32_t(R.sw) << 4)));
    const uint32_t sbits = lds_u16(R.sblk + ((cc >> 6) & ~1u));
    // - sign s_blk: +s_blk where the bit is 1 (weight -1), -s_blk where it is 0
    const float nsb = __uint_as_float(__float_as_uint(h2f(sbits)) ^ ((~__funnelshift_r(word, word, cc)) << 31));
    const float wq = ok ? fmaf(q, R.srow, nsb) : 0.f;
    const uint32_t fo = 4u * (cc >> 10);
    corr0 = fmaf(wq * lds_f32(f0 + fo), h2f(lds_u16(x0 + 2u * cc)), corr0);
    if (ntok > 1)
        corr1 = fmaf(wq * lds_f32(f0 + uint32_t(tstride) + fo), h2f(lds_u16(x0 + uint32_t(tstride) + 2u * cc)), corr1);
}

// Outlier corrections of one row over outliers j0 <= j < j1:
//   sum_j (q_j s_row - sign_j s_blk) x_{c_j}
// for up to two tokens (the MMA part counted the sign weight at c_j); written
// to out (two floats).  Values are read a byte (two nibbles) at a time.
__device__ __noinline__ void outlier_row(const RowRef R, int j0, int j1, int C, uint32_t slot, int tstride,
                                         TokMap tm, int ntok, uint32_t out) {
    float corr0 = 0.f, corr1 = 0.f;
    const uint32_t x0 = slot + tm.x16, f0 = slot + tm.f16;
    int j = j0;
    int n = R.n0 + j0;   // nibble index of outlier j, counted from byte qb
    if (j < j1 && (n & 1)) {
        outlier_one(R, lds_u16(R.idx + 2 * j), lds_u8(R.qb + (n >> 1)) >> 4, C, x0, f0, tstride, ntok, corr0, corr1);
        ++j;
        ++n;
    }
#pragma unroll 2
    for (; j + 1 < j1; j += 2, n += 2) {
        const uint32_t qb = lds_u8(R.qb + (n >> 1));
        const uint32_t c0 = lds_u16(R.idx + 2 * j), c1 = lds_u16(R.idx + 2 * j + 2);
        outlier_one(R, c0, qb & 0xFu, C, x0, f0, tstride, ntok, corr0, corr1);
        outlier_one(R, c1, qb >> 4, C, x0, f0, tstride, ntok, corr0, corr1);
    }
    if (j < j1)
        outlier_one(R, lds_u16(R.idx + 2 * j), lds_u8(R.qb + (n >> 1)) & 0xFu, C, x0, f0, tstride, ntok, corr0, corr1);
    sts_f32(out, corr0);
    sts_f32(out + 4, corr1);
}

// ----------------------------------------------------------------------------
// finishing a unit
// ----------------------------------------------------------------------------

__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// RMSNorm of token t once all its 64-row blocks are combined: v (x + y) is
// in the workspace, the blocks' sums of squares in ssq.
__device__ __noinline__ void normalize_token(const StreamArgs& A, int t) {
    const int lane = threadIdx.x & 31;
    const int d = A.d_model, nb = d / 64;
    float ss = 0.f;
#pragma unroll 1
    for (int i = lane; i < nb; i += 32) ss += __ldcg(A.ws.ssq + t * nb + i);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / float(d) + A.eps);
    const float4* v = reinterpret_cast<const float4*>(A.ws.v + t * d);
    uint2* o = reinterpret_cast<uint2*>(static_cast<uint16_t*>(A.out) + t * d);
#pragma unroll 4
    for (int i = lane; i < d / 4; i += 32) {
        const float4 a = __ldcg(v + i);
        uint2 w;
        w.x = uint32_t(f32_to_bf16(a.x * inv)) | (uint32_t(f32_to_bf16(a.y * inv)) << 16);
        w.y = uint32_t(f32_to_bf16(a.z * inv)) | (uint32_t(f32_to_bf16(a.w * inv)) << 16);
        o[i] = w;
    }
    // the token's output (a chain's next input) is complete
    __syncwarp();
    if (lane == 0) red_release_add(A.xready, 1);
}

// y of token t over the 64 rows of block `tile`, once all its experts' o are
// in: the K outputs in fixed k order, eight loads in flight at a time.
__device__ __noinline__ void combine_block(const StreamArgs& A, const Ctl& c, int t, int tile) {
    const int lane = threadIdx.x & 31;
    const int d = A.d_model, K = A.K, nb = d / 64;
    const uint32_t vm = c.vmask[t];
    float y0 = 0.f, y1 = 0.f;
#pragma unroll 1
    for (int k0 = 0; k0 < K; k0 += 8) {
        float g[8], o0[8], o1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = k0 + j;
            const bool ok = k < K && ((vm >> k) & 1u);
            const float* o = A.ws.o + (t * K + (ok ? k : 0)) * d + tile * 64 + lane;
            g[j] = ok ? (A.fixed_e >= 0 ? 1.f : __ldg(A.gates + t * K + k)) : 0.f;
            o0[j] = ok ? __ldcg(o) : 0.f;
            o1[j] = ok ? __ldcg(o + 32) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            y0 = fmaf(g[j], o0[j], y0);
            y1 = fmaf(g[j], o1[j], y1);
        }
    }
    const int r0 = t * d + tile * 64 + lane;
    if (!A.fuse_norm) {
        if (A.out_dtype == GALE_F32) {
            static_cast<float*>(A.out)[r0] = y0;
            static_cast<float*>(A.out)[r0 + 32] = y1;
        } else {
            static_cast<uint16_t*>(A.out)[r0] = f32_to_bf16(y0);
            static_cast<uint16_t*>(A.out)[r0 + 32] = f32_to_bf16(y1);
        }
        return;
    }
    const float v0 = bf16_to_f32(__ldcg(A.x + r0)) + y0;
    const float v1 = bf16_to_f32(__ldcg(A.x + r0 + 32)) + y1;
    A.ws.v[r0] = v0;
    A.ws.v[r0 + 32] = v1;
    const float ss = warp_sum(fmaf(v0, v0, v1 * v1));
    if (lane == 0) A.ws.ssq[t * nb + tile] = ss;
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atom_acq_rel_add(A.ws.tokcnt + t, 1) == nb - 1;
    if (__shfl_sync(0xffffffffu, last, 0)) {
        __syncwarp();
        normalize_token(A, t);
    }
}

// Tokens with no valid pair: y = 0 (out = 0, or the norm of x alone).
__device__ __noinline__ void empty_token(const StreamArgs& A, int t) {
    const int lane = threadIdx.x & 31;
    const int d = A.d_model;
    float ss = 0.f;
#pragma unroll 1
    for (int r = lane; r < d; r += 32) {
        const float v = bf16_to_f32(__ldcg(A.x + t * d + r));
        ss = fmaf(v, v, ss);
    }
    const float inv = rsqrtf(warp_sum(ss) / float(d) + A.eps);
#pragma unroll 1
    for (int r = lane; r < d; r += 32) {
        if (A.fuse_norm) static_cast<uint16_t*>(A.out)[t * d + r] = f32_to_bf16(bf16_to_f32(__ldcg(A.x + t * d + r)) * inv);
        else if (A.out_dtype == GALE_F32) static_cast<float*>(A.out)[t * d + r] = 0.f;
        else static_cast<uint16_t*>(A.out)[t * d + r] = 0;
    }
    __syncwarp();
    if (lane == 0) red_release_add(A.xready, 1);
}

// ----------------------------------------------------------------------------
// the kernel
// ----------------------------------------------------------------------------

struct UnitRef {
    bool p1;
    int U, s, q, tile, e, n, first, st, par;
};

__device__ __forceinline__ UnitRef unit_ref(const Ctl& c, const Plan& P, int u) {
    UnitRef r;
    const int n1 = c.u1e - c.u1b;
    r.p1 = u < n1;
    if (r.p1) {
        r.U = c.u1b + u;
        r.s = fdiv(r.U, P.dt1);
        r.tile = r.U - r.s * P.tiles1;
        r.q = r.s - c.s1b;
    } else {
        r.U = c.u2b + (u - n1);
        r.s = fdiv(r.U, P.dt2);
        r.tile = r.U - r.s * P.tiles2;
        r.q = c.nl1 + r.s - c.s2b;
    }
    const int sg = c.seg[r.s];
    r.e = seg_e(sg);
    r.n = seg_n(sg);
    r.first = seg_first(sg);
    const int gu = c.ubase + u;   // the ring's running unit index (all layers)
    const int lap = fdiv(gu, c.dst);
    r.st = gu - lap * c.stages;
    r.par = lap & 1;
    return r;
}

// One activation piece `cl` (token cl / blocks, 1024-block cl % blocks) of
// group g into its slot.  A phase-2 piece first waits until the segment's h
// block is complete in every CTA (bounded).
__device__ __noinline__ void act_piece(const StreamArgs& A, const Plan& P, Ctl& c, int g, int cl, uint32_t slot) {
    const int lane = threadIdx.x & 31;
    const int q = c.grp_seg[g];
    const bool p1 = q < c.nl1;
    const int s = p1 ? c.s1b + q : c.s2b + (q - c.nl1);
    const int sg = c.seg[s];
    const int nb = p1 ? P.nch1 : P.nch2;
    const int tk = cl / nb, blk = cl - tk * nb;
    const int pair = c.sorted[seg_first(sg) + tk];
    if (p1) {
        if (A.xf)
            build_block(A.xf + (pair / A.K) * A.d_model, 0, blk, slot + uint32_t(tk * P.t1.bytes), P.t1);
        else
            build_block(A.x + (pair / A.K) * A.d_model, 1, blk, slot + uint32_t(tk * P.t1.bytes), P.t1);
    } else {
        int v = 1;
        if (lane == 0) v = wait_global(A.ws.hcnt + s * P.nch2 + blk, 1024 / kR1, &c.abort, c.wait_ns);
        v = __shfl_sync(0xffffffffu, v, 0);
        __syncwarp();
        if (!v) {
            set_status(A.ws.status, GALE_ERR_TIMEOUT);
            atomicExch(&c.abort, 1);
        }
        build_block(A.ws.h + pair * A.d_ff, 0, blk, slot + uint32_t(tk * P.t2.bytes), P.t2);
    }
}

// Whether the phase-2 activation piece `cl` of group g could start now (its
// h block complete); phase-1 pieces always can.
__device__ __forceinline__ bool act_ready(const StreamArgs& A, const Plan& P, const Ctl& c, int g, int cl) {
    const int q = c.grp_seg[g];
    if (q < c.nl1) return true;
    const int s = c.s2b + (q - c.nl1);
    return vload(A.ws.hcnt + s * P.nch2 + cl % P.nch2) >= 1024 / kR1;
}

__device__ __forceinline__ int grp_need(const Ctl& c, const Plan& P, int g) {
    const int q = c.grp_seg[g];
    const bool p1 = q < c.nl1;
    const int sg = c.seg[p1 ? c.s1b + q : c.s2b + (q - c.nl1)];
    return seg_n(sg) * (p1 ? P.nch1 : P.nch2);
}

__global__ void __launch_bounds__(kThreads, 1)
moe_stream_kernel(const __grid_constant__ CUtensorMap map13, const __grid_constant__ CUtensorMap map2,
                  const StreamArgs A, const Plan P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    Ctl& c = *reinterpret_cast<Ctl*>(smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == kCW * 32) {
        prefetch_tensormap(&map13);
        prefetch_tensormap(&map2);
    }
    // the ring's barriers and counters live across the layers of a chain
    if (tid < kMaxStages) {
        c.stage_done[tid] = 0;
        mbar_init(&c.full[tid], 1);
        mbar_init(&c.empty[tid], 1);
    }
    if (tid == 0) {
        c.abort = 0;
        c.issued = 0;
        c.ubase = 0;
        fence_mbar_init();
    }
    __syncthreads();
    int S = 2;
#pragma unroll 1
    for (int layer = 0; layer < A.n_layers; ++layer) {
    // the layer's arguments: its pairs, its input and output, its counters
    StreamArgs Al = A;
    {
        const int64_t lpairs = int64_t(layer) * A.B * A.K;
        Al.ids = A.ids + lpairs;
        Al.gates = A.gates + lpairs;
        Al.e_off = int64_t(layer) * A.layer_experts;
        Al.x = layer == 0 ? A.x : A.ws.xbuf + int64_t((layer - 1) & 1) * A.B * A.d_model;
        Al.out = layer == A.n_layers - 1 ? A.out : static_cast<void*>(A.ws.xbuf + int64_t(layer & 1) * A.B * A.d_model);
        Al.ws.hcnt = A.ws.hcnt + layer * A.ws.layer_ints;
        Al.ws.comb = A.ws.comb + layer * A.ws.layer_ints;
        Al.ws.tokcnt = A.ws.tokcnt + layer * A.ws.layer_ints;
        Al.xready = A.ws.xready + layer;
    }
    route_and_plan(Al, P, c, *reinterpret_cast<RouteScratch*>(smem + kScratchOff));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t slot_base = s_base + uint32_t(align_i(int(sizeof(Ctl)), 1024));
    const uint32_t ring = s_base + uint32_t(c.ring);
    S = c.stages;
    const int n1 = c.u1e - c.u1b, n2 = c.u2e - c.u2b;
    const int nunits = n1 + n2;
    int32_t* status = A.ws.status;

    if (warp == kCW) {
        // ---------------- producer ----------------
        if (lane == 0 && !c.abort) {
#pragma unroll 1
            for (int u = 0; u < nunits; ++u) {
                const UnitRef R = unit_ref(c, P, u);
                if (c.ubase + u >= S && !wait_phase(&c.empty[R.st], R.par ^ 1, c.wait_ns)) {
                    set_status(status, GALE_ERR_TIMEOUT);
                    atomicExch(&c.abort, 1);
                    break;
                }
                if (vload(&c.abort)) break;
                uint8_t* stage = smem + (ring - s_base) + size_t(R.st) * P.stage_bytes;
                uint64_t* bar = &c.full[R.st];
                const char* rec = A.base + (Al.e_off + R.e) * A.stride;
                const int rows = R.p1 ? kR1 : kR2;
                const int k = R.p1 ? P.k1 : P.k2;
                const StageMap& M = R.p1 ? P.m1 : P.m2;
                const Layout& L = R.p1 ? P.L1 : P.L2;
                const int nmat = R.p1 ? 2 : 1;
                const int64_t qs = int64_t(R.tile) * rows * k / 2;   // first value byte
                const int64_t qa = qs & ~int64_t(15), qe = align_up(qs + int64_t(rows) * k / 2, 16);
                const uint32_t qbytes = uint32_t(qe - qa);
                const uint32_t per_mat = uint32_t(M.sb_bytes) + uint32_t(rows * 2) + uint32_t(M.idx_bytes) + qbytes;
                mbar_arrive_expect_tx(bar, uint32_t(nmat * (R.p1 ? P.nch1 : P.nch2) * rows * 128) + nmat * per_mat);
                tma_load_5d(stage, R.p1 ? &map13 : &map2, bar, 0, R.tile * rows, 0, 0, int(Al.e_off) + R.e);
#pragma unroll 1
                for (int m = 0; m < nmat; ++m) {
                    const char* mat = rec + A.off_w[R.p1 ? m : 2];
                    bulk_load(stage + M.sb + m * M.sb_bytes, mat + L.off_sblk + int64_t(R.tile) * M.sb_bytes,
                              M.sb_bytes, bar);
                    bulk_load(stage + M.sr + m * 32, mat + L.off_srow + int64_t(R.tile) * rows * 2, rows * 2, bar);
                    bulk_load(stage + M.idx + m * align_i(M.idx_bytes, 16),
                              mat + L.off_idx + int64_t(R.tile) * M.idx_bytes, M.idx_bytes, bar);
                    bulk_load(stage + M.q + m * M.q_bytes, mat + L.off_q + qa, qbytes, bar);
                }
                c.issued = c.ubase + u + 1;
            }
        }
    } else {
        // ---------------- consumers ----------------
        // tokens without a valid pair get their output here (nothing combines them)
#pragma unroll 1
        for (int t = blockIdx.x * kCW + warp; t < A.B; t += gridDim.x * kCW)
            if (c.vmask[t] == 0u) empty_token(Al, t);
        const int tot_pieces = n1 * P.pp1 + n2 * P.pp2;
        const int nhb = P.nch2;
#pragma unroll 1
        for (;;) {
            int pc = 0;
            if (lane == 0) pc = atomicAdd(&c.next_piece, 1);
            pc = __shfl_sync(0xffffffffu, pc, 0);
            if (pc >= tot_pieces || vload(&c.abort)) break;
            const bool p1 = pc < n1 * P.pp1;
            const int pr = p1 ? pc : pc - n1 * P.pp1;
            const int ur = fdiv(pr, p1 ? P.dpp1 : P.dpp2);
            const int u = p1 ? ur : n1 + ur;
            const int sub = pr - ur * (p1 ? P.pp1 : P.pp2);
            const UnitRef R = unit_ref(c, P, u);
            // ---- the activations of the unit's group, in slot g & 1 ----
            const int g = c.grp_of[R.q];
            const int sl = g & 1;
            const int need = grp_need(c, P, g);
            const int tstride = R.p1 ? P.t1.bytes : P.t2.bytes;
            const uint32_t slot = slot_base + uint32_t(sl * c.slot_bytes);
            {
                bool ok = vload(&c.slot_grp[sl]) == g || wait_smem(&c.slot_grp[sl], g, true, &c.abort, c.wait_ns);
#pragma unroll 1
                while (ok && vload(&c.slot_done[sl]) < need) {
                    // the slot cannot move on while this unit is unfinished,
                    // so the claim word is the group's
                    int cl = 0;
                    if (lane == 0) cl = atomicAdd(&c.slot_claim[sl], 1) & 0xFFFF;
                    cl = __shfl_sync(0xffffffffu, cl, 0);
                    if (cl < need) {
                        act_piece(Al, P, c, g, cl, slot);
                        __syncwarp();
                        __threadfence_block();
                        if (lane == 0) atomicAdd(&c.slot_done[sl], 1);
                    } else {
                        ok = wait_smem(&c.slot_done[sl], need, false, &c.abort, c.wait_ns);
                    }
                }
                if (!ok) {
                    if (!vload(&c.abort)) set_status(status, GALE_ERR_TIMEOUT);
                    atomicExch(&c.abort, 1);
                    break;
                }
                __threadfence_block();
            }
            // ---- the unit's rows ----
            if (!wait_phase(&c.full[R.st], R.par, c.wait_ns)) {
                set_status(status, GALE_ERR_TIMEOUT);
                atomicExch(&c.abort, 1);
                break;
            }
            const uint32_t stage = ring + uint32_t(R.st * P.stage_bytes);
            const uint32_t part = stage + P.part;
            if (R.p1) {
                const int nch = P.nch1;
                if (sub < nch) {
                    mma_piece(stage + uint32_t(sub * 2048), stage + uint32_t((nch + sub) * 2048), stage + P.m1.sb,
                              stage + P.m1.sb + P.m1.sb_bytes, P.C1 / 64, sub, slot, tstride, P.t1, R.n,
                              part + uint32_t(sub * 32 * 8), 0, 16);
                } else {
                    const int o = sub - nch;
                    const int m = lane >> 4, r = lane & 15;
                    RowRef RR;
                    RR.idx = stage + P.m1.idx + m * align_i(P.m1.idx_bytes, 16) + r * P.k1 * 2;
                    const int64_t qs = int64_t(R.tile) * kR1 * P.k1 / 2;
                    RR.qb = stage + P.m1.q + m * P.m1.q_bytes + uint32_t(qs & 15);
                    RR.n0 = r * P.k1;
                    RR.sign = stage + uint32_t(m * nch * 2048 + r * 128);
                    RR.chunk_stride = 2048;
                    RR.sw = r & 7;
                    RR.sblk = stage + P.m1.sb + m * P.m1.sb_bytes + r * (P.C1 / 64);
                    RR.srow = h2f(lds_u16(stage + P.m1.sr + m * 32 + 2 * r));
                    const int jh = (P.k1 + 1) / 2;
                    outlier_row(RR, o ? jh : 0, o ? P.k1 : jh, P.C1, slot, tstride, P.t1, R.n,
                                part + uint32_t(((nch + o) * 32 + lane) * 8));
                }
            } else {
                const int nch = P.nch2;
                if (sub < 2 * nch) {
                    const int ch = sub % nch, half = sub / nch;
                    const int sbp = P.C2 / 64;
                    mma_piece(stage + uint32_t(ch * kR2 * 128 + (2 * half) * 2048),
                              stage + uint32_t(ch * kR2 * 128 + (2 * half + 1) * 2048),
                              stage + P.m2.sb + uint32_t((2 * half) * 16 * sbp),
                              stage + P.m2.sb + uint32_t((2 * half + 1) * 16 * sbp), sbp, ch, slot, tstride, P.t2,
                              R.n, part + uint32_t(ch * 64 * 8), half * 32, half * 32 + 16);
                } else {
                    const int o = sub - 2 * nch;
                    const int r = o * 32 + lane;
                    RowRef RR;
                    RR.idx = stage + P.m2.idx + r * P.k2 * 2;
                    RR.qb = stage + P.m2.q;
                    RR.n0 = r * P.k2;
                    RR.sign = stage + uint32_t(r * 128);
                    RR.chunk_stride = kR2 * 128;
                    RR.sw = r & 7;
                    RR.sblk = stage + P.m2.sb + r * (P.C2 / 64);
                    RR.srow = h2f(lds_u16(stage + P.m2.sr + 2 * r));
                    outlier_row(RR, 0, P.k2, P.C2, slot, tstride, P.t2, R.n, part + uint32_t((nch * 64 + r) * 8));
                }
            }
            // ---- the last piece of the unit finishes it: the partial sums
            //      go to registers, the stage goes back to the producer, then
            //      the rows are written and published ----
            __syncwarp();
            __threadfence_block();
            int last = 0;
            if (lane == 0) last = atomicAdd(&c.stage_done[R.st], 1) == (R.p1 ? P.pp1 : P.pp2) - 1;
            if (__shfl_sync(0xffffffffu, last, 0)) {
                __threadfence_block();
                constexpr int kY = kSegTok * kR2 / 32;
                float hv = 0.f, yv[kY];
                if (R.p1) {
                    // h row lane & 15 of token lane >> 4: silu(w1 x) * (w3 x) over
                    // slices 0..nch-1 (chunks), nch, nch+1 (outliers)
                    if (lane < kR1 * R.n) {
                        const int r = lane & 15, t = lane >> 4;
                        float g1 = 0.f, g3 = 0.f;
#pragma unroll 1
                        for (int s2 = 0; s2 < P.nch1 + 2; ++s2) {
                            g1 += lds_f32(part + uint32_t(((s2 * 32 + r) * 2 + t) * 4));
                            g3 += lds_f32(part + uint32_t(((s2 * 32 + 16 + r) * 2 + t) * 4));
                        }
                        hv = silu_fast(g1) * g3;
                    }
                } else {
                    // o rows over slices 0..nch-1 (chunks), nch (outliers)
#pragma unroll
                    for (int i = 0; i < kY; ++i) {
                        const int it = lane + 32 * i, r = it & 63, t = it >> 6;
                        float y = 0.f;
                        if (it < kR2 * R.n) {
#pragma unroll 1
                            for (int s2 = 0; s2 < P.nch2 + 1; ++s2)
                                y += lds_f32(part + uint32_t(((s2 * 64 + r) * 2 + t) * 4));
                        }
                        yv[i] = y;
                    }
                }
                // release the stage and count the unit into its group
                __syncwarp();
                if (lane == 0) {
                    c.stage_done[R.st] = 0;
                    __threadfence_block();
                    mbar_arrive(&c.empty[R.st]);
                    if (atomicSub(&c.grp_left[g], 1) == 1 && g + 2 < c.ngrp) {
                        c.slot_claim[sl] = (g + 2) << 16;
                        c.slot_done[sl] = 0;
                        __threadfence_block();
                        atomicExch(&c.slot_grp[sl], g + 2);
                    }
                }
                if (R.p1) {
                    if (lane < kR1 * R.n) {
                        const int pair = c.sorted[R.first + (lane >> 4)];
                        A.ws.h[pair * A.d_ff + R.tile * kR1 + (lane & 15)] = hv;
                    }
                    __syncwarp();
                    if (lane == 0 && int(blockIdx.x) != A.withhold_cta)
                        red_release_add(Al.ws.hcnt + R.s * nhb + (R.tile * kR1) / 1024, 1);
                } else {
#pragma unroll
                    for (int i = 0; i < kY; ++i) {
                        const int it = lane + 32 * i;
                        if (it < kR2 * R.n) {
                            const int pair = c.sorted[R.first + (it >> 6)];
                            A.ws.o[pair * A.d_model + R.tile * kR2 + (it & 63)] = yv[i];
                        }
                    }
                    __syncwarp();
                    const int nb = A.d_model / 64;
#pragma unroll 1
                    for (int t = 0; t < R.n; ++t) {
                        const int tk = c.sorted[R.first + t] / A.K;
                        int lastc = 0;
                        if (lane == 0)
                            lastc = atom_acq_rel_add(Al.ws.comb + tk * nb + R.tile, 1) == __popc(c.vmask[tk]) - 1;
                        if (__shfl_sync(0xffffffffu, lastc, 0)) {
                            __syncwarp();
                            combine_block(Al, c, tk, R.tile);
                        }
                    }
                }
            }
            // ---- work ahead: one activation piece of the next group, if its
            //      slot is free and (phase 2) its h block is complete ----
            // (a phase-2 group only from a phase-2 piece: its readiness test
            // reads a global counter, a round trip that a phase-1 piece would
            // add to every hand-off)
            const int gn = g + 1;
            if (gn < c.ngrp && (!R.p1 || c.grp_seg[gn] < c.nl1) && vload(&c.slot_grp[gn & 1]) == gn) {
                const int sln = gn & 1;
                const int needn = grp_need(c, P, gn);
                // claim only if the claim word still belongs to group gn: a
                // warp ahead holds no unit of gn, so the slot may move on
                int cl = needn;
                if (lane == 0) {
                    const int v = vload(&c.slot_claim[sln]);
                    if ((v >> 16) == gn && (v & 0xFFFF) < needn && act_ready(Al, P, c, gn, v & 0xFFFF) &&
                        atomicCAS(&c.slot_claim[sln], v, v + 1) == v)
                        cl = v & 0xFFFF;
                }
                cl = __shfl_sync(0xffffffffu, cl, 0);
                if (cl < needn) {
                    act_piece(Al, P, c, gn, cl, slot_base + uint32_t(sln * c.slot_bytes));
                    __syncwarp();
                    __threadfence_block();
                    if (lane == 0) atomicAdd(&c.slot_done[sln], 1);
                }
            }
        }
    }
    // ---- end of the layer: the next one starts once every token's output
    //      (its input) is written by whichever CTAs finished them ----
    __syncthreads();
    if (tid == 0) {
        c.ubase += nunits;
        if (layer + 1 < A.n_layers && !vload(&c.abort) &&
            !wait_global(Al.xready, A.B, &c.abort, c.wait_ns)) {
            set_status(status, GALE_ERR_TIMEOUT);
            atomicExch(&c.abort, 1);
        }
    }
    __syncthreads();
    if (vload(&c.abort)) break;
    }   // layers
    // every copy the producer issued has landed before the CTA exits
    __syncthreads();
    if (tid == 0 && vload(&c.abort)) {
        const int iss = c.issued;
#pragma unroll 1
        for (int u = iss - S > 0 ? iss - S : 0; u < iss; ++u) wait_phase(&c.full[u % S], (u / S) & 1, 100000000ull);
    }
}

// Failure-path testing settings (process-wide, see gale_debug_set_failure).
uint64_t g_wait_ns = kWaitNs;
int g_withhold_cta = -1;

}  // namespace

StreamWs carve_stream_ws(void* ws, const gale_layer& L, int B, int K, int n_layers) {
    StreamWs w{};
    char* p = static_cast<char*>(ws);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        char* q = p ? p + o : nullptr;
        o = align_up(o + bytes, 256);
        return q;
    };
    const int64_t BK = int64_t(B) * K, dm = L.d_model, df = L.d_ff;
    const int64_t nb = dm / 64;
    // counters first: one memset clears them all.  Per layer, [hcnt | comb | tokcnt].
    w.status = reinterpret_cast<int32_t*>(take(256));
    const int64_t nh = BK * (df / 1024), nc = int64_t(B) * nb;
    w.layer_ints = align_up(nh + nc + B, 64);
    int32_t* cnt = reinterpret_cast<int32_t*>(take(4 * w.layer_ints * n_layers));
    w.hcnt = cnt;
    w.comb = cnt ? cnt + nh : nullptr;
    w.tokcnt = cnt ? cnt + nh + nc : nullptr;
    w.xready = reinterpret_cast<int32_t*>(take(4 * int64_t(n_layers)));
    w.counter_bytes = size_t(o);
    w.ssq = reinterpret_cast<float*>(take(4 * int64_t(B) * nb));
    w.h = reinterpret_cast<float*>(take(4 * BK * df));
    w.o = reinterpret_cast<float*>(take(4 * BK * dm));
    w.v = reinterpret_cast<float*>(take(4 * int64_t(B) * dm));
    w.xbuf = n_layers > 1 ? reinterpret_cast<uint16_t*>(take(2 * 2 * int64_t(B) * dm)) : nullptr;
    w.bytes = size_t(o);
    return w;
}

bool stream_supported(const gale_layer& L, int B, int K) {
    if (B < 1 || K > 16 || int64_t(B) * K > kDecodeMaxPairsStream || L.n_experts > 1023) return false;
    if (L.d_model % 1024 || L.d_ff % 1024 || L.d_model > 4096 || L.d_ff > 2048) return false;
    const Plan P = make_stream_plan(L.d_model, L.d_ff);
    const int ctl = align_i(int(sizeof(Ctl)), 1024);
    const int slot = kSegTok * (P.t1.bytes > P.t2.bytes ? P.t1.bytes : P.t2.bytes);
    return kSmemBytes - 1024 - align_i(ctl + 2 * slot, 1024) >= 2 * P.stage_bytes;
}

int launch_moe_stream(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                      void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st, int n_layers,
                      int64_t layer_experts, const float* xf, int fixed_e) {
    StreamArgs A{};
    A.base = static_cast<const char*>(L.base);
    A.stride = L.expert_stride;
    A.E = L.n_experts;
    A.d_model = L.d_model;
    A.d_ff = L.d_ff;
    A.B = B;
    A.K = K;
    const Plan P = make_stream_plan(L.d_model, L.d_ff);
    A.off_w[0] = 0;
    A.off_w[1] = P.L1.total;
    A.off_w[2] = 2 * P.L1.total;
    A.x = x;
    A.ids = ids;
    A.gates = gates;
    A.out = out;
    A.out_dtype = out_dtype;
    A.fuse_norm = fuse_norm ? 1 : 0;
    A.eps = eps;
    A.wait_ns = g_wait_ns;
    A.withhold_cta = g_withhold_cta;
    A.n_layers = n_layers;
    A.xf = xf;
    A.fixed_e = fixed_e;
    A.layer_experts = n_layers > 1 ? layer_experts : 0;
    A.e_off = 0;
    A.ws = carve_stream_ws(ws, L, B, K, n_layers);
    A.xready = A.ws.xready;
    GALE_CUDA_TRY(cudaMemsetAsync(A.ws.status, 0, A.ws.counter_bytes, st));
    CUtensorMap map13, map2;
    // one map over the expert records of every layer (a chain's layers are
    // records l * layer_experts + e of the same array)
    const int64_t n_rec = int64_t(n_layers - 1) * A.layer_experts + L.n_experts;
    if (n_rec > 0x7FFFFFFF) return GALE_ERR_UNSUPPORTED;
    int rc = cached_sign_map5b(&map13, A.base, L.d_ff, L.d_model, 2, P.L1.total, int(n_rec), L.expert_stride, kR1, 2);
    if (rc == GALE_OK)
        rc = cached_sign_map5b(&map2, A.base + A.off_w[2], L.d_model, L.d_ff, 1, P.L1.total, int(n_rec),
                               L.expert_stride, kR2, 1);
    if (rc != GALE_OK) return rc;
    rc = ensure_smem(reinterpret_cast<const void*>(moe_stream_kernel), kSmemBytes);
    if (rc != GALE_OK) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(sm_count()));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = size_t(kSmemBytes);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_stream_kernel, map13, map2, A, P) == cudaSuccess ? GALE_OK : GALE_ERR_CUDA;
}

}  // namespace gale

extern "C" int gale_debug_set_failure(uint64_t wait_limit_ns, int withhold_cta) {
    gale::g_wait_ns = wait_limit_ns ? wait_limit_ns : gale::kWaitNs;
    gale::g_withhold_cta = withhold_cta;
    return GALE_OK;
}

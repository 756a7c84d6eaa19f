// Tensor-core decode GEMV over GALE-1bit tiles (mma.sync m16n8k32, int8).
//
// For a row r and a 128-column block b the packed signs give
//     sum_c sign(r,c) x_c = X_b - 2 * P_b,   X_b = sum_{c in b} x_c,
//     P_b = sum_{c in b, bit(r,c) = 1} x_c,
// and the row result is  y_r = sum_b s_blk[r,b] (X_b - 2 P_b)  + outliers.
//
// P_b runs on the integer tensor cores.  The A operand is built from a sign
// word w with one AND per four weights: the int8 byte (w & (0x01010101 << s))
// of bit position s is bit * a(s), a(s) = 2^s for s < 7 and -128 for s = 7.
// The B operand holds the activation in fixed point, X_c = x_c * S / a(c mod 8)
// rounded to an integer (S a power of two with |X| <= 2^20), split into three
// int8 digits X = p1 * 2^14 + p2 * 2^7 + p3; the digits of a token are three
// MMA columns.  Products and int32 sums are exact; the only error is the
// fixed-point rounding of X (at most 2^-14 of max |x| per weight).
//
// Outlier columns keep their sign bit in the MMA part; their correction
// (q * s_row - sign * s_blk) * x_c is added separately.
//
// Digit storage of one vector of length C, per 128-column block b:
//   bytes [b][digit j (3)][tig (4)][32]: register q (0..7) of lane-quad tig is
//   bytes 4q..4q+3, byte i of it being column 128 b + 32 tig + 8 i + q.
// This is exactly the B fragment of MMA m = q/2 (b0 for even q, b1 for odd q)
// for the A fragment built from sign word tig of the block with s = q.
#pragma once
#include "common.cuh"
#include "ptx.cuh"
#include "tma.cuh"

namespace gale {

constexpr int kPieces = 3;
constexpr int kPieceBlockBytes = kPieces * 4 * 32;   // 384 bytes per 128 columns
constexpr int kWarpScratchFloats = 16 * 8;
constexpr float kFixedMax = 1048576.0f;              // |X| <= 2^20

// 1 / a(s)
__device__ __forceinline__ float inv_a(int s) { return s < 7 ? __int_as_float((127 - s) << 23) : -0.0078125f; }

// Largest power of two S with m * S <= 2^20 (m = max |x|); 1 when m == 0.
__device__ __forceinline__ float fixed_scale(float m) {
    if (!(m > 0.f)) return 1.0f;
    int e;
    frexpf(kFixedMax / m, &e);        // 2^20/m = f * 2^e, f in [0.5, 1)
    return ldexpf(1.0f, e - 1);       // 2^(e-1) <= 2^20 / m
}

// The three int8 digits of round(u), |u| <= 2^20, each in the low byte.
__device__ __forceinline__ void fixed_digits(float u, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
    // round(u) through the 1.5 * 2^23 addition: exact for |u| < 2^22 and
    // ties to even, the same as a round-to-nearest conversion
    const int X = __float_as_int(__fadd_rn(u, 12582912.0f)) - 0x4B400000;
    const int p1 = (X + 8192) >> 14;
    const int r = X - (p1 << 14);
    const int p2 = (r + 64) >> 7;
    const int p3 = r - (p2 << 7);
    d1 = uint32_t(p1) & 0xFFu;
    d2 = uint32_t(p2) & 0xFFu;
    d3 = uint32_t(p3) & 0xFFu;
}

// Build the digits and the 128-block sums of one rotated vector xr[0..C)
// held in shared memory.  Every thread of the CTA calls it (contains
// __syncthreads).  `red` is shared scratch of at least 33 floats.
// Returns 1/S (the reconstruction factor) on every thread.
__device__ inline float build_pieces(const float* xr, int C, uint8_t* pieces, float* xsum, float* red) {
    const int tid = threadIdx.x, nt = blockDim.x;
    float m = 0.f;
    for (int c = tid; c < C; c += nt) m = fmaxf(m, fabsf(xr[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
        float mm = 0.f;
        for (int w = 0; w < (nt + 31) / 32; ++w) mm = fmaxf(mm, red[w]);
        red[32] = fixed_scale(mm);
    }
    __syncthreads();
    const float S = red[32];
    for (int w = tid; w < C / 4; w += nt) {   // word positions (b, tig, q)
        const int q = w & 7, tig = (w >> 3) & 3, b = w >> 5;
        uint32_t word[kPieces] = {0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t d1, d2, d3;
            fixed_digits(xr[128 * b + 32 * tig + 8 * i + q] * S * inv_a(q), d1, d2, d3);
            word[0] |= d1 << (8 * i);
            word[1] |= d2 << (8 * i);
            word[2] |= d3 << (8 * i);
        }
        uint32_t* dst = reinterpret_cast<uint32_t*>(pieces + b * kPieceBlockBytes + tig * 32 + q * 4);
#pragma unroll
        for (int j = 0; j < kPieces; ++j) dst[j * 32] = word[j];   // digit stride 128 bytes
    }
    for (int b = tid; b < C / 128; b += nt) {
        float s = 0.f;
        for (int i = 0; i < 128; ++i) s += xr[128 * b + i];
        xsum[b] = s;
    }
    __syncthreads();
    return 1.0f / S;
}

// ---------------------------------------------------------------------------
// One 16-row tile of one matrix, staged in shared memory by TMA.
// ---------------------------------------------------------------------------

struct StageLayout {
    int signs, scales, idx, q, srow, bytes;   // byte offsets inside a stage, total
};

__host__ __device__ inline StageLayout stage_layout(int C) {
    StageLayout s;
    const int k = outliers_per_row(C);
    s.signs = 0;                                   // C/1024 boxes of 2 KB, 1024-aligned
    s.scales = 2 * C;                              // 16 rows x C/64 bytes
    s.idx = s.scales + 16 * (C / 64);              // 16 rows x k uint16
    s.q = s.idx + int(align_up(32 * k, 16));       // up to 8k nibble bytes + 16 alignment slack
    s.srow = s.q + int(align_up(8 * k + 16, 16));  // 16 row scales (32 bytes)
    s.bytes = int(align_up(s.srow + 32, 1024));
    return s;
}

// The token vectors a tile job multiplies: up to two tokens, each with its
// digits, 128-block sums, reconstruction factor 1/S and rotated values (fp32
// in global memory, or fp16 in shared memory) for the outliers.
struct TokRef {
    const uint8_t* pieces;   // nullptr: no token in this slot
    const float* xsum;
    const float* xr;         // fp32 rotated vector (global), or null
    float sigma;             // 1 / S
    const __half* x16;       // fp16 rotated vector (shared), or null
};

// Issue the TMA / bulk loads of tile (rows r0.., expert coordinate e) of a
// matrix into `stage` and arm `bar`.  Called by one lane.
__device__ inline void issue_tile(uint8_t* stage, uint64_t* bar, const CUtensorMap* smap, const CUtensorMap* bmap,
                                  const MatView& m, int e, int r0) {
    const StageLayout L = stage_layout(m.cols);
    const int nrows = min(16, m.rows - r0);
    const uint32_t idx_bytes = uint32_t(align_up(int64_t(nrows) * m.k * 2, 16));
    const int64_t q0 = int64_t(r0) * m.k / 2;                          // r0 % 16 == 0 -> even nibble
    const char* q_src = reinterpret_cast<const char*>(m.q) + q0;
    const int q_delta = int(reinterpret_cast<uintptr_t>(q_src) & 15);
    const uint32_t q_bytes = uint32_t(align_up(q_delta + (int64_t(nrows) * m.k + 1) / 2, 16));
    const uint32_t total = uint32_t(2 * m.cols + 16 * (m.cols / 64)) + (m.k ? idx_bytes + q_bytes : 0u);
    mbar_arrive_expect_tx(bar, total);
    for (int ch = 0; ch < m.cols / 1024; ++ch) tma_load_3d(stage + L.signs + ch * 2048, smap, bar, ch * 32, r0, e);
    tma_load_3d(stage + L.scales, bmap, bar, 0, r0, e);
    if (m.k) {
        bulk_load(stage + L.idx, m.idx + int64_t(r0) * m.k, idx_bytes, bar);
        bulk_load(stage + L.q, q_src - q_delta, q_bytes, bar);
    }
}

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const volatile uint32_t*>(p); }

// The four int8 A registers of MMA mm (0..3) from the sign words of rows g and
// g + 8: s = 2 mm for a0/a1, s = 2 mm + 1 for a2/a3.
__device__ __forceinline__ void a_regs(uint32_t wg, uint32_t wg8, int mm, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                       uint32_t& a3) {
    const uint32_t m0 = 0x01010101u << (2 * mm), m1 = m0 << 1;
    a0 = wg & m0;
    a1 = wg8 & m0;
    a2 = wg & m1;
    a3 = wg8 & m1;
}

// Compute one staged full-width tile for up to two tokens.  On return lanes
// 0..15 hold y[t] for row r0 + lane (t = 0, 1).  `scratch`: 128 floats of
// per-warp shared memory.  Used by the single-matrix GEMV entry point.
__device__ __forceinline__ void tile_compute(uint8_t* stage, const MatView& m, int r0, const TokRef (&tok)[2],
                                             float* scratch, float (&y)[2]) {
    const int lane = threadIdx.x & 31;
    const int C = m.cols, nb = C / 128, k = m.k;
    const StageLayout L = stage_layout(C);
    uint8_t* signs = stage + L.signs;
    const __half* sblk = reinterpret_cast<const __half*>(stage + L.scales);
    const uint16_t* idx = reinterpret_cast<const uint16_t*>(stage + L.idx);
    const int nrows = min(16, m.rows - r0);
    const int q_delta = int(reinterpret_cast<uintptr_t>(reinterpret_cast<const char*>(m.q) + int64_t(r0) * k / 2) & 15);
    const uint8_t* qn = stage + L.q + q_delta;

    // 1. outliers: (q * s_row - sign * s_blk) * x_c per token, lane (row, half)
    const int row = lane & 15, half = lane >> 4;
    float corr[2] = {0.f, 0.f};
    if (row < nrows && k) {
        const float srow = __half2float(m.s_row[r0 + row]);
        const int j0 = half ? (k + 1) / 2 : 0, j1 = half ? k : (k + 1) / 2;
        for (int j = j0; j < j1; ++j) {
            const int c = idx[row * k + j];
            if (c >= C) continue;   // only records that failed validation
            const int n = row * k + j;
            const int qb = qn[n >> 1];
            int qv = (n & 1) ? (qb >> 4) : (qb & 15);
            qv = qv >= 8 ? qv - 16 : qv;
            const int w = (c >> 5) & 31;
            const uint32_t word =
                lds32(signs + (c >> 10) * 2048 + row * 128 + (((w >> 2) ^ (row & 7)) << 4) + (w & 3) * 4);
            const float sb = __half2float(sblk[row * nb + (c >> 7)]);
            const float wq = fmaf(float(qv), srow, ((word >> (c & 31)) & 1u) ? sb : -sb);
#pragma unroll
            for (int t = 0; t < 2; ++t)
                if (tok[t].pieces) corr[t] = fmaf(wq, tok[t].xr[c], corr[t]);
        }
    }
    // 2. block-scale-weighted sums of x: sum_b s_blk[row, b] X_b, split in halves
    float xt[2] = {0.f, 0.f};
    {
        const int b0 = half ? nb / 2 : 0, b1 = half ? nb : nb / 2;
        for (int b = b0; b < b1; ++b) {
            const float s = __half2float(sblk[row * nb + b]);
#pragma unroll
            for (int t = 0; t < 2; ++t)
                if (tok[t].pieces) xt[t] = fmaf(s, tok[t].xsum[b], xt[t]);
        }
    }

    // 3. tensor-core loop over the 128-column blocks
    const int g = lane >> 2, tig = lane & 3;
    const uint8_t* src = nullptr;
    {
        const uint8_t* pc = g < 3 ? tok[0].pieces : tok[1].pieces;   // a select: no local-memory copy of tok
        if (g < 6 && pc) src = pc + (g % 3) * 128 + tig * 32;
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int b = 0; b < nb; ++b) {
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
        if (src) {
            q0 = *reinterpret_cast<const uint4*>(src + b * kPieceBlockBytes);
            q1 = *reinterpret_cast<const uint4*>(src + b * kPieceBlockBytes + 16);
        }
        const int ch = b >> 3, bb = b & 7;
        const int off = ch * 2048 + g * 128 + ((bb ^ (g & 7)) << 4) + tig * 4;
        const uint32_t wg = lds32(signs + off), wg8 = lds32(signs + off + 1024);
        const uint32_t breg[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        int c[4] = {0, 0, 0, 0};
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
            uint32_t a0, a1, a2, a3;
            a_regs(wg, wg8, mm, a0, a1, a2, a3);
            mma_s8(c, a0, a1, a2, a3, breg[2 * mm], breg[2 * mm + 1]);
        }
        const float sg = __half2float(sblk[g * nb + b]);
        const float sg8 = __half2float(sblk[(g + 8) * nb + b]);
        acc[0] = fmaf(sg, float(c[0]), acc[0]);
        acc[1] = fmaf(sg, float(c[1]), acc[1]);
        acc[2] = fmaf(sg8, float(c[2]), acc[2]);
        acc[3] = fmaf(sg8, float(c[3]), acc[3]);
    }
    // 4. epilogue: gather the 8 columns of every row through shared memory
    scratch[g * 8 + 2 * tig] = acc[0];
    scratch[g * 8 + 2 * tig + 1] = acc[1];
    scratch[(g + 8) * 8 + 2 * tig] = acc[2];
    scratch[(g + 8) * 8 + 2 * tig + 1] = acc[3];
    __syncwarp();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        float v = xt[t] + corr[t];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        const float* col = scratch + row * 8 + 3 * t;
        const float P = tok[t].pieces ? tok[t].sigma * (col[0] * 16384.0f + col[1] * 128.0f + col[2]) : 0.f;
        y[t] = v - 2.0f * P;
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Register layout of a warp-held 1024-block used for building digits: lane l
// register r holds element
//     (l & 7) + 8 (r & 3) + 32 (l >> 3) + 128 (r >> 2),
// so that lane l = q + 8 tig holds, in registers 4 bb .. 4 bb + 3, the four
// elements 128 bb + 32 tig + 8 i + q (i = 0..3) of digit word (bb, tig, q).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int piece_elem(int lane, int r) {
    return (lane & 7) + 8 * (r & 3) + 32 * (lane >> 3) + 128 * (r >> 2);
}

// Digits, the eight 128-block sums and the fp16 copy of one rotated
// 1024-block in the layout above (values already scaled by 1/32).
__device__ __forceinline__ void pieces_from_regs(const float (&v)[32], float S, uint8_t* pieces_blk,
                                                 float* xsum_blk, __half* x16_blk) {
    const int lane = threadIdx.x & 31;
    const int q = lane & 7, tig = lane >> 3;
    const float scale = S * inv_a(q);
#pragma unroll
    for (int r = 0; r < 32; ++r) x16_blk[piece_elem(lane, r)] = __float2half_rn(v[r]);
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) {
        const float s = warp_sum(v[4 * bb] + v[4 * bb + 1] + v[4 * bb + 2] + v[4 * bb + 3]);
        if (lane == 0) xsum_blk[bb] = s;
        uint32_t word[kPieces] = {0u, 0u, 0u};
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
            uint32_t d1, d2, d3;
            fixed_digits(v[4 * bb + i4] * scale, d1, d2, d3);
            word[0] |= d1 << (8 * i4);
            word[1] |= d2 << (8 * i4);
            word[2] |= d3 << (8 * i4);
        }
        uint32_t* dst = reinterpret_cast<uint32_t*>(pieces_blk + bb * kPieceBlockBytes + tig * 32 + q * 4);
#pragma unroll
        for (int j = 0; j < kPieces; ++j) dst[j * 32] = word[j];
    }
}

// Largest |x| over a warp-held block (all lanes get it).
__device__ __forceinline__ float block_absmax(const float (&v)[32]) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// Bytes that issue_tile_copies moves for tile (rows r0..) of matrix m.
__device__ __forceinline__ uint32_t tile_tx_bytes(const MatView& m, int r0) {
    const int nrows = min(16, m.rows - r0);
    const uint32_t idx_bytes = uint32_t(align_up(int64_t(nrows) * m.k * 2, 16));
    const char* q_src = reinterpret_cast<const char*>(m.q) + int64_t(r0) * m.k / 2;
    const int q_delta = int(reinterpret_cast<uintptr_t>(q_src) & 15);
    const uint32_t q_bytes = uint32_t(align_up(q_delta + (int64_t(nrows) * m.k + 1) / 2, 16));
    return uint32_t(2 * m.cols + 16 * (m.cols / 64)) + (m.k ? idx_bytes + q_bytes + 32u : 0u);
}

// The copies of issue_tile without arming the barrier (the caller arms it
// once for all the tiles of a job); the 16 row scales go to L.srow (32 bytes:
// the record continues past the section, so the copy stays inside it).
__device__ inline void issue_tile_copies(uint8_t* stage, uint64_t* bar, const CUtensorMap* smap,
                                         const CUtensorMap* bmap, const MatView& m, int e, int r0) {
    const StageLayout L = stage_layout(m.cols);
    const int nrows = min(16, m.rows - r0);
    for (int ch = 0; ch < m.cols / 1024; ++ch) tma_load_3d(stage + L.signs + ch * 2048, smap, bar, ch * 32, r0, e);
    tma_load_3d(stage + L.scales, bmap, bar, 0, r0, e);
    if (m.k) {
        const uint32_t idx_bytes = uint32_t(align_up(int64_t(nrows) * m.k * 2, 16));
        const char* q_src = reinterpret_cast<const char*>(m.q) + int64_t(r0) * m.k / 2;
        const int q_delta = int(reinterpret_cast<uintptr_t>(q_src) & 15);
        const uint32_t q_bytes = uint32_t(align_up(q_delta + (int64_t(nrows) * m.k + 1) / 2, 16));
        bulk_load(stage + L.idx, m.idx + int64_t(r0) * m.k, idx_bytes, bar);
        bulk_load(stage + L.q, q_src - q_delta, q_bytes, bar);
        bulk_load(stage + L.srow, m.s_row + r0, 32, bar);
    }
}

// One 1024-column chunk `ch` of a staged 16-row tile, for up to two tokens
// whose digits, sums and fp16 values live in shared memory.  On return lanes
// 0..15 hold the chunk's contribution to row r0 + lane for tokens 0 and 1:
//   sum_{b in chunk} s_blk (X_b - 2 P_b) + sum_{outliers in chunk} (q s_row - sign s_blk) x_c.
// Contributions of the chunks of a row add up to the row result.
__device__ __forceinline__ void chunk_compute(uint8_t* tile, const MatView& m, int r0, int ch,
                                              const TokRef (&tok)[2], float* scratch, float (&part)[2]) {
    const int lane = threadIdx.x & 31;
    const int C = m.cols, nb = C / 128, k = m.k;
    const StageLayout L = stage_layout(C);
    const uint32_t t_s = smem_u32(tile);
    const uint32_t signs_s = t_s + L.signs, sblk_s = t_s + L.scales, idx_s = t_s + L.idx;
    const int nrows = min(16, m.rows - r0);
    const int q_delta = int(reinterpret_cast<uintptr_t>(reinterpret_cast<const char*>(m.q) + int64_t(r0) * k / 2) & 15);
    const uint32_t qn_s = t_s + L.q + q_delta;
    const int row = lane & 15, half = lane >> 4;
    const bool has0 = tok[0].pieces != nullptr, has1 = tok[1].pieces != nullptr;
    const uint32_t x16_0 = has0 ? smem_u32(tok[0].x16) : 0u, x16_1 = has1 ? smem_u32(tok[1].x16) : 0u;

    // 1. outliers of this chunk: the row's columns are ascending, so the
    //    chunk's outliers are the range [lo, hi) found by binary search; the
    //    two half-warps split it.
    float corr0 = 0.f, corr1 = 0.f;
    if (row < nrows && k) {
        const uint32_t ri = idx_s + 2 * row * k;
        int a0 = 0, a1 = k;   // first j with idx >= 1024 ch
        while (a0 < a1) {
            const int mid = (a0 + a1) >> 1;
            if (int(lds_u16(ri + 2 * mid)) < (ch << 10)) a0 = mid + 1;
            else a1 = mid;
        }
        const int lo = a0;
        a1 = k;               // first j with idx >= 1024 (ch + 1)
        while (a0 < a1) {
            const int mid = (a0 + a1) >> 1;
            if (int(lds_u16(ri + 2 * mid)) < ((ch + 1) << 10)) a0 = mid + 1;
            else a1 = mid;
        }
        const int hi = a0;
        const int mid = (lo + hi + 1) >> 1;
        const int j0 = half ? mid : lo, j1 = half ? hi : mid;
        const float srow = __half2float(__ushort_as_half(uint16_t(lds_u16(t_s + L.srow + 2 * row))));
        for (int j = j0; j < j1; ++j) {
            const int c = int(lds_u16(ri + 2 * j));
            const int n = row * k + j;
            const int qb = int(lds_u8(qn_s + (n >> 1))) >> ((n & 1) * 4);
            const int qv = (qb & 15) - ((qb & 8) << 1);
            const int w = (c >> 5) & 31;
            const uint32_t word =
                lds_u32(signs_s + ch * 2048 + row * 128 + (((w >> 2) ^ (row & 7)) << 4) + (w & 3) * 4);
            const float sb = __half2float(__ushort_as_half(uint16_t(lds_u16(sblk_s + 2 * (row * nb + (c >> 7))))));
            const float wq = fmaf(float(qv), srow, ((word >> (c & 31)) & 1u) ? sb : -sb);
            if (has0) corr0 = fmaf(wq, __half2float(__ushort_as_half(uint16_t(lds_u16(x16_0 + 2 * c)))), corr0);
            if (has1) corr1 = fmaf(wq, __half2float(__ushort_as_half(uint16_t(lds_u16(x16_1 + 2 * c)))), corr1);
        }
    }
    // 2. block-scale-weighted 128-block sums of x over the chunk (4 blocks per half)
    float xt0 = 0.f, xt1 = 0.f;
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
        const int b = ch * 8 + half * 4 + bb;
        const float s = __half2float(__ushort_as_half(uint16_t(lds_u16(sblk_s + 2 * (row * nb + b)))));
        if (has0) xt0 = fmaf(s, tok[0].xsum[b], xt0);
        if (has1) xt1 = fmaf(s, tok[1].xsum[b], xt1);
    }

    // 3. tensor-core loop over the chunk's eight 128-column blocks
    const int g = lane >> 2, tig = lane & 3;
    const bool bsrc = g < 6 && (g < 3 ? has0 : has1);
    const uint32_t src = bsrc ? smem_u32(g < 3 ? tok[0].pieces : tok[1].pieces) + (g % 3) * 128 + tig * 32 : 0u;
    const uint32_t w_base = signs_s + ch * 2048 + g * 128 + tig * 4;
    const uint32_t sc_base = sblk_s + 2 * (ch * 8);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int bp = 0; bp < 4; ++bp) {
        int c2[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
        const uint32_t sc_g = lds_u32(sc_base + 2 * (g * nb + 2 * bp));
        const uint32_t sc_g8 = lds_u32(sc_base + 2 * ((g + 8) * nb + 2 * bp));
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int bb = 2 * bp + h2;
            uint4 q0 = make_uint4(0, 0, 0, 0), q1 = make_uint4(0, 0, 0, 0);
            if (bsrc) {
                const uint32_t a = src + (ch * 8 + bb) * kPieceBlockBytes;
                q0 = lds_v4(a);
                q1 = lds_v4(a + 16);
            }
            const uint32_t wa = w_base + ((bb ^ (g & 7)) << 4);
            const uint32_t wg = lds_u32(wa), wg8 = lds_u32(wa + 1024);
            const uint32_t breg[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                uint32_t a0, a1, a2, a3;
                a_regs(wg, wg8, mm, a0, a1, a2, a3);
                mma_s8(c2[h2], a0, a1, a2, a3, breg[2 * mm], breg[2 * mm + 1]);
            }
        }
        const float2 sg = __half22float2(*reinterpret_cast<const __half2*>(&sc_g));
        const float2 sg8 = __half22float2(*reinterpret_cast<const __half2*>(&sc_g8));
        acc[0] = fmaf(sg.x, float(c2[0][0]), fmaf(sg.y, float(c2[1][0]), acc[0]));
        acc[1] = fmaf(sg.x, float(c2[0][1]), fmaf(sg.y, float(c2[1][1]), acc[1]));
        acc[2] = fmaf(sg8.x, float(c2[0][2]), fmaf(sg8.y, float(c2[1][2]), acc[2]));
        acc[3] = fmaf(sg8.x, float(c2[0][3]), fmaf(sg8.y, float(c2[1][3]), acc[3]));
    }
    // 4. gather the 8 columns of every row through shared memory
    scratch[g * 8 + 2 * tig] = acc[0];
    scratch[g * 8 + 2 * tig + 1] = acc[1];
    scratch[(g + 8) * 8 + 2 * tig] = acc[2];
    scratch[(g + 8) * 8 + 2 * tig + 1] = acc[3];
    __syncwarp();
    {
        float v0 = xt0 + corr0, v1 = xt1 + corr1;
        v0 += __shfl_xor_sync(0xffffffffu, v0, 16);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 16);
        const float* col = scratch + row * 8;
        part[0] = has0 ? v0 - 2.0f * tok[0].sigma * (col[0] * 16384.0f + col[1] * 128.0f + col[2]) : 0.f;
        part[1] = has1 ? v1 - 2.0f * tok[1].sigma * (col[3] * 16384.0f + col[4] * 128.0f + col[5]) : 0.f;
    }
    __syncwarp();
}

}  // namespace gale

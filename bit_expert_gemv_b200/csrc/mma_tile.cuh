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
// digits, 128-block sums, reconstruction factor 1/S and, for the outliers,
// its rotated values (fp32 in global memory, or an fp16 copy of v S / 64 in
// shared memory).
struct TokRef {
    const uint8_t* pieces;   // nullptr: no token in this slot
    const float* xsum;
    const float* xr;         // fp32 rotated vector (global), or null
    float sigma;             // 1 / S
    const __half* x16;       // fp16 copy of the rotated vector times S / 64 (shared), or null
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

}  // namespace gale

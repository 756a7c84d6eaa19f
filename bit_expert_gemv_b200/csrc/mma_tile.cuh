// Tensor-core decode GEMV over GALE-1bit tiles (mma.sync m16n8k32, e4m3).
//
// For a row r and a 128-column block b the packed signs give
//     sum_c sign(r,c) x_c = X_b - 2 * P_b,   X_b = sum_{c in b} x_c,
//     P_b = sum_{c in b, bit(r,c) = 1} x_c,
// and the row result is  y_r = sum_b s_blk[r,b] (X_b - 2 P_b)  + outliers.
//
// P_b runs on the tensor cores.  The A operand is built from a sign word w
// with one AND per four weights: the e4m3 byte (w & (0x01010101 << s)) is
// bit * v(s), where v(s) is the e4m3 value of the byte 1 << s
// (2^-9, 2^-8, 2^-7, 2^-6, 2^-5, 2^-3, 2^1; bit 7 is shifted to bit 6, v = 2^1).
// The B operand holds x'_c = x_c / v(c mod 8), so A*B = bit * x_c exactly,
// split into three e4m3 pieces x'/sigma ~ p1 + p2/16 + p3/256 (about 12
// significant bits); the three pieces of a token are three MMA columns.
//
// Outlier columns are removed from the MMA by clearing their sign bits in
// shared memory after the tile lands, and added back as q * s_row * x_c.
//
// Piece storage of one vector of length C, per 128-column block b:
//   bytes [b][piece j (3)][tig (4)][32]: register q (0..7) of lane-quad tig is
//   bytes 4q..4q+3, byte i of it being column 128 b + 32 tig + 8 i + q.
// This is exactly the B fragment of MMA m = q/2 (b0 for even q, b1 for odd q)
// for the A fragment built from sign word tig of the block with s = q.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tma.cuh"

namespace gale {

constexpr int kPieces = 3;
constexpr int kPieceBlockBytes = kPieces * 4 * 32;   // 384 bytes per 128 columns
constexpr int kWarpScratchFloats = 16 * 8;

__device__ __forceinline__ float inv_v(int s) {
    // 1 / v(s) for the AND-mask operand values above
    return s < 5 ? float(512 >> s) : (s == 5 ? 8.0f : 0.5f);
}

__device__ __forceinline__ uint8_t to_e4m3(float v) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float from_e4m3(uint8_t p) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(p), __NV_E4M3);
    return __half2float(__half(h));
}

// Smallest power of two sigma with m / sigma <= 448 (the e4m3 maximum).
__device__ __forceinline__ float piece_sigma(float m) {
    if (!(m > 0.f)) return 1.0f;
    int e;
    frexpf(m / 448.0f, &e);           // m/448 = f * 2^e, f in [0.5, 1)
    float s = ldexpf(1.0f, e);
    if (m / s > 448.0f) s *= 2.0f;
    if (m / (0.5f * s) <= 448.0f) s *= 0.5f;
    return s;
}

// Build the pieces and the 128-block sums of one rotated vector xr[0..C)
// held in shared memory.  Every thread of the CTA calls it (contains
// __syncthreads).  `red` is shared scratch of at least 33 floats.
// Returns sigma on every thread.
__device__ inline float build_pieces(const float* xr, int C, uint8_t* pieces, float* xsum, float* red) {
    const int tid = threadIdx.x, nt = blockDim.x;
    float m = 0.f;
    for (int c = tid; c < C; c += nt) m = fmaxf(m, fabsf(xr[c] * inv_v(c & 7)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
        float mm = 0.f;
        for (int w = 0; w < (nt + 31) / 32; ++w) mm = fmaxf(mm, red[w]);
        red[32] = piece_sigma(mm);
    }
    __syncthreads();
    const float sigma = red[32];
    const float inv_sigma = 1.0f / sigma;   // power of two: exact
    // one thread per output word position (b, tig, q): 4 columns, 3 pieces
    const int n_words = C / 4;   // word positions (b, tig, q)
    for (int w = tid; w < n_words; w += nt) {
        const int q = w & 7, tig = (w >> 3) & 3, b = w >> 5;
        uint32_t word[kPieces] = {0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = 128 * b + 32 * tig + 8 * i + q;
            float u = xr[c] * inv_v(q) * inv_sigma;
#pragma unroll
            for (int j = 0; j < kPieces; ++j) {
                const uint8_t p = to_e4m3(u);
                word[j] |= uint32_t(p) << (8 * i);
                u = (u - from_e4m3(p)) * 16.0f;
            }
        }
        uint32_t* dst = reinterpret_cast<uint32_t*>(pieces + b * kPieceBlockBytes + tig * 32 + q * 4);
#pragma unroll
        for (int j = 0; j < kPieces; ++j) dst[j * 32] = word[j];   // piece stride 128 bytes
    }
    for (int b = tid; b < C / 128; b += nt) {
        float s = 0.f;
        for (int i = 0; i < 128; ++i) s += xr[128 * b + i];
        xsum[b] = s;
    }
    __syncthreads();
    return sigma;
}

// ---------------------------------------------------------------------------
// One 16-row tile of one matrix, staged in shared memory by TMA.
// ---------------------------------------------------------------------------

struct StageLayout {
    int signs, scales, idx, q, bytes;   // byte offsets inside a stage, total
};

__host__ __device__ inline StageLayout stage_layout(int C) {
    StageLayout s;
    const int k = outliers_per_row(C);
    s.signs = 0;                                   // C/1024 boxes of 2 KB, 1024-aligned
    s.scales = 2 * C;                              // 16 rows x C/64 bytes
    s.idx = s.scales + 16 * (C / 64);              // 16 rows x k uint16
    s.q = s.idx + int(align_up(32 * k, 16));       // up to 8k nibble bytes + 16 alignment slack
    s.bytes = int(align_up(s.q + int(align_up(8 * k + 16, 16)), 1024));
    return s;
}

// The token vectors a tile job multiplies: up to two tokens, each with its
// pieces, 128-block sums, sigma and fp32 rotated values (for the outliers).
struct TokRef {
    const uint8_t* pieces;   // nullptr: no token in this slot
    const float* xsum;
    const float* xr;
    float sigma;
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

// Compute one staged tile for up to two tokens.  On return lanes 0..15 hold
// y[t] for row r0 + lane (t = 0, 1); lanes 16..31 hold garbage.
// `scratch`: 128 floats of per-warp shared memory.
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

    // 1. outliers: clear their sign bits (MMA sees 0 there) and accumulate
    //    q * x_c per token; lane (row = lane & 15, half = lane >> 4)
    const int row = lane & 15, half = lane >> 4;
    float corr[2] = {0.f, 0.f};
    if (row < nrows) {
        const int j0 = half ? (k + 1) / 2 : 0, j1 = half ? k : (k + 1) / 2;
        for (int j = j0; j < j1; ++j) {
            const int c = idx[row * k + j];
            if (c >= C) continue;   // only records that failed validation
            const int n = row * k + j;
            const int qb = qn[n >> 1];
            int qv = (n & 1) ? (qb >> 4) : (qb & 15);
            qv = qv >= 8 ? qv - 16 : qv;
            const int w = (c >> 5) & 31;
            const int off = (c >> 10) * 2048 + row * 128 + ((((w >> 2) ^ (row & 7))) << 4) + (w & 3) * 4;
            atomicAnd(reinterpret_cast<unsigned int*>(signs + off), ~(1u << (c & 31)));
#pragma unroll
            for (int t = 0; t < 2; ++t)
                if (tok[t].pieces) corr[t] = fmaf(float(qv), tok[t].xr[c], corr[t]);
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
    __syncwarp();

    // 3. tensor-core loop over the 128-column blocks
    const int g = lane >> 2, tig = lane & 3;
    const uint8_t* src = nullptr;
    if (g < 6 && tok[g / 3].pieces) src = tok[g / 3].pieces + (g % 3) * 128 + tig * 32;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint4 bq0 = make_uint4(0, 0, 0, 0), bq1 = make_uint4(0, 0, 0, 0);
    if (src) {
        bq0 = *reinterpret_cast<const uint4*>(src);
        bq1 = *reinterpret_cast<const uint4*>(src + 16);
    }
    for (int b = 0; b < nb; ++b) {
        uint4 nq0 = make_uint4(0, 0, 0, 0), nq1 = make_uint4(0, 0, 0, 0);
        if (src && b + 1 < nb) {
            nq0 = *reinterpret_cast<const uint4*>(src + (b + 1) * kPieceBlockBytes);
            nq1 = *reinterpret_cast<const uint4*>(src + (b + 1) * kPieceBlockBytes + 16);
        }
        const int ch = b >> 3, bb = b & 7;
        const int off = ch * 2048 + g * 128 + ((bb ^ (g & 7)) << 4) + tig * 4;
        const uint32_t wg = lds32(signs + off), wg8 = lds32(signs + off + 1024);
        const uint32_t breg[8] = {bq0.x, bq0.y, bq0.z, bq0.w, bq1.x, bq1.y, bq1.z, bq1.w};
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
            const uint32_t m0 = 0x01010101u << (2 * mm);
            const uint32_t a0 = wg & m0, a1 = wg8 & m0;
            uint32_t a2, a3;
            if (mm == 3) {
                a2 = (wg >> 1) & 0x40404040u;
                a3 = (wg8 >> 1) & 0x40404040u;
            } else {
                a2 = wg & (m0 << 1);
                a3 = wg8 & (m0 << 1);
            }
            mma_e4m3(c, a0, a1, a2, a3, breg[2 * mm], breg[2 * mm + 1]);
        }
        const float sg = __half2float(sblk[g * nb + b]);
        const float sg8 = __half2float(sblk[(g + 8) * nb + b]);
        acc[0] = fmaf(sg, c[0], acc[0]);
        acc[1] = fmaf(sg, c[1], acc[1]);
        acc[2] = fmaf(sg8, c[2], acc[2]);
        acc[3] = fmaf(sg8, c[3], acc[3]);
        bq0 = nq0;
        bq1 = nq1;
    }
    // 4. epilogue: gather the 8 columns of every row through shared memory
    scratch[g * 8 + 2 * tig] = acc[0];
    scratch[g * 8 + 2 * tig + 1] = acc[1];
    scratch[(g + 8) * 8 + 2 * tig] = acc[2];
    scratch[(g + 8) * 8 + 2 * tig + 1] = acc[3];
    __syncwarp();
    const float srow = k ? __half2float(m.s_row[min(r0 + row, m.rows - 1)]) : 0.f;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        float v = xt[t] + srow * corr[t];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        const float* col = scratch + row * 8 + 3 * t;
        const float P = tok[t].pieces ? tok[t].sigma * (col[0] + col[1] * 0.0625f + col[2] * 0.00390625f) : 0.f;
        y[t] = v - 2.0f * P;
    }
    __syncwarp();
}

}  // namespace gale

// 4-bit weights of the non-expert matrices (W4, g128): symmetric int4 codes
// with one fp16 scale per 128-column block of a row, as the
// DeepSeek-V4-Pro-671B-GALE-1bit-v4 card describes them (paragraph under the
// weights table), kept 4-bit in VRAM as the DeepSeek-V4-Flash card's
// "What is in the pack" table says for attention, shared experts and head.
//
// Readings (the pages leave them open): codes q in [-7, 7], s = amax / 7 per
// block (amax / 7 in fp32, rounded to fp16), q = rint(w / s) in fp32 with
// ties to even, clamped; a block of zeros has s = 0 and q = 0.  Storage:
// [rows][cols / 2] bytes of two's complement nibbles (low nibble = even
// column), then fp16 scales [rows][cols / 128], each section 256-byte aligned.
//
// GEMV (decode, 1..8 tokens).  y[t, r] = sum_c s(r, c / 128) q(r, c) x(t, c).
// The weights are streamed once with 16-byte loads and fed, still packed, to
// the int8 tensor cores: a 32-bit word of eight nibbles gives two A registers
// of (q + 8) as unsigned bytes, (w & 0x0F0F0F0F) ^ 0x08080808 and the same of
// w >> 4, one LOP3 each.  The activations are prepared once per call in fixed
// point: per 1024-column chunk a power-of-two S with max |x S| <= 2^20,
// X = rint(x S) as three balanced int8 digits (X = 2^14 d1 + 2^7 d2 + d3).  A
// block's MMA sum over (q + 8) X is corrected exactly in int32 by the block
// sum of X (times 8), then scaled by s in fp32; 1/S is applied per chunk.
// MMA columns hold two tokens x three digits, so 1..8 tokens are up to four
// column groups over the same A registers (weights read once).
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace gale {

namespace {

constexpr int kW4Block = 128;
constexpr int kW4Chunk = 1024;
constexpr int kW4Rows = 16;       // rows of a CTA tile
constexpr int kW4MaxStages = 4;   // shared-memory stages per warp (fewer when the activations need room)
constexpr int kW4KBlk = 4;        // 128-column blocks per streamed unit
constexpr int kW4UnitW = kW4Rows * kW4KBlk * 64;            // code bytes of a unit (4 KB)
constexpr int kW4UnitBytes = kW4UnitW + kW4Rows * kW4KBlk * 2;   // + scales (128 B)
constexpr int kW4SmemMax = 227 * 1024;

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// One warp per (row, 128-column block): lane l quantizes columns 4l .. 4l + 3.
__global__ void __launch_bounds__(256) w4_quantize_kernel(const float* __restrict__ w, int64_t rows, int64_t cols,
                                                         uint8_t* __restrict__ q, __half* __restrict__ s) {
    const int64_t nb = cols / kW4Block;
    const int64_t item = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (item >= rows * nb) return;
    const int lane = threadIdx.x & 31;
    const int64_t r = item / nb, b = item - r * nb;
    const float4 v = *reinterpret_cast<const float4*>(w + r * cols + b * kW4Block + 4 * lane);
    const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    const __half sh = __float2half_rn(__fdiv_rn(amax, 7.0f));
    const float sf = __half2float(sh);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int c = 0;
        if (sf > 0.f) c = max(-7, min(7, int(rintf(__fdiv_rn(vv[i], sf)))));
        packed |= (uint32_t(c) & 0xFu) << (4 * i);
    }
    *reinterpret_cast<uint16_t*>(q + r * (cols / 2) + b * (kW4Block / 2) + 2 * lane) = uint16_t(packed);
    if (lane == 0) s[r * nb + b] = sh;
}

// Activation digits of one (token, 1024-column chunk) per warp.  Lane
// l = 8 tig + 2 i + par writes, for each block bb of the chunk and digit j,
// the word of the four columns 128 bb + 32 tig + 8 i + 2 e + par (e = 0..3),
// at xd + ((t * 3 + j) * nblk + block) * 128 + tig * 32 + i * 8 + par * 4:
// the B fragment of MMA i for the lanes of quad index tig.
__global__ void __launch_bounds__(256) w4_xprep_kernel(const uint16_t* __restrict__ x, int B, int64_t cols,
                                                      uint8_t* __restrict__ xd, int32_t* __restrict__ xsum,
                                                      float* __restrict__ xsig) {
    const int64_t nch = cols / kW4Chunk, nblk = cols / kW4Block;
    const int64_t item = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (item >= int64_t(B) * nch) return;
    const int lane = threadIdx.x & 31;
    const int t = int(item / nch);
    const int64_t ch = item - int64_t(t) * nch;
    const int tig = lane >> 3, i = (lane >> 1) & 3, par = lane & 1;
    const uint16_t* xs = x + int64_t(t) * cols + ch * kW4Chunk + 32 * tig + 8 * i + par;
    float v[8][4];
    float m = 0.f;
#pragma unroll
    for (int bb = 0; bb < 8; ++bb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[bb][e] = bf16_to_f32(__ldg(xs + 128 * bb + 2 * e));
            m = fmaxf(m, fabsf(v[bb][e]));
        }
    m = warp_max(m);
    // largest power of two S with m S <= 2^20 (1 for a zero chunk; at most 2^100)
    float S = 1.0f;
    if (m > 0.f) {
        int e2;
        frexpf(m, &e2);                       // m = f 2^e2, 0.5 <= f < 1
        S = ldexpf(1.0f, min(20 - e2, 100));  // m S < 2^20
    }
#pragma unroll
    for (int bb = 0; bb < 8; ++bb) {
        uint32_t wd[3] = {0u, 0u, 0u};
        int sx = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int X = __float2int_rn(v[bb][e] * S);
            sx += X;
            const int d1 = (X + 8192) >> 14;
            const int r = X - (d1 << 14);
            const int d2 = (r + 64) >> 7;
            const int d3 = r - (d2 << 7);
            wd[0] |= (uint32_t(d1) & 0xFFu) << (8 * e);
            wd[1] |= (uint32_t(d2) & 0xFFu) << (8 * e);
            wd[2] |= (uint32_t(d3) & 0xFFu) << (8 * e);
        }
        const int64_t blk = ch * 8 + bb;
#pragma unroll
        for (int j = 0; j < 3; ++j)
            *reinterpret_cast<uint32_t*>(xd + ((int64_t(t) * 3 + j) * nblk + blk) * 128 + tig * 32 + i * 8 + par * 4) =
                wd[j];
        const int tot = __reduce_add_sync(0xffffffffu, sx);
        if (lane == 0) xsum[int64_t(t) * nblk + blk] = tot;
    }
    if (lane == 0) xsig[int64_t(t) * nch + ch] = 1.0f / S;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// wait until at most n - 1 groups of this thread are pending (n = 2..4)
__device__ __forceinline__ void cp_wait_stages(int n) {
    if (n == 4) asm volatile("cp.async.wait_group 3;" ::: "memory");
    else if (n == 3) asm volatile("cp.async.wait_group 2;" ::: "memory");
    else asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Persistent GEMV: every warp owns whole 16-row tiles (tile = global warp +
// k x all warps) and streams each tile in units of four 128-column blocks
// (4 KB of codes + 128 B of scales) through its own ring of `nst` shared-memory
// stages, filled with 16-byte asynchronous copies nst - 1 units ahead of the
// arithmetic.  In a stage, row r's 16-byte chunk c (block c / 4, quad lane
// c % 4) sits at chunk c ^ (r & 7) of the row's 256 bytes, so the eight rows
// a load touches fall in eight different bank groups.  The activation digits
// of all 2 NP tokens are copied into shared memory once (one block-wide
// barrier at the start), rows of (token, digit) `xpitch` bytes apart.  NP
// column groups of two tokens (tokens 2p, 2p + 1) share the A registers of a
// block.
template <int NP, int NW>
__global__ void __launch_bounds__(NW * 32, 1) w4_gemv_kernel(const uint8_t* __restrict__ q,
                                                             const __half* __restrict__ s, int64_t cols, int B,
                                                             const uint8_t* __restrict__ xd,
                                                             const int32_t* __restrict__ xsum,
                                                             const float* __restrict__ xsig, float* __restrict__ y,
                                                             int64_t rows, int nst, int xpitch) {
    extern __shared__ __align__(16) uint8_t w4_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, tig = lane & 3;
    const int nblk = int(cols / kW4Block), nch = int(cols / kW4Chunk);
    const int nk = nblk / kW4KBlk;                            // units per tile
    const int64_t ntiles = rows / kW4Rows;
    const int64_t gw = int64_t(blockIdx.x) * NW + warp, nw = int64_t(gridDim.x) * NW;
    const int64_t my_tiles = gw < ntiles ? (ntiles - gw + nw - 1) / nw : 0;
    const uint32_t ring = smem_u32(w4_smem) + uint32_t(warp * nst * kW4UnitBytes);
    const uint32_t xs = smem_u32(w4_smem) + uint32_t(NW * nst * kW4UnitBytes);
    const int swz = g & 7;
    const int64_t rowb = cols / 2;                            // code bytes of a row
    // the activation digits, once: 6 NP rows of cols bytes
    {
        const int nrow = 6 * NP, per_row = int(cols / 16);
        for (int i = threadIdx.x; i < nrow * per_row; i += blockDim.x) {
            const int r = i / per_row, c = i - r * per_row;
            cp_async16(xs + uint32_t(r * xpitch + 16 * c), xd + int64_t(r) * cols + 16 * c);
        }
        cp_commit();
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
    }
    if (my_tiles == 0) return;

    // issue pointer: (tile i_t, unit i_k) into stage i_s; this lane's own chunks
    int64_t i_t = 0;
    int i_k = 0, i_s = 0;
    auto issue_next = [&]() {
        if (i_t < my_tiles) {
            const int64_t r0 = (gw + i_t * nw) * kW4Rows;
            const uint32_t base = ring + uint32_t(i_s * kW4UnitBytes);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = g + 8 * h;
                const uint8_t* src = q + (r0 + row) * rowb + 64 * (i_k * kW4KBlk) + 16 * tig;
#pragma unroll
                for (int j = 0; j < kW4KBlk; ++j)
                    cp_async16(base + uint32_t(row * 256 + (((4 * j + tig) ^ swz) << 4)), src + 64 * j);
                if (tig == 0) cp_async8(base + uint32_t(kW4UnitW + row * 8), s + (r0 + row) * nblk + i_k * kW4KBlk);
            }
            if (++i_k == nk) {
                i_k = 0;
                ++i_t;
            }
            if (++i_s == nst) i_s = 0;
        }
        cp_commit();
    };
#pragma unroll 1
    for (int i = 0; i < nst - 1; ++i) issue_next();
    // B fragment of this lane: column g = (token g / 3 of the group, digit g % 3); 6, 7 unused
    const bool bl = g < 6;
    const int tk = g / 3, dg = g % 3;
    // the lanes holding a token's d3 column take the 8 X_b correction
    const int cor = tig == 1 ? 0 : (tig == 2 ? 1 : -1);     // which of the lane's two columns
    const int ctok = tig == 2 ? 1 : 0;                      // its token within the group
    // tokens of the lane's two columns n = 2 tig, 2 tig + 1
    const int tc0 = (2 * tig) / 3, tc1 = (2 * tig + 1) / 3;
    // digits -> value: token 0 = 2^14 n0 + 2^7 n1 + n2, token 1 = 2^14 n3 + 2^7 n4 + n5
    const float wa = tig == 0 ? 16384.0f : tig == 1 ? 1.0f : tig == 2 ? 128.0f : 0.f;    // weight of column 2 tig
    const float wc = tig == 0 ? 128.0f : tig == 1 ? 16384.0f : tig == 2 ? 1.0f : 0.f;    // of column 2 tig + 1
    const uint32_t xrow = xs + uint32_t((tk * 3 + dg) * xpitch + tig * 32);
    float acc[NP][4], tot[NP][4];
    int c_s = 0;
#pragma unroll 1
    for (int64_t t_i = 0; t_i < my_tiles; ++t_i) {
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[p][i] = tot[p][i] = 0.f;
#pragma unroll 1
        for (int kc = 0; kc < nk; ++kc) {
            issue_next();
            cp_wait_stages(nst);
            __syncwarp();
            const uint32_t base = ring + uint32_t(c_s * kW4UnitBytes);
            if (++c_s == nst) c_s = 0;
#pragma unroll
            for (int j = 0; j < kW4KBlk; ++j) {
                const int b = kc * kW4KBlk + j;
                const uint32_t co = uint32_t(((4 * j + tig) ^ swz) << 4);
                const uint4 ua = lds_v4(base + uint32_t(g * 256) + co);
                const uint4 ub = lds_v4(base + uint32_t((g + 8) * 256) + co);
                const float s0 =
                    __half2float(__ushort_as_half(uint16_t(lds_u16(base + uint32_t(kW4UnitW + g * 8 + 2 * j)))));
                const float s1 =
                    __half2float(__ushort_as_half(uint16_t(lds_u16(base + uint32_t(kW4UnitW + (g + 8) * 8 + 2 * j)))));
                const uint32_t wa4[4] = {ua.x, ua.y, ua.z, ua.w}, wb4[4] = {ub.x, ub.y, ub.z, ub.w};
                uint32_t lo[4], lo8[4], hi[4], hi8[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    lo[i] = (wa4[i] & 0x0F0F0F0Fu) ^ 0x08080808u;
                    hi[i] = ((wa4[i] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
                    lo8[i] = (wb4[i] & 0x0F0F0F0Fu) ^ 0x08080808u;
                    hi8[i] = ((wb4[i] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
                }
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (bl) {
                        const uint32_t xb = xrow + uint32_t(6 * p * xpitch + b * 128);
                        x0 = lds_v4(xb);
                        x1 = lds_v4(xb + 16);
                    }
                    // two independent MMA chains (columns of words 0, 1 and 2, 3)
                    int ca[4] = {0, 0, 0, 0}, cb[4] = {0, 0, 0, 0};
                    mma_u8s8(ca, lo[0], lo8[0], hi[0], hi8[0], x0.x, x0.y);
                    mma_u8s8(cb, lo[2], lo8[2], hi[2], hi8[2], x1.x, x1.y);
                    mma_u8s8(ca, lo[1], lo8[1], hi[1], hi8[1], x0.z, x0.w);
                    mma_u8s8(cb, lo[3], lo8[3], hi[3], hi8[3], x1.z, x1.w);
                    int cc[4] = {ca[0] + cb[0], ca[1] + cb[1], ca[2] + cb[2], ca[3] + cb[3]};
                    if (cor >= 0) {
                        const int xb8 = 8 * __ldg(xsum + (2 * p + ctok) * nblk + b);
                        cc[cor] -= xb8;
                        cc[cor + 2] -= xb8;
                    }
                    acc[p][0] = fmaf(s0, float(cc[0]), acc[p][0]);
                    acc[p][1] = fmaf(s0, float(cc[1]), acc[p][1]);
                    acc[p][2] = fmaf(s1, float(cc[2]), acc[p][2]);
                    acc[p][3] = fmaf(s1, float(cc[3]), acc[p][3]);
                }
            }
            __syncwarp();
            // a 1024-column chunk is two units: its sums take 1/S of each column's token
            if (kc & 1) {
                const int ch = kc / 2;
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    const float f0 = tc0 < 2 ? __ldg(xsig + (2 * p + tc0) * nch + ch) : 0.f;
                    const float f1 = tc1 < 2 ? __ldg(xsig + (2 * p + tc1) * nch + ch) : 0.f;
                    tot[p][0] = fmaf(f0, acc[p][0], tot[p][0]);
                    tot[p][1] = fmaf(f1, acc[p][1], tot[p][1]);
                    tot[p][2] = fmaf(f0, acc[p][2], tot[p][2]);
                    tot[p][3] = fmaf(f1, acc[p][3], tot[p][3]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[p][i] = 0.f;
                }
            }
        }
        // sums over the lane quad, then lane (g, tig) writes row g + 8 (tig >> 1), token tig & 1
        const int64_t r0 = (gw + t_i * nw) * kW4Rows;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float v[2][2];   // [row g, g + 8][token]
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float a = wa * tot[p][2 * h], c = wc * tot[p][2 * h + 1];
                float t0v = (tc0 == 0 ? a : 0.f) + (tc1 == 0 ? c : 0.f);
                float t1v = (tc0 == 1 ? a : 0.f) + (tc1 == 1 ? c : 0.f);
                t0v += __shfl_xor_sync(0xffffffffu, t0v, 1);
                t0v += __shfl_xor_sync(0xffffffffu, t0v, 2);
                t1v += __shfl_xor_sync(0xffffffffu, t1v, 1);
                t1v += __shfl_xor_sync(0xffffffffu, t1v, 2);
                v[h][0] = t0v;
                v[h][1] = t1v;
            }
            const int t = 2 * p + (tig & 1);
            if (t < B) y[int64_t(t) * rows + r0 + g + 8 * (tig >> 1)] = v[tig >> 1][tig & 1];
        }
    }
    cp_wait_all();
}

}  // namespace

}  // namespace gale

extern "C" int gale_w4_layout(int64_t rows, int64_t cols, gale_w4_layout_t* out) {
    if (!out || rows < 1 || cols < gale::kW4Block || cols % gale::kW4Block) return GALE_ERR_ARG;
    out->rows = rows;
    out->cols = cols;
    out->q_offset = 0;
    out->q_bytes = rows * cols / 2;
    out->s_offset = gale::align_up(out->q_bytes, 256);
    out->s_bytes = rows * (cols / gale::kW4Block) * 2;
    out->total = gale::align_up(out->s_offset + out->s_bytes, 256);
    return GALE_OK;
}

extern "C" int gale_w4_quantize(const float* w, int64_t rows, int64_t cols, void* packed, void* stream) {
    gale_w4_layout_t L;
    if (gale_w4_layout(rows, cols, &L) != GALE_OK || !w || !packed) return GALE_ERR_ARG;
    if (!gale::aligned(w, 16) || !gale::aligned(packed, 256)) return GALE_ERR_ALIGN;
    const int64_t warps = rows * (cols / gale::kW4Block);
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks > 0x7FFFFFFF) return GALE_ERR_UNSUPPORTED;
    uint8_t* base = static_cast<uint8_t*>(packed);
    gale::w4_quantize_kernel<<<unsigned(blocks), 256, 0, gale::as_stream(stream)>>>(
        w, rows, cols, base, reinterpret_cast<__half*>(base + L.s_offset));
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

namespace {
// workspace: digits [Bp][3][cols], block sums [Bp][cols/128], 1/S [Bp][cols/1024]
struct W4Ws {
    uint8_t* xd;
    int32_t* xsum;
    float* xsig;
    int64_t bytes;
};
W4Ws carve_w4_ws(void* ws, int64_t cols, int B) {
    const int64_t bp = B + (B & 1);
    char* p = static_cast<char*>(ws);
    W4Ws w{};
    int64_t o = 0;
    w.xd = reinterpret_cast<uint8_t*>(p ? p + o : nullptr);
    o = gale::align_up(o + bp * 3 * cols, 256);
    w.xsum = reinterpret_cast<int32_t*>(p ? p + o : nullptr);
    o = gale::align_up(o + bp * (cols / 128) * 4, 256);
    w.xsig = reinterpret_cast<float*>(p ? p + o : nullptr);
    o = gale::align_up(o + bp * (cols / 1024) * 4, 256);
    w.bytes = o;
    return w;
}
bool w4_gemv_shape_ok(int64_t rows, int64_t cols, int B) {
    return rows >= 16 && rows % 16 == 0 && cols >= 1024 && cols % 1024 == 0 && B >= 1 && B <= 8 &&
           rows / 16 <= 0x7FFFFFFF;
}
}  // namespace

extern "C" size_t gale_w4_workspace_size(int64_t rows, int64_t cols, int B) {
    if (!w4_gemv_shape_ok(rows, cols, B)) return 0;
    return size_t(carve_w4_ws(nullptr, cols, B).bytes);
}

extern "C" int gale_w4_gemv(const void* packed, int64_t rows, int64_t cols, const uint16_t* x, int B, float* y,
                            void* ws, size_t ws_bytes, void* stream) {
    if (!w4_gemv_shape_ok(rows, cols, B) || !packed || !x || !y) return GALE_ERR_ARG;
    if (!gale::aligned(packed, 256) || !gale::aligned(x, 2) || !gale::aligned(y, 4)) return GALE_ERR_ALIGN;
    const W4Ws w = carve_w4_ws(ws, cols, B);
    if (!ws || ws_bytes < size_t(w.bytes)) return GALE_ERR_WORKSPACE;
    if (!gale::aligned(ws, 256)) return GALE_ERR_ALIGN;
    gale_w4_layout_t L;
    gale_w4_layout(rows, cols, &L);
    cudaStream_t st = gale::as_stream(stream);
    if (B & 1) {   // the unused token of the last column group reads zeros
        const int64_t bp = B + 1;
        if (cudaMemsetAsync(w.xd + int64_t(B) * 3 * cols, 0, size_t(3 * cols), st) != cudaSuccess ||
            cudaMemsetAsync(w.xsum + int64_t(B) * (cols / 128), 0, size_t(cols / 128 * 4), st) != cudaSuccess ||
            cudaMemsetAsync(w.xsig + int64_t(B) * (cols / 1024), 0, size_t(cols / 1024 * 4), st) != cudaSuccess)
            return GALE_ERR_CUDA;
        (void)bp;
    }
    const int64_t warps = int64_t(B) * (cols / 1024);
    gale::w4_xprep_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, st>>>(x, B, cols, w.xd, w.xsum, w.xsig);
    GALE_LAUNCH_CHECK();
    const uint8_t* qb = static_cast<const uint8_t*>(packed);
    const __half* sb = reinterpret_cast<const __half*>(qb + L.s_offset);
    const int np = (B + 1) / 2;
    // shared memory: the activation digits of 2 np tokens, then the ring
    // stages of the 8 warps, as many (2..4) as fit (16 warps with fewer stages
    // each measured slower on the [65536 x 4096] case: 80 against 71 us)
    const int xpitch = int(cols) + 16;
    const int xbytes = 6 * np * xpitch;
    auto stages_for = [&](int warps) {
        int n = gale::kW4MaxStages;
        while (n >= 2 && xbytes + warps * n * gale::kW4UnitBytes > gale::kW4SmemMax) --n;
        return n;
    };
    const int nw = 8;
    const int nst = stages_for(nw);
    if (nst < 2) return GALE_ERR_UNSUPPORTED;
    const int smem = xbytes + nw * nst * gale::kW4UnitBytes;
    const int64_t ctas = (rows / 16 + nw - 1) / nw;
    const unsigned grid = unsigned(ctas < gale::sm_count() ? ctas : gale::sm_count());
    auto launch = [&](auto kern) {
        // (set on every call: the attribute belongs to the current device)
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return false;
        kern<<<grid, nw * 32, smem, st>>>(qb, sb, cols, B, w.xd, w.xsum, w.xsig, y, rows, nst, xpitch);
        return true;
    };
    bool ok = false;
    if (np == 1) ok = launch(gale::w4_gemv_kernel<1, 8>);
    else if (np == 2) ok = launch(gale::w4_gemv_kernel<2, 8>);
    else if (np == 3) ok = launch(gale::w4_gemv_kernel<3, 8>);
    else ok = launch(gale::w4_gemv_kernel<4, 8>);
    if (!ok) return GALE_ERR_CUDA;
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

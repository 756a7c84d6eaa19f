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
// One launch: the weights are streamed once by bulk copies into a ring of
// shared-memory stages and fed, still packed, to the int8 tensor cores: a 32-bit word of eight nibbles gives two A registers
// of (q + 8) as unsigned bytes, (w & 0x0F0F0F0F) ^ 0x08080808 and the same of
// w >> 4, one LOP3 each.  The activations are prepared in fixed point by
// every CTA while its first copies are in flight: per 1024-column
// chunk a power-of-two S with max |x S| <= 2^20,
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
constexpr int kW4MaxStages = 8;   // ring stages of a CTA (fewer when the activations need room)
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

// Launch parameters of the GEMV.  Shared memory, in this order: nst ring
// stages (the 16 code rows, then 16 scale rows of `spitch` bytes from byte
// `sreg` of the stage), the activation digits (6 NP rows of `xpitch` bytes),
// the block sums of X (int32 [2 NP][cols / 128]), 1 / S (fp32
// [2 NP][cols / 1024]), the per-warp partial sums (fp32 [2 consumer groups]
// [2 alternating buffers][NWC / 2][NP][32]), then 2 nst mbarriers and an
// abort flag.  Offsets in bytes from the start of dynamic shared memory.
struct W4Args {
    const uint8_t* q;
    const __half* s;
    const uint16_t* x;
    float* y;
    int32_t* status;
    int64_t rows, cols;
    int B, nst, uc;                 // tokens, ring stages, columns of a unit
    // whole rows (a tile is one unit): codes as 8 copies of two rows, pair p at
    // p ppitch (ppitch = cols + 64: consecutive pairs 64 bytes apart modulo
    // 128), scales as one copy; else one copy per row at ppitch / 2 and one per
    // row of scales at a padded spitch.  Row g of a stage starts at
    // (g >> 1) ppitch + (g & 1) rstride.
    int whole, ppitch, rstride, spitch, sreg, xpitch, stage_bytes;
    int off_x, off_xsum, off_xsig, off_red, off_bar;
};

// Activation digits of one (token t, 1024-column chunk ch) by one warp, into
// shared memory.  Lane l = 8 tig + 2 i + par writes, for each block bb of the
// chunk and digit j, the word of the four columns 128 bb + 32 tig + 8 i +
// 2 e + par (e = 0..3) at row (3 t + j), byte 128 block + 32 tig + 8 i + 4 par:
// the B fragment of MMA i for the lanes of quad index tig.  Tokens t >= B
// (the pad of an odd count) get zero digits and zero sums.
__device__ __forceinline__ void w4_prep_chunk(const W4Args& a, uint8_t* smem, int t, int ch, int lane) {
    const int tig = lane >> 3, i = (lane >> 1) & 3, par = lane & 1;
    const int nblk = int(a.cols / kW4Block), nch = int(a.cols / kW4Chunk);
    float v[8][4];
    float m = 0.f;
    const uint16_t* xs = a.x + int64_t(t) * a.cols + int64_t(ch) * kW4Chunk + 32 * tig + 8 * i + par;
#pragma unroll
    for (int bb = 0; bb < 8; ++bb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[bb][e] = t < a.B ? bf16_to_f32(__ldg(xs + 128 * bb + 2 * e)) : 0.f;
            m = fmaxf(m, fabsf(v[bb][e]));
        }
    m = warp_max(m);
    // largest power of two S with m S <= 2^20 (1 for a zero chunk; at most 2^100)
    // (m = f 2^e2 with 0.5 <= f < 1 gives e2 = biased exponent - 126; a
    // subnormal m takes e2 = -126, which the cap at 2^100 makes exact)
    float S = 1.0f;
    if (m > 0.f) {
        const int e2 = int((__float_as_uint(m) >> 23) & 0xFFu) - 126;
        S = __uint_as_float(uint32_t(min(20 - e2, 100) + 127) << 23);   // m S < 2^20
    }
    uint8_t* xd = smem + a.off_x;
    int32_t* xsum = reinterpret_cast<int32_t*>(smem + a.off_xsum);
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
        const int blk = ch * 8 + bb;
#pragma unroll
        for (int j = 0; j < 3; ++j)
            *reinterpret_cast<uint32_t*>(xd + (t * 3 + j) * a.xpitch + blk * 128 + tig * 32 + i * 8 + par * 4) = wd[j];
        const int tot = __reduce_add_sync(0xffffffffu, sx);
        if (lane == 0) xsum[t * nblk + blk] = tot;
    }
    if (lane == 0) reinterpret_cast<float*>(smem + a.off_xsig)[t * nch + ch] = 1.0f / S;
}

__device__ __forceinline__ void w4_fail(const W4Args& a, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(a.status, GALE_ERR_TIMEOUT);
}

// Persistent GEMV, one CTA per SM: CTA c owns the 16-row tiles c, c + grid,
// ...; a tile is read as units of 16 rows x `uc` columns (the last unit of a
// row may be narrower).  Warp NWC copies each unit into the next ring stage
// with bulk copies: when a tile is one unit, lanes 0-7 copy two whole rows
// each and lane 8 the tile's scales; else lane r < 16 copies row r's segment
// and lane 16 + r its scales.  The row placement (see W4Args) puts the eight
// rows of an A fragment in distinct bank groups.  The NWC consumer
// warps form two groups of NWG = NWC / 2 that take alternate tiles (group k:
// the CTA's tiles k, k + 2, ...), so one group's per-unit hand-off overlaps
// the other's arithmetic.  Warp w of a group multiplies columns
// [w sw, (w + 1) sw) of every unit of its tiles (sw = uc / NWG, inside one
// 1024-column chunk) and frees the stage; at the end of a tile the NWG
// partial sums of every (row, token) are added in warp order by one warp of
// the group.
// The activation digits are built by the consumer warps at the start, while
// the first copies are in flight.  NP column groups of two tokens (tokens
// 2p, 2p + 1) share the A registers of a block.  Every wait is bounded: on
// time-out the status word takes GALE_ERR_TIMEOUT, the other waits are
// skipped, and the copy warp waits (bounded) for its copies in flight.
template <int NP, int NWC, int NBW>
__global__ void __launch_bounds__((NWC + 1) * 32, 1) w4_gemv_kernel(const W4Args a) {
    extern __shared__ __align__(128) uint8_t w4_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nblk = int(a.cols / kW4Block), nch = int(a.cols / kW4Chunk);
    const int64_t ntiles = a.rows / kW4Rows;
    const int64_t my_tiles = int64_t(blockIdx.x) < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int upt = int((a.cols + a.uc - 1) / a.uc);          // units per tile
    const int nst = a.nst;
    uint64_t* full = reinterpret_cast<uint64_t*>(w4_smem + a.off_bar);
    uint64_t* empty = full + nst;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + nst);
    if (threadIdx.x == 0) {
        for (int i = 0; i < nst; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, NWC / 2);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NWC) {
        // ---- copy warp ----
        const int64_t my_units = my_tiles * upt;
        const int r = lane & 15;
        int64_t gu = 0;
        int st = 0, u = 0;
        // parity of the empty phase a stage's next reuse waits for: the first
        // reuse (units nst .. 2 nst - 1) waits for phase 0, and so on
        uint32_t eph = 1;
        int64_t tile = blockIdx.x;
#pragma unroll 1
        for (; gu < my_units; ++gu) {
            if (*abort_flag) break;
            if (gu >= nst) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait(empty + st, eph);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) w4_fail(a, abort_flag);
                    break;
                }
            }
            const int wid = int(min(int64_t(a.uc), a.cols - int64_t(u) * a.uc));
            uint8_t* stage = w4_smem + st * a.stage_bytes;
            if (lane == 0) mbar_arrive_expect_tx(full + st, uint32_t(16 * (wid / 2 + wid / 64)));
            __syncwarp();
            if (a.whole) {
                if (lane < 8)
                    bulk_load(stage + lane * a.ppitch, a.q + (tile * kW4Rows + 2 * lane) * (a.cols / 2),
                              uint32_t(a.cols), full + st);
                else if (lane == 8)
                    bulk_load(stage + a.sreg, a.s + tile * kW4Rows * nblk, uint32_t(16 * nblk * 2), full + st);
            } else {
                const int64_t row = tile * kW4Rows + r;
                if (lane < 16)
                    bulk_load(stage + (r >> 1) * a.ppitch + (r & 1) * a.rstride,
                              a.q + row * (a.cols / 2) + int64_t(u) * (a.uc / 2), uint32_t(wid / 2), full + st);
                else
                    bulk_load(stage + a.sreg + r * a.spitch, a.s + row * nblk + int64_t(u) * (a.uc / kW4Block),
                              uint32_t(wid / 64), full + st);
            }
            if (++st == nst) {
                st = 0;
                eph ^= 1;
            }
            if (++u == upt) {
                u = 0;
                tile += gridDim.x;
            }
        }
        // the copies of the last units issued land before the CTA may exit
        if (lane == 0) {
            const int64_t first = gu > nst ? gu - nst : 0;
            for (int64_t v = first; v < gu; ++v)
                if (!mbar_wait(full + (v % nst), uint32_t((v / nst) & 1))) {
                    w4_fail(a, abort_flag);
                    break;
                }
        }
        return;
    }

    // ---- consumer warps ----
    for (int it = warp; it < 2 * NP * nch; it += NWC) w4_prep_chunk(a, w4_smem, it / nch, it % nch, lane);
    named_bar_sync(3, NWC * 32);
    if (my_tiles == 0) return;

    constexpr int NWG = NWC / 2;                // warps of a consumer group
    const int grp = warp / NWG, wg = warp - grp * NWG;

    const int g = lane >> 2, tig = lane & 3;
    constexpr int sw = NBW * kW4Block;          // columns of this warp's slice of a unit (uc = NWG sw)
    const uint32_t sbase = smem_u32(w4_smem);
    const uint32_t xs = sbase + uint32_t(a.off_x);
    const int32_t* xsum = reinterpret_cast<const int32_t*>(w4_smem + a.off_xsum);
    const float* xsig = reinterpret_cast<const float*>(w4_smem + a.off_xsig);
    float* red = reinterpret_cast<float*>(w4_smem + a.off_red);
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
    const uint32_t xrow = xs + uint32_t((tk * 3 + dg) * a.xpitch + tig * 32);
    // row g, this slice, chunk tig (row g + 8 is four pairs further)
    const uint32_t aoff = uint32_t((g >> 1) * a.ppitch + (g & 1) * a.rstride + wg * (sw / 2) + 16 * tig);
    const uint32_t boff = uint32_t(4 * a.ppitch);
    const uint32_t soff = uint32_t(a.sreg + g * a.spitch + 2 * wg * NBW);
    bool live = true;   // false once a wait ran out: the remaining waits are skipped
    // stage and phase parity of the group's next unit (unit index ti upt + u of the CTA)
    int st = (grp * upt) % nst;
    uint32_t ph = uint32_t(((grp * upt) / nst) & 1);
#pragma unroll 1
    for (int64_t ti = grp; ti < my_tiles; ti += 2) {
        float tot[NP][4];
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[p][i] = 0.f;
#pragma unroll 1
        for (int u = 0; u < upt; ++u) {
            // one lane waits for the stage (the warp barrier orders the others' reads after it)
            if (live && !*abort_flag) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait(full + st, ph);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    if (lane == 0) w4_fail(a, abort_flag);
                    live = false;
                }
            } else {
                live = false;
            }
            __syncwarp();
            const int c0 = u * a.uc + wg * sw;                 // first column of the slice
            if (c0 < a.cols && c0 < u * a.uc + min(int64_t(a.uc), a.cols - int64_t(u) * a.uc)) {
                const uint32_t base = sbase + uint32_t(st * a.stage_bytes);
                float acc[NP][4];
#pragma unroll
                for (int p = 0; p < NP; ++p)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[p][i] = 0.f;
#pragma unroll
                for (int j = 0; j < NBW; ++j) {
                    const int b = c0 / kW4Block + j;
                    const uint4 ua = lds_v4(base + aoff + uint32_t(64 * j));
                    const uint4 ub = lds_v4(base + aoff + boff + uint32_t(64 * j));
                    const float s0 = __half2float(__ushort_as_half(uint16_t(lds_u16(base + soff + uint32_t(2 * j)))));
                    const float s1 = __half2float(
                        __ushort_as_half(uint16_t(lds_u16(base + soff + uint32_t(8 * a.spitch + 2 * j)))));
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
                            const uint32_t xb = xrow + uint32_t(6 * p * a.xpitch + b * 128);
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
                            const int xb8 = 8 * xsum[(2 * p + ctok) * nblk + b];
                            cc[cor] -= xb8;
                            cc[cor + 2] -= xb8;
                        }
                        acc[p][0] = fmaf(s0, float(cc[0]), acc[p][0]);
                        acc[p][1] = fmaf(s0, float(cc[1]), acc[p][1]);
                        acc[p][2] = fmaf(s1, float(cc[2]), acc[p][2]);
                        acc[p][3] = fmaf(s1, float(cc[3]), acc[p][3]);
                    }
                }
                // the slice lies in one 1024-column chunk: its sums take 1/S of each column's token
                const int ch = c0 / kW4Chunk;
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    const float f0 = tc0 < 2 ? xsig[(2 * p + tc0) * nch + ch] : 0.f;
                    const float f1 = tc1 < 2 ? xsig[(2 * p + tc1) * nch + ch] : 0.f;
                    tot[p][0] = fmaf(f0, acc[p][0], tot[p][0]);
                    tot[p][1] = fmaf(f1, acc[p][1], tot[p][1]);
                    tot[p][2] = fmaf(f0, acc[p][2], tot[p][2]);
                    tot[p][3] = fmaf(f1, acc[p][3], tot[p][3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + st);
            if (++st == nst) {
                st = 0;
                ph ^= 1;
            }
        }
        // skip the other group's tile
#pragma unroll 1
        for (int k = 0; k < upt; ++k)
            if (++st == nst) {
                st = 0;
                ph ^= 1;
            }
        // sums over the lane quad; lane (g, tig) holds row g + 8 (tig >> 1), token tig & 1 of each group
        const int li = int(ti >> 1);                          // the tile's index within the group
        float* gred = red + (grp * 2 + (li & 1)) * NWG * NP * 32;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            float v[2][2];   // [row g, g + 8][token]
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float x0 = wa * tot[p][2 * h], x1 = wc * tot[p][2 * h + 1];
                float t0v = (tc0 == 0 ? x0 : 0.f) + (tc1 == 0 ? x1 : 0.f);
                float t1v = (tc0 == 1 ? x0 : 0.f) + (tc1 == 1 ? x1 : 0.f);
                t0v += __shfl_xor_sync(0xffffffffu, t0v, 1);
                t0v += __shfl_xor_sync(0xffffffffu, t0v, 2);
                t1v += __shfl_xor_sync(0xffffffffu, t1v, 1);
                t1v += __shfl_xor_sync(0xffffffffu, t1v, 2);
                v[h][0] = t0v;
                v[h][1] = t1v;
            }
            const float mine = (tig >> 1) ? ((tig & 1) ? v[1][1] : v[1][0]) : ((tig & 1) ? v[0][1] : v[0][0]);
            gred[(wg * NP + p) * 32 + lane] = mine;
        }
        named_bar_sync(1 + grp, NWG * 32);
        // one warp adds the NWG partials in warp order (a group's buffers
        // alternate by tile, so its next tile's writes never meet this read)
        if (wg == li % NWG) {
            const int64_t r0 = (int64_t(blockIdx.x) + ti * gridDim.x) * kW4Rows;
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < NWG; ++w) sum += gred[(w * NP + p) * 32 + lane];
                const int t = 2 * p + (tig & 1);
                if (t < a.B) a.y[int64_t(t) * a.rows + r0 + g + 8 * (tig >> 1)] = sum;
            }
        }
    }
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
bool w4_gemv_shape_ok(int64_t rows, int64_t cols, int B) {
    return rows >= 16 && rows % 16 == 0 && cols >= 1024 && cols % 1024 == 0 && B >= 1 && B <= 8 &&
           rows / 16 <= 0x7FFFFFFF && cols <= (int64_t(1) << 20);
}

// Shared-memory plan for NWC consumer warps: the widest unit (4096, 2048 or
// 1024 columns, at least 128 per warp, no wider than the row needs) that
// leaves room for three ring stages, else for two.  False when none fits.
bool w4_plan(int64_t cols, int B, int nwc, gale::W4Args& a, int& smem) {
    const int np = (B + 1) / 2;
    const int nblk = int(cols / gale::kW4Block), nch = int(cols / gale::kW4Chunk);
    a.xpitch = int(cols) + 16;
    const int64_t xbytes = int64_t(6) * np * a.xpitch;
    const int64_t sums = gale::align_up(int64_t(2) * np * nblk * 4, 16) + gale::align_up(int64_t(2) * np * nch * 4, 16);
    const int64_t redb = int64_t(2) * nwc * np * 32 * 4;
    const int64_t bars = 2 * gale::kW4MaxStages * 8 + 16;
    for (int need = 3; need >= 2; --need) {
        for (int uc = 4096; uc >= 1024; uc /= 2) {
            if (uc < 64 * nwc) break;                                // a block per warp of a group
            if (uc / 2 >= 64 * nwc && uc / 2 >= cols) continue;     // a narrower unit covers the row
            const int whole = cols <= uc;
            const int ppitch = whole ? int(cols) + 64 : uc + 32;
            const int spitch = whole ? int(cols / 64) : uc / 64 + 16;
            const int sreg = 8 * ppitch;
            const int64_t stage = sreg + int64_t(16) * spitch;
            const int64_t room = gale::kW4SmemMax - xbytes - sums - redb - bars;
            if (room < need * stage) continue;
            a.uc = uc;
            a.whole = whole;
            a.ppitch = ppitch;
            a.rstride = whole ? int(cols / 2) : ppitch / 2;
            a.spitch = spitch;
            a.sreg = sreg;
            a.stage_bytes = int(stage);
            a.nst = int(room / stage < gale::kW4MaxStages ? room / stage : gale::kW4MaxStages);
            int64_t o = int64_t(a.nst) * stage;
            a.off_x = int(o);
            o += xbytes;
            a.off_xsum = int(o);
            o += gale::align_up(int64_t(2) * np * nblk * 4, 16);
            a.off_xsig = int(o);
            o += gale::align_up(int64_t(2) * np * nch * 4, 16);
            a.off_red = int(o);
            o += redb;
            a.off_bar = int(o);
            o += bars;
            smem = int(o);
            return true;
        }
    }
    return false;
}

// Consumer warps (two groups): 16 up to 4 tokens (on [65536 x 4096]: 47.1
// against 55.3 us at 1-2 tokens, 67.6 against 90.1 us at 4), 8 from 5 (172
// against 240 us at 8 tokens, where 16 warps' 96-register cap spills).
int w4_nwc(int B) { return B >= 5 ? 8 : 16; }
}  // namespace

extern "C" size_t gale_w4_workspace_size(int64_t rows, int64_t cols, int B) {
    if (!w4_gemv_shape_ok(rows, cols, B)) return 0;
    gale::W4Args a{};
    int smem = 0;
    if (!w4_plan(cols, B, w4_nwc(B), a, smem) && !w4_plan(cols, B, 8, a, smem)) return 0;   // unsupported
    return 256;   // the status word
}

extern "C" int gale_w4_gemv(const void* packed, int64_t rows, int64_t cols, const uint16_t* x, int B, float* y,
                            void* ws, size_t ws_bytes, void* stream) {
    if (!w4_gemv_shape_ok(rows, cols, B) || !packed || !x || !y) return GALE_ERR_ARG;
    if (!gale::aligned(packed, 256) || !gale::aligned(x, 2) || !gale::aligned(y, 4)) return GALE_ERR_ALIGN;
    if (!ws || ws_bytes < 256) return GALE_ERR_WORKSPACE;
    if (!gale::aligned(ws, 256)) return GALE_ERR_ALIGN;
    gale_w4_layout_t L;
    gale_w4_layout(rows, cols, &L);
    int nwc = w4_nwc(B);
    gale::W4Args a{};
    int smem = 0;
    if (!w4_plan(cols, B, nwc, a, smem)) {
        nwc = 8;   // fewer partial-sum buffers leave room for wider rows
        if (!w4_plan(cols, B, nwc, a, smem)) return GALE_ERR_UNSUPPORTED;
    }
    const uint8_t* qb = static_cast<const uint8_t*>(packed);
    a.q = qb;
    a.s = reinterpret_cast<const __half*>(qb + L.s_offset);
    a.x = x;
    a.y = y;
    a.status = static_cast<int32_t*>(ws);
    a.rows = rows;
    a.cols = cols;
    a.B = B;
    cudaStream_t st = gale::as_stream(stream);
    const int64_t tiles = rows / 16;
    const unsigned grid = unsigned(tiles < gale::sm_count() ? tiles : gale::sm_count());
    auto launch = [&](auto kern, int threads) {
        // (set on every call: the attribute belongs to the current device)
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return false;
        kern<<<grid, threads, smem, st>>>(a);
        return true;
    };
    const int np = (B + 1) / 2;
    const int nbw = a.uc / (64 * nwc);   // blocks of a warp's slice (nwc / 2 warps per group)
    bool ok = false;
    auto by_np = [&](auto k1, auto k2, auto k3, auto k4) {
        const int threads = (nwc + 1) * 32;
        return np == 1 ? launch(k1, threads) : np == 2 ? launch(k2, threads) : np == 3 ? launch(k3, threads)
                                                                                 : launch(k4, threads);
    };
    using namespace gale;
    if (nwc == 16) {
        if (nbw == 4)
            ok = by_np(w4_gemv_kernel<1, 16, 4>, w4_gemv_kernel<2, 16, 4>, w4_gemv_kernel<3, 16, 4>,
                       w4_gemv_kernel<4, 16, 4>);
        else if (nbw == 2)
            ok = by_np(w4_gemv_kernel<1, 16, 2>, w4_gemv_kernel<2, 16, 2>, w4_gemv_kernel<3, 16, 2>,
                       w4_gemv_kernel<4, 16, 2>);
        else
            ok = by_np(w4_gemv_kernel<1, 16, 1>, w4_gemv_kernel<2, 16, 1>, w4_gemv_kernel<3, 16, 1>,
                       w4_gemv_kernel<4, 16, 1>);
    } else if (nbw == 8) {
        ok = by_np(w4_gemv_kernel<1, 8, 8>, w4_gemv_kernel<2, 8, 8>, w4_gemv_kernel<3, 8, 8>, w4_gemv_kernel<4, 8, 8>);
    } else if (nbw == 4) {
        ok = by_np(w4_gemv_kernel<1, 8, 4>, w4_gemv_kernel<2, 8, 4>, w4_gemv_kernel<3, 8, 4>, w4_gemv_kernel<4, 8, 4>);
    } else {
        ok = by_np(w4_gemv_kernel<1, 8, 2>, w4_gemv_kernel<2, 8, 2>, w4_gemv_kernel<3, 8, 2>, w4_gemv_kernel<4, 8, 2>);
    }
    if (!ok) return GALE_ERR_CUDA;
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

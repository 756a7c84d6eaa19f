// Tensor-core path of gale_expert_gemv for one or two tokens: each warp
// streams 16-row tiles of the packed matrix (TMA, two stages per warp) and
// runs the int8 AND-mask MMA of mma_tile.cuh on them.
#include "common.cuh"
#include "gemv_mma.cuh"
#include "mma_tile.cuh"

namespace gale {

namespace {

constexpr int kGemvWarps = 4;
constexpr int kGemvStages = 2;

struct GemvSmem {
    int stages, pieces, xsum, xr, red, scratch, bars, bytes;
};

GemvSmem gemv_smem(int C, int warps) {
    GemvSmem s;
    const StageLayout L = stage_layout(C);
    int o = 0;
    s.stages = o;
    o += warps * kGemvStages * L.bytes;
    s.pieces = o;
    o += 2 * C * kPieces;
    s.xsum = o;
    o += 2 * (C / 128) * 4;
    s.xr = o;
    o += C * 4;
    s.red = o;
    o += 64 * 4;
    s.scratch = o;
    o += warps * kWarpScratchFloats * 4;
    s.bars = o;
    o += warps * kGemvStages * 8;
    s.bytes = int(align_up(o, 1024)) + 1024;   // + slack to align the base to 1024
    return s;
}

template <bool SWIGLU>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_mma_kernel(
    const __grid_constant__ CUtensorMap smap_a, const __grid_constant__ CUtensorMap bmap_a,
    const __grid_constant__ CUtensorMap smap_b, const __grid_constant__ CUtensorMap bmap_b, MatView a, MatView b,
    const float* __restrict__ x, int ntok, float* __restrict__ y, GemvSmem S) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = a.cols;
    const StageLayout L = stage_layout(C);
    constexpr int nmat = SWIGLU ? 2 : 1;
    const int tiles = (a.rows + 15) / 16;
    // warp-major numbering spreads the first tiles over all CTAs
    const int gw = warp * gridDim.x + blockIdx.x, nw = gridDim.x * kGemvWarps;
    const int my_tiles = tiles > gw ? (tiles - gw + nw - 1) / nw : 0;
    const int njobs = my_tiles * nmat;
    uint8_t* stages = smem + S.stages + warp * kGemvStages * L.bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.bars) + warp * kGemvStages;
    float* scratch = reinterpret_cast<float*>(smem + S.scratch) + warp * kWarpScratchFloats;

    auto issue = [&](int i) {
        const int tile = gw + (i / nmat) * nw;
        const bool second = SWIGLU && (i % nmat);
        uint8_t* st = stages + (i % kGemvStages) * L.bytes;
        issue_tile(st, bars + (i % kGemvStages), second ? &smap_b : &smap_a, second ? &bmap_b : &bmap_a,
                   second ? b : a, 0, tile * 16);
    };
    if (lane == 0) {
        for (int s = 0; s < kGemvStages; ++s) mbar_init(bars + s, 1);
        fence_mbar_init();
        for (int i = 0; i < min(kGemvStages, njobs); ++i) issue(i);
    }
    __syncwarp();

    // activation pieces of the (one or two) tokens, built by the whole CTA
    uint8_t* pieces = smem + S.pieces;
    float* xsum = reinterpret_cast<float*>(smem + S.xsum);
    float* xr = reinterpret_cast<float*>(smem + S.xr);
    float* red = reinterpret_cast<float*>(smem + S.red);
    TokRef tok[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {   // unrolled: tok stays in registers
        tok[t] = TokRef{nullptr, nullptr, nullptr, 1.f};
        if (t >= ntok) continue;
        for (int c = threadIdx.x; c < C; c += blockDim.x) xr[c] = x[int64_t(t) * C + c];
        __syncthreads();
        const float sigma = build_pieces(xr, C, pieces + t * C * kPieces, xsum + t * (C / 128), red);
        tok[t] = TokRef{pieces + t * C * kPieces, xsum + t * (C / 128), x + int64_t(t) * C, sigma};
    }

    float y1[2] = {0.f, 0.f};
    for (int i = 0; i < njobs; ++i) {
        const int tile = gw + (i / nmat) * nw;
        const bool second = SWIGLU && (i % nmat);
        uint8_t* st = stages + (i % kGemvStages) * L.bytes;
        if (!mbar_wait(bars + (i % kGemvStages), (i / kGemvStages) & 1)) return;   // bounded: gives up
        float yv[2];
        tile_compute(st, second ? b : a, tile * 16, tok, scratch, yv);
        __syncwarp();
        if (lane == 0 && i + kGemvStages < njobs) {
            fence_proxy_async();
            issue(i + kGemvStages);
        }
        const int r = tile * 16 + lane;
        if (SWIGLU && !second) {
            y1[0] = yv[0];
            y1[1] = yv[1];
            continue;
        }
        if (lane < 16 && r < a.rows) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {   // static indices keep y1 / yv in registers
                if (t >= ntok) break;
                const float v = SWIGLU ? silu(y1[t]) * yv[t] : yv[t];
                y[int64_t(t) * a.rows + r] = v;
            }
        }
    }
}

}  // namespace

bool gemv_mma_supported(int cols, int ntok) {
    return ntok >= 1 && ntok <= kMmaMaxTok && cols <= 4096 && cols % 1024 == 0;
}

int launch_gemv_mma(const MatView& a, const MatView& b, bool swiglu, const float* x, int ntok, float* y,
                    cudaStream_t st) {
    CUtensorMap sa, ba, sb, bb;
    const Layout La = make_layout(a.rows, a.cols);
    const int64_t stride = align_up(La.total, 256);
    int rc = cached_map(&sa, false, a.signs, a.rows, a.cols, 1, stride);
    if (rc == GALE_OK) rc = cached_map(&ba, true, a.signs, a.rows, a.cols, 1, stride);
    if (rc == GALE_OK) rc = cached_map(&sb, false, b.signs, b.rows, b.cols, 1, stride);
    if (rc == GALE_OK) rc = cached_map(&bb, true, b.signs, b.rows, b.cols, 1, stride);
    if (rc != GALE_OK) return rc;
    const GemvSmem S = gemv_smem(a.cols, kGemvWarps);
    const int tiles = (a.rows + 15) / 16;
    const int grid = tiles < sm_count() ? tiles : sm_count();
    if (swiglu) {
        rc = ensure_smem(reinterpret_cast<const void*>(gemv_mma_kernel<true>), S.bytes);
        if (rc != GALE_OK) return rc;
        gemv_mma_kernel<true><<<grid, kGemvWarps * 32, S.bytes, st>>>(sa, ba, sb, bb, a, b, x, ntok, y, S);
    } else {
        rc = ensure_smem(reinterpret_cast<const void*>(gemv_mma_kernel<false>), S.bytes);
        if (rc != GALE_OK) return rc;
        gemv_mma_kernel<false><<<grid, kGemvWarps * 32, S.bytes, st>>>(sa, ba, sa, ba, a, a, x, ntok, y, S);
    }
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

}  // namespace gale

// Blocked FWHT-1024 with warp-shuffle butterflies (one warp per 1024-block).
//
// Lane l holds elements n = 32*i + l (i = 0..31) of its block.  The five
// butterfly stages whose stride is below 32 pair lanes (shuffle xor), the
// five with stride >= 32 pair registers of one lane; all ten commute.  The
// result is scaled by 1/32, which makes the transform orthonormal and its
// own inverse (Sylvester order: DeepSeek-V4-Pro-671B-GALE-1bit-v4 card,
// knobs paragraph, single-kernel butterfly Walsh-Hadamard transform).
#include "common.cuh"
#include "fwht.cuh"

namespace {

using namespace gale;

__global__ void __launch_bounds__(256) fwht1024_kernel(const void* __restrict__ x, int x_dtype,
                                                       void* __restrict__ y, int y_dtype,
                                                       int64_t n_blocks) {
    const int lane = threadIdx.x & 31;
    int64_t blk = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
    if (blk >= n_blocks) return;
    const int64_t base = blk * 1024;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = load_as_f32(x, x_dtype, base + 32 * i + lane);
    fwht1024_warp(v, lane);
#pragma unroll
    for (int i = 0; i < 32; ++i) store_from_f32(y, y_dtype, base + 32 * i + lane, v[i] * (1.0f / 32.0f));
}

}  // namespace

extern "C" int gale_fwht1024(const void* x, int x_dtype, void* y, int y_dtype, int64_t rows, int cols,
                             void* stream) {
    if (rows < 0 || cols < kRot || cols % kRot) return GALE_ERR_ARG;
    if (x_dtype < GALE_F32 || x_dtype > GALE_F16 || y_dtype < GALE_F32 || y_dtype > GALE_F16)
        return GALE_ERR_ARG;
    if (rows == 0) return GALE_OK;
    if (!x || !y) return GALE_ERR_ARG;
    if (!aligned(x, 4) || !aligned(y, 4)) return GALE_ERR_ALIGN;
    if (x == y && x_dtype != y_dtype) return GALE_ERR_ARG;
    int64_t n_blocks = rows * (cols / kRot);
    int64_t grid = (n_blocks * 32 + 255) / 256;
    if (grid > 0x7FFFFFFF) return GALE_ERR_UNSUPPORTED;
    fwht1024_kernel<<<unsigned(grid), 256, 0, as_stream(stream)>>>(x, x_dtype, y, y_dtype, n_blocks);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

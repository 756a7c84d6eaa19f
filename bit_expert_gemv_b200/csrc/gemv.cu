// gale_expert_gemv: one packed matrix (or a SwiGLU w1/w3 pair) times rotated
// activations, straight from the packed record (DeepSeek-V4-Pro-671B-GALE-1bit-v4
// card, knobs paragraph: direct GEMV, signs, block scales and int4 outliers
// decoded in registers).
#include "common.cuh"
#include "gemv_simple.cuh"
#include "gemv_mma.cuh"

namespace gale {

constexpr int kRowsPerWarp = 8;
constexpr int kWarps = 8;

int simple_chunk_tokens(int cols) {
    int nt = int((200 * 1024) / (int64_t(cols) * 4));
    return nt < 1 ? 1 : (nt > kSimpleNT ? kSimpleNT : nt);
}

template <bool SWIGLU>
__global__ void __launch_bounds__(256) gemv_simple_kernel(MatView a, MatView b, const float* __restrict__ x,
                                                          int ntok, int chunk, float* __restrict__ y) {
    extern __shared__ float xs[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cols = a.cols;
    for (int t0 = 0; t0 < ntok; t0 += chunk) {
        const int nt = min(chunk, ntok - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < nt * cols; i += blockDim.x) xs[i] = x[int64_t(t0) * cols + i];
        __syncthreads();
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int r = blockIdx.x * (kWarps * kRowsPerWarp) + i * kWarps + warp;
            if (r >= a.rows) break;
            float acc[kSimpleNT];
            row_dot_simple(a, r, xs, nt, acc, lane);
            if (SWIGLU) {
                float acc3[kSimpleNT];
                row_dot_simple(b, r, xs, nt, acc3, lane);
#pragma unroll
                for (int t = 0; t < kSimpleNT; ++t) acc[t] = silu(acc[t]) * acc3[t];
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kSimpleNT; ++t)
                    if (t < nt) y[int64_t(t0 + t) * a.rows + r] = acc[t];
            }
        }
    }
}

}  // namespace gale

extern "C" int gale_expert_gemv(const gale_matrix* W, const gale_matrix* W3, const float* x_rot,
                                int ntok, float* y, int mode, void* stream) {
    using namespace gale;
    if (!W || !W->packed || !x_rot || !y || ntok < 1 || ntok > 64) return GALE_ERR_ARG;
    if (W->rows < 1 || !valid_cols(W->cols) || W->cols > 16384) return GALE_ERR_ARG;
    if (mode == GALE_MODE_PLAIN) {
        if (W3) return GALE_ERR_ARG;
    } else if (mode == GALE_MODE_SWIGLU) {
        if (!W3 || !W3->packed || W3->rows != W->rows || W3->cols != W->cols) return GALE_ERR_ARG;
    } else {
        return GALE_ERR_ARG;
    }
    if (!aligned(W->packed, 16) || (W3 && !aligned(W3->packed, 16)) || !aligned(x_rot, 16) || !aligned(y, 4))
        return GALE_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    MatView a = make_view(W->packed, W->rows, W->cols);
    MatView b = W3 ? make_view(W3->packed, W3->rows, W3->cols) : a;
    // decode-sized token counts take the tensor-core path
    if (gemv_mma_supported(W->cols, ntok)) return launch_gemv_mma(a, b, mode == GALE_MODE_SWIGLU, x_rot, ntok, y, st);
    const int chunk = simple_chunk_tokens(W->cols);
    const size_t smem = size_t(chunk) * W->cols * sizeof(float);
    const int grid = (W->rows + kWarps * kRowsPerWarp - 1) / (kWarps * kRowsPerWarp);
    if (mode == GALE_MODE_SWIGLU) {
        GALE_CUDA_TRY(cudaFuncSetAttribute(gemv_simple_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem)));
        gemv_simple_kernel<true><<<grid, 256, smem, st>>>(a, b, x_rot, ntok, chunk, y);
    } else {
        GALE_CUDA_TRY(cudaFuncSetAttribute(gemv_simple_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem)));
        gemv_simple_kernel<false><<<grid, 256, smem, st>>>(a, b, x_rot, ntok, chunk, y);
    }
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

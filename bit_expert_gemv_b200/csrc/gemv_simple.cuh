// Reference-structure GEMV on CUDA cores: one warp per output row, lane l
// takes column 32*w + l of every sign word w (conflict-free shared-memory
// reads of the activations), multiplies by the signed block scale and
// accumulates in fp32; the row's outliers are then patched by
// (q * s_row - sign * s_blk) * x[c]; a warp reduction finishes the row.
// Used for groups of tokens of any size and as the correctness baseline of
// the tensor-core decode path.
#pragma once
#include "common.cuh"

namespace gale {

constexpr int kSimpleNT = 8;   // tokens per pass

// xs: shared fp32 [nt][cols]; acc[t] receives the full row dot (all lanes).
__device__ __forceinline__ void row_dot_simple(const MatView& m, int r, const float* xs, int nt,
                                               float (&acc)[kSimpleNT], int lane) {
#pragma unroll
    for (int t = 0; t < kSimpleNT; ++t) acc[t] = 0.f;
    const int cols = m.cols;
    const uint32_t* sw = m.signs + int64_t(r) * (cols / 32);
    const __half* sb = m.s_blk + int64_t(r) * (cols / kBlock);
    for (int w4 = 0; w4 < cols / 128; ++w4) {
        const uint4 words = reinterpret_cast<const uint4*>(sw)[w4];
        const float s = __half2float(sb[w4]);
        const uint32_t wv[4] = {words.x, words.y, words.z, words.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float sv = ((wv[j] >> lane) & 1u) ? -s : s;
            const int c = 128 * w4 + 32 * j + lane;
#pragma unroll
            for (int t = 0; t < kSimpleNT; ++t)
                if (t < nt) acc[t] = fmaf(sv, xs[t * cols + c], acc[t]);
        }
    }
    const int k = m.k;
    if (k > 0) {
        const float srow = __half2float(m.s_row[r]);
        for (int j = lane; j < k; j += 32) {
            const int64_t n = int64_t(r) * k + j;
            const int c = m.idx[n];
            if (c >= cols) continue;   // only records that failed validation
            const float sblk = __half2float(sb[c / kBlock]);
            const float w_sign = ((sw[c >> 5] >> (c & 31)) & 1u) ? -sblk : sblk;
            const float corr = float(load_q(m.q, n)) * srow - w_sign;
#pragma unroll
            for (int t = 0; t < kSimpleNT; ++t)
                if (t < nt) acc[t] = fmaf(corr, xs[t * cols + c], acc[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < kSimpleNT; ++t) acc[t] = warp_sum(acc[t]);
}

}  // namespace gale

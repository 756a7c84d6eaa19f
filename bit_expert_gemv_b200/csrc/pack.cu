// gale_pack / gale_unpack: canonical unpacked arrays <-> packed record.
// Layout of the record: see gale.h (five 256-byte aligned sections).
#include "common.cuh"

namespace {

using namespace gale;

// One thread per 32-bit sign word: bit i of word w of row r is column 32w + i.
__global__ void pack_signs_kernel(const uint8_t* __restrict__ signs, int64_t n_words,
                                  uint32_t* __restrict__ out) {
    for (int64_t w = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; w < n_words;
         w += int64_t(gridDim.x) * blockDim.x) {
        const uint8_t* s = signs + w * 32;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) word |= uint32_t(s[i] != 0) << i;
        out[w] = word;
    }
}

__global__ void copy_u16_kernel(const uint16_t* __restrict__ src, int64_t n, uint16_t* __restrict__ dst) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
         i += int64_t(gridDim.x) * blockDim.x)
        dst[i] = src[i];
}

// One thread per row: validates and copies the row's outlier columns, and ORs
// its int4 values into the (zeroed) nibble section through 32-bit atomics,
// since neighbouring rows may share a byte when k is odd.
__global__ void pack_outliers_kernel(const uint16_t* __restrict__ idx, const int8_t* __restrict__ q,
                                     int rows, int cols, int k, uint16_t* __restrict__ idx_out,
                                     uint32_t* __restrict__ q_words, int32_t* status) {
    int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    int prev = -1;
    for (int j = 0; j < k; ++j) {
        int64_t n = int64_t(r) * k + j;
        int c = idx[n];
        int v = q[n];
        if (c <= prev || c >= cols || v < -8 || v > 7) set_status(status, GALE_ERR_ARG);
        prev = c;
        idx_out[n] = uint16_t(c);
        uint32_t nib = uint32_t(v) & 0xFu;
        int64_t byte = n >> 1;
        int shift = int((byte & 3) * 8 + (n & 1) * 4);
        atomicOr(q_words + (byte >> 2), nib << shift);
    }
}

__global__ void unpack_dense_kernel(MatView m, float* __restrict__ dense) {
    int64_t total = int64_t(m.rows) * m.cols;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        int64_t r = i / m.cols;
        int c = int(i - r * m.cols);
        uint32_t w = m.signs[i >> 5];
        float s = __half2float(m.s_blk[r * (m.cols / kBlock) + c / kBlock]);
        dense[i] = ((w >> (c & 31)) & 1u) ? -s : s;
    }
}

__global__ void unpack_outliers_kernel(MatView m, float* __restrict__ dense) {
    int64_t total = int64_t(m.rows) * m.k;
    for (int64_t n = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; n < total;
         n += int64_t(gridDim.x) * blockDim.x) {
        int64_t r = n / m.k;
        int c = m.idx[n];
        if (c < m.cols) dense[r * m.cols + c] = float(load_q(m.q, n)) * __half2float(m.s_row[r]);
    }
}

inline int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    int cap = gale::sm_count() * 8;
    return int(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

extern "C" int gale_pack(const uint8_t* signs, const uint16_t* s_blk, const uint16_t* s_row,
                         const uint16_t* idx, const int8_t* q, int rows, int cols, void* dst,
                         int32_t* status, void* stream) {
    if (rows < 1 || !valid_cols(cols) || !signs || !s_blk || !s_row || !dst || !status)
        return GALE_ERR_ARG;
    Layout L = make_layout(rows, cols);
    if (L.k > 0 && (!idx || !q)) return GALE_ERR_ARG;
    if (!aligned(dst, 16) || !aligned(s_blk, 2) || !aligned(s_row, 2) || (L.k && !aligned(idx, 2)) ||
        !aligned(status, 4))
        return GALE_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    char* d = static_cast<char*>(dst);
    GALE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    GALE_CUDA_TRY(cudaMemsetAsync(dst, 0, size_t(L.total), st));
    int64_t n_words = int64_t(rows) * cols / 32;
    pack_signs_kernel<<<grid_for(n_words, 256), 256, 0, st>>>(signs, n_words,
                                                              reinterpret_cast<uint32_t*>(d + L.off_signs));
    GALE_LAUNCH_CHECK();
    int64_t n_blk = int64_t(rows) * (cols / kBlock);
    copy_u16_kernel<<<grid_for(n_blk, 256), 256, 0, st>>>(s_blk, n_blk,
                                                          reinterpret_cast<uint16_t*>(d + L.off_sblk));
    GALE_LAUNCH_CHECK();
    copy_u16_kernel<<<grid_for(rows, 256), 256, 0, st>>>(s_row, rows,
                                                         reinterpret_cast<uint16_t*>(d + L.off_srow));
    GALE_LAUNCH_CHECK();
    if (L.k > 0) {
        pack_outliers_kernel<<<(rows + 127) / 128, 128, 0, st>>>(
            idx, q, rows, cols, L.k, reinterpret_cast<uint16_t*>(d + L.off_idx),
            reinterpret_cast<uint32_t*>(d + L.off_q), status);
        GALE_LAUNCH_CHECK();
    }
    return GALE_OK;
}

extern "C" int gale_unpack(const void* packed, int rows, int cols, float* dense, void* stream) {
    if (!packed || !dense || rows < 1 || !valid_cols(cols)) return GALE_ERR_ARG;
    if (!aligned(packed, 16) || !aligned(dense, 4)) return GALE_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    MatView m = make_view(packed, rows, cols);
    int64_t n = int64_t(rows) * cols;
    unpack_dense_kernel<<<grid_for(n, 256), 256, 0, st>>>(m, dense);
    GALE_LAUNCH_CHECK();
    if (m.k > 0) {
        unpack_outliers_kernel<<<grid_for(int64_t(rows) * m.k, 256), 256, 0, st>>>(m, dense);
        GALE_LAUNCH_CHECK();
    }
    return GALE_OK;
}

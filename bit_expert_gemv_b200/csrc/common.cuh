// Shared device/host helpers of libgale (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gale.h"

#define GALE_CUDA_TRY(expr)                                  \
    do {                                                     \
        cudaError_t e_ = (expr);                             \
        if (e_ != cudaSuccess) return GALE_ERR_CUDA;         \
    } while (0)

#define GALE_LAUNCH_CHECK()                                  \
    do {                                                     \
        if (cudaGetLastError() != cudaSuccess) return GALE_ERR_CUDA; \
    } while (0)

namespace gale {

constexpr int kBlock = 128;       // weights per block scale
constexpr int kRot = 1024;        // rotation block
constexpr int kAlign = 256;       // section alignment

// Layout of one packed matrix, computed identically on host and device.
struct Layout {
    int rows, cols, k;
    int64_t off_signs, off_sblk, off_srow, off_idx, off_q, total;
};

__host__ __device__ inline int64_t align_up(int64_t n, int64_t a) { return (n + a - 1) / a * a; }

// Outliers per row: the nearest integer to cols / 100.
__host__ __device__ inline int outliers_per_row(int cols) { return (cols + 50) / 100; }

__host__ __device__ inline Layout make_layout(int rows, int cols) {
    Layout L;
    L.rows = rows;
    L.cols = cols;
    L.k = outliers_per_row(cols);
    int64_t r = rows;
    L.off_signs = 0;
    L.off_sblk = align_up(r * cols / 8, kAlign);
    L.off_srow = align_up(L.off_sblk + r * (cols / kBlock) * 2, kAlign);
    L.off_idx = align_up(L.off_srow + r * 2, kAlign);
    L.off_q = align_up(L.off_idx + r * L.k * 2, kAlign);
    L.total = align_up(L.off_q + (r * L.k + 1) / 2, kAlign);
    return L;
}

// Typed views of one packed matrix.
struct MatView {
    const uint32_t* signs;   // [rows][cols/32]
    const __half* s_blk;     // [rows][cols/128]
    const __half* s_row;     // [rows]
    const uint16_t* idx;     // [rows][k]
    const uint8_t* q;        // nibbles
    int rows, cols, k;
};

__host__ __device__ inline MatView make_view(const void* base, int rows, int cols) {
    Layout L = make_layout(rows, cols);
    const char* b = static_cast<const char*>(base);
    MatView v;
    v.signs = reinterpret_cast<const uint32_t*>(b + L.off_signs);
    v.s_blk = reinterpret_cast<const __half*>(b + L.off_sblk);
    v.s_row = reinterpret_cast<const __half*>(b + L.off_srow);
    v.idx = reinterpret_cast<const uint16_t*>(b + L.off_idx);
    v.q = reinterpret_cast<const uint8_t*>(b + L.off_q);
    v.rows = rows;
    v.cols = cols;
    v.k = L.k;
    return v;
}

// int4 outlier value j of row r (nibble r*k + j, low nibble first).
__device__ __forceinline__ int load_q(const uint8_t* q, int64_t n) {
    int byte = q[n >> 1];
    int nib = (n & 1) ? (byte >> 4) : (byte & 0xF);
    return nib >= 8 ? nib - 16 : nib;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// fp32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return uint16_t(u >> 16);
}

__device__ __forceinline__ float load_as_f32(const void* p, int dtype, int64_t i) {
    if (dtype == GALE_F32) return static_cast<const float*>(p)[i];
    if (dtype == GALE_BF16) return bf16_to_f32(static_cast<const uint16_t*>(p)[i]);
    return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ void store_from_f32(void* p, int dtype, int64_t i, float v) {
    if (dtype == GALE_F32) static_cast<float*>(p)[i] = v;
    else if (dtype == GALE_BF16) static_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
    else static_cast<__half*>(p)[i] = __float2half_rn(v);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Set the device status word to `code` if it is still zero.
__device__ __forceinline__ void set_status(int32_t* status, int code) {
    if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_cols(int cols) { return cols >= kRot && cols % kRot == 0 && cols <= 65536; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Per-device attribute cache (SM count), filled on first use.
int sm_count();

}  // namespace gale

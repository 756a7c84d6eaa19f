// Tensor maps over packed records (host side).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gale {

constexpr int kTileRows = 16;   // rows of one MMA tile (and of one TMA box)

int make_map_3d(CUtensorMap* m, bool u16, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, bool swizzle128);
int make_sign_map(CUtensorMap* m, const void* first_matrix, int rows, int cols, int experts, int64_t stride);
int make_scale_map(CUtensorMap* m, const void* first_matrix, int rows, int cols, int experts, int64_t stride);
int cached_map(CUtensorMap* out, bool scale, const void* first_matrix, int rows, int cols, int experts,
               int64_t stride);
int make_sign_map5(CUtensorMap* m, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                   int experts, int64_t stride, int box_rows);
int cached_sign_map5(CUtensorMap* out, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                     int experts, int64_t stride, int box_rows);
int make_sign_map5b(CUtensorMap* m, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                    int experts, int64_t stride, int box_rows, int box_mats);
int cached_sign_map5b(CUtensorMap* out, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                      int experts, int64_t stride, int box_rows, int box_mats);
// Raise a kernel's dynamic shared-memory limit once per device.
int ensure_smem(const void* kernel, int bytes);

}  // namespace gale

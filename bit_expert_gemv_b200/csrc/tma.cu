// Host-side tensor-map encoding (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library does not link libcuda directly).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tma.cuh"

namespace gale {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}
}  // namespace

int make_map_3d(CUtensorMap* m, bool u16, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, bool swizzle128) {
    auto fn = encode_fn();
    if (!fn) return GALE_ERR_CUDA;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, u16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 3,
                    const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GALE_OK : GALE_ERR_CUDA;
}

// Sign words of one matrix kind across experts: [experts][rows][cols/32] uint32,
// boxes of 32 words (1024 columns) x 16 rows, 128-byte swizzle.
int make_sign_map(CUtensorMap* m, const void* first_matrix, int rows, int cols, int experts, int64_t stride) {
    return make_map_3d(m, false, first_matrix, uint64_t(cols) / 32, uint64_t(rows), uint64_t(experts),
                       uint64_t(cols) / 8, uint64_t(stride), 32, kTileRows, true);
}

// Block scales of one matrix kind across experts: [experts][rows][cols/128] fp16,
// boxes of a full row of scales x 16 rows.
int make_scale_map(CUtensorMap* m, const void* first_matrix, int rows, int cols, int experts, int64_t stride) {
    const Layout L = make_layout(rows, cols);
    const char* p = static_cast<const char*>(first_matrix) + L.off_sblk;
    return make_map_3d(m, true, p, uint64_t(cols) / 128, uint64_t(rows), uint64_t(experts), uint64_t(cols) / 64,
                       uint64_t(stride), uint32_t(cols / 128), kTileRows, false);
}

// Sign words of up to two same-shaped matrices of every expert, as a 5-D view
// (word in a 128-byte piece, row, piece, matrix, expert) with strides (row
// pitch cols/8, 128, mat_stride, stride).  A box of (32 words, box_rows rows,
// every piece) lands as [piece][row][128 bytes] with 128-byte swizzle: the
// 16-byte chunk c of row r sits at chunk position c ^ (r & 7).
int make_sign_map5(CUtensorMap* m, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                   int experts, int64_t stride, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return GALE_ERR_CUDA;
    cuuint64_t dims[5] = {32, cuuint64_t(rows), cuuint64_t(cols / 1024), cuuint64_t(n_mat), cuuint64_t(experts)};
    cuuint64_t strides[4] = {cuuint64_t(cols / 8), 128, cuuint64_t(mat_stride), cuuint64_t(stride)};
    cuuint32_t box[5] = {32, cuuint32_t(box_rows), cuuint32_t(cols / 1024), 1, 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, const_cast<void*>(first_matrix), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GALE_OK : GALE_ERR_CUDA;
}

// The same 5-D view with a box over `box_mats` matrices at once (every
// matrix of the view when box_mats == n_mat): a box of (32 words, box_rows
// rows, every piece, box_mats matrices) lands as [matrix][piece][row][128 B].
int make_sign_map5b(CUtensorMap* m, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                    int experts, int64_t stride, int box_rows, int box_mats) {
    auto fn = encode_fn();
    if (!fn) return GALE_ERR_CUDA;
    cuuint64_t dims[5] = {32, cuuint64_t(rows), cuuint64_t(cols / 1024), cuuint64_t(n_mat), cuuint64_t(experts)};
    cuuint64_t strides[4] = {cuuint64_t(cols / 8), 128, cuuint64_t(mat_stride), cuuint64_t(stride)};
    cuuint32_t box[5] = {32, cuuint32_t(box_rows), cuuint32_t(cols / 1024), cuuint32_t(box_mats), 1};
    cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, const_cast<void*>(first_matrix), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GALE_OK : GALE_ERR_CUDA;
}

namespace {
struct Map5Entry {
    const void* base;
    int rows, cols, n_mat, experts, box_rows, box_mats;
    int64_t mat_stride, stride;
    CUtensorMap map;
};
constexpr int kMap5Cache = 32;
thread_local Map5Entry g_maps5[kMap5Cache];
thread_local int g_map5_next = 0;
}  // namespace

int cached_sign_map5(CUtensorMap* out, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                     int experts, int64_t stride, int box_rows) {
    return cached_sign_map5b(out, first_matrix, rows, cols, n_mat, mat_stride, experts, stride, box_rows, 1);
}

int cached_sign_map5b(CUtensorMap* out, const void* first_matrix, int rows, int cols, int n_mat, int64_t mat_stride,
                      int experts, int64_t stride, int box_rows, int box_mats) {
    for (int i = 0; i < kMap5Cache; ++i) {
        const Map5Entry& e = g_maps5[i];
        if (e.base == first_matrix && e.rows == rows && e.cols == cols && e.n_mat == n_mat &&
            e.experts == experts && e.box_rows == box_rows && e.box_mats == box_mats && e.mat_stride == mat_stride &&
            e.stride == stride) {
            *out = e.map;
            return GALE_OK;
        }
    }
    Map5Entry e{first_matrix, rows, cols, n_mat, experts, box_rows, box_mats, mat_stride, stride, {}};
    const int rc = make_sign_map5b(&e.map, first_matrix, rows, cols, n_mat, mat_stride, experts, stride, box_rows,
                                   box_mats);
    if (rc != GALE_OK) return rc;
    g_maps5[g_map5_next] = e;
    g_map5_next = (g_map5_next + 1) % kMap5Cache;
    *out = e.map;
    return GALE_OK;
}

namespace {
struct MapEntry {
    const void* base;
    int rows, cols, experts;
    int64_t stride;
    bool scale;
    CUtensorMap map;
};
constexpr int kMapCache = 128;
thread_local MapEntry g_maps[kMapCache];
thread_local int g_map_next = 0;
}  // namespace

// Tensor maps depend only on (base, shape, stride), so they are encoded once
// and kept in a small per-thread cache (encoding costs microseconds of host
// time per map).
int cached_map(CUtensorMap* out, bool scale, const void* first_matrix, int rows, int cols, int experts,
               int64_t stride) {
    for (int i = 0; i < kMapCache; ++i) {
        const MapEntry& e = g_maps[i];
        if (e.base == first_matrix && e.rows == rows && e.cols == cols && e.experts == experts &&
            e.stride == stride && e.scale == scale) {
            *out = e.map;
            return GALE_OK;
        }
    }
    MapEntry e{first_matrix, rows, cols, experts, stride, scale, {}};
    const int rc = scale ? make_scale_map(&e.map, first_matrix, rows, cols, experts, stride)
                         : make_sign_map(&e.map, first_matrix, rows, cols, experts, stride);
    if (rc != GALE_OK) return rc;
    g_maps[g_map_next] = e;
    g_map_next = (g_map_next + 1) % kMapCache;
    *out = e.map;
    return GALE_OK;
}

int ensure_smem(const void* kernel, int bytes) {
    constexpr int kMaxDev = 64, kMaxKernels = 32;
    static const void* kernels[kMaxDev][kMaxKernels] = {};
    static int set_bytes[kMaxDev][kMaxKernels] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return GALE_ERR_CUDA;
    int slot = -1;
    for (int i = 0; i < kMaxKernels; ++i) {
        if (kernels[dev][i] == kernel) { slot = i; break; }
        if (!kernels[dev][i]) { slot = i; kernels[dev][i] = kernel; break; }
    }
    if (slot >= 0 && set_bytes[dev][slot] >= bytes) return GALE_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return GALE_ERR_CUDA;
    if (slot >= 0) set_bytes[dev][slot] = bytes;
    return GALE_OK;
}

}  // namespace gale

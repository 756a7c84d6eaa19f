// gale_encode: a dense fp32 matrix -> one packed GALE 1-bit record, on the
// device, with the same decisions as the encoder readings in gale.h (the
// DeepSeek-V4-Pro-671B-GALE-1bit-v4 card's weights table and the paragraph
// under it: "the v3 pack rounded each weight to its sign"; the format of the
// DeepSeek-V4-Flash card's "What is in the pack").
//
// One CTA per row.  Every warp rotates 1024-blocks of the row in fp64 (the
// butterfly stages in the order h = 1, 2, ..., 512, then 1/32) into shared
// memory; then the row's sign words, its k outliers (k rounds of a block-wide
// arg-max of |w| with the lower column first on ties), their symmetric int4
// codes with the row scale fp16(max |w| / 7), and the block scales
// fp16(mean |w| over the kept weights, summed in column order) are written.
// Each decision is taken on the same fp64 values in the same order as the
// host-side definition, so the record is bit-exact with it.
#include <cuda_fp16.h>

#include "common.cuh"

namespace gale {

namespace {

constexpr int kEncThreads = 256;
constexpr int kEncMaxCols = 16384;   // the row's fp64 values live in shared memory

// Register layout of a warp-held 1024-block: lane l, register r holds element
// (l & 7) + 8 (r & 3) + 32 (l >> 3) + 128 (r >> 2).
__device__ __forceinline__ int enc_elem(int lane, int r) {
    return (lane & 7) + 8 * (r & 3) + 32 * (lane >> 3) + 128 * (r >> 2);
}

// Butterfly on element bit held by lane bit `lb`: lower element a + b, upper a - b.
__device__ __forceinline__ void lane_stage(double (&v)[32], int lane, int lb) {
    const bool upper = (lane >> lb) & 1;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        const double o = __shfl_xor_sync(0xffffffffu, v[r], 1 << lb);
        v[r] = upper ? o - v[r] : v[r] + o;
    }
}

// Butterfly on element bit held by register bit `rb`.
template <int RB>
__device__ __forceinline__ void reg_stage(double (&v)[32]) {
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        if (r & (1 << RB)) continue;
        const double a = v[r], b = v[r | (1 << RB)];
        v[r] = a + b;
        v[r | (1 << RB)] = a - b;
    }
}

struct EncKey {
    unsigned long long mag;   // |w| as fp64 bits (monotone for non-negative values)
    int col;
};
__device__ __forceinline__ bool enc_better(const EncKey& a, const EncKey& b) {
    return a.mag > b.mag || (a.mag == b.mag && a.col < b.col);
}

__global__ void __launch_bounds__(kEncThreads) encode_kernel(const float* __restrict__ w, int rows, int cols, int k,
                                                             char* __restrict__ dst, Layout L) {
    extern __shared__ __align__(16) uint8_t enc_smem[];
    double* wr = reinterpret_cast<double*>(enc_smem);                       // [cols]
    uint32_t* outmap = reinterpret_cast<uint32_t*>(wr + cols);              // [cols / 32] selected columns
    int* sel = reinterpret_cast<int*>(outmap + cols / 32);                  // [k] in pick order
    EncKey* wbest = reinterpret_cast<EncKey*>(sel + ((k + 1) & ~1));        // [8] per-warp winners
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x;
    const float* wrow = w + int64_t(row) * cols;

    // 1. rotate every 1024-block in fp64
    for (int b = warp; b < cols / 1024; b += kEncThreads / 32) {
        double v[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = double(__ldg(wrow + 1024 * b + enc_elem(lane, r)));
        lane_stage(v, lane, 0);   // element bit 0
        lane_stage(v, lane, 1);   // 1
        lane_stage(v, lane, 2);   // 2
        reg_stage<0>(v);          // 3
        reg_stage<1>(v);          // 4
        lane_stage(v, lane, 3);   // 5
        lane_stage(v, lane, 4);   // 6
        reg_stage<2>(v);          // 7
        reg_stage<3>(v);          // 8
        reg_stage<4>(v);          // 9
#pragma unroll
        for (int r = 0; r < 32; ++r) wr[1024 * b + enc_elem(lane, r)] = v[r] * 0.03125;
    }
    for (int i = tid; i < cols / 32; i += kEncThreads) outmap[i] = 0u;
    __syncthreads();

    // 2. sign words: bit 1 where the rotated weight is negative
    uint32_t* signs = reinterpret_cast<uint32_t*>(dst + L.off_signs) + int64_t(row) * (cols / 32);
    for (int wd = tid; wd < cols / 32; wd += kEncThreads) {
        uint32_t bits = 0;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) bits |= uint32_t(wr[32 * wd + i] < 0.0) << i;
        signs[wd] = bits;
    }

    // 3. the k outliers: k rounds of a block-wide arg-max over the columns not taken
    const int per = cols / kEncThreads;   // columns tid + 256 j, j < per (<= 64)
    unsigned long long taken = 0ull;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        EncKey best{0ull, 0x7FFFFFFF};
        bool have = false;
#pragma unroll 1
        for (int i = 0; i < per; ++i) {
            if ((taken >> i) & 1ull) continue;
            const int c = tid + kEncThreads * i;
            const EncKey kk{static_cast<unsigned long long>(__double_as_longlong(fabs(wr[c]))), c};
            if (!have || enc_better(kk, best)) {
                best = kk;
                have = true;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            EncKey other;
            other.mag = __shfl_xor_sync(0xffffffffu, best.mag, o);
            other.col = __shfl_xor_sync(0xffffffffu, best.col, o);
            if (enc_better(other, best)) best = other;
        }
        if (lane == 0) wbest[warp] = best;
        __syncthreads();
        if (tid == 0) {
            EncKey b = wbest[0];
            for (int x = 1; x < kEncThreads / 32; ++x)
                if (enc_better(wbest[x], b)) b = wbest[x];
            sel[j] = b.col;
            outmap[b.col >> 5] |= 1u << (b.col & 31);
        }
        __syncthreads();
        const int c = sel[j];
        if ((c & (kEncThreads - 1)) == tid) taken |= 1ull << (c / kEncThreads);
    }

    // 4. outlier columns in ascending order, their codes and the row scale
    if (k > 0) {
        const double amax = fabs(wr[sel[0]]);
        const __half sr = __double2half(amax / 7.0);
        const double srd = double(__half2float(sr));
        if (tid == 0) reinterpret_cast<__half*>(dst + L.off_srow)[row] = sr;
        for (int j = tid; j < k; j += kEncThreads) {
            const int c = sel[j];
            int rank = 0;
            for (int i = 0; i < k; ++i) rank += sel[i] < c;
            reinterpret_cast<uint16_t*>(dst + L.off_idx)[int64_t(row) * k + rank] = uint16_t(c);
            int qv = 0;
            if (srd > 0.0) qv = max(-7, min(7, int(rint(wr[c] / srd))));
            const int64_t n = int64_t(row) * k + rank;              // nibble index
            const int64_t byte = n >> 1;
            unsigned int* word = reinterpret_cast<unsigned int*>(dst + L.off_q + (byte & ~int64_t(3)));
            atomicOr(word, (uint32_t(qv) & 0xFu) << (8 * (byte & 3) + 4 * (n & 1)));
        }
    }
    __syncthreads();

    // 5. block scales: mean |w| over the block's kept weights, summed in column order
    const int nb = cols / 128;
    for (int b = tid; b < nb; b += kEncThreads) {
        double sum = 0.0;
        int cnt = 0;
#pragma unroll 4
        for (int i = 0; i < 128; ++i) {
            const int c = 128 * b + i;
            if ((outmap[c >> 5] >> (c & 31)) & 1u) continue;
            sum += fabs(wr[c]);
            ++cnt;
        }
        reinterpret_cast<__half*>(dst + L.off_sblk)[int64_t(row) * nb + b] =
            __double2half(cnt > 0 ? sum / double(cnt) : 0.0);
    }
}

}  // namespace

}  // namespace gale

extern "C" int gale_encode(const float* w, int rows, int cols, void* dst, void* stream) {
    using namespace gale;
    if (rows < 1 || cols < 1024 || cols % 1024 || cols > 65536 || !w || !dst) return GALE_ERR_ARG;
    if (cols > kEncMaxCols) return GALE_ERR_UNSUPPORTED;
    if (!aligned(dst, 16) || !aligned(w, 4)) return GALE_ERR_ALIGN;
    const Layout L = make_layout(rows, cols);
    cudaStream_t st = as_stream(stream);
    GALE_CUDA_TRY(cudaMemsetAsync(dst, 0, size_t(L.total), st));
    const int smem = cols * 8 + cols / 8 + 4 * ((L.k + 1) & ~1) + 8 * int(sizeof(EncKey));
    if (cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return GALE_ERR_CUDA;
    encode_kernel<<<unsigned(rows), kEncThreads, smem, st>>>(w, rows, cols, L.k, static_cast<char*>(dst), L);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

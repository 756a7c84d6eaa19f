// gale_selftest: start-up self-verification (the card's "optional fast paths
// verify themselves at startup" -- here with no fallback, only a status).
//
// Checks two closed forms on a tiny case:
//  1. A unit-scale matrix (every s_blk = s_row = 1) times an integer vector is
//     an exact integer sum: sum_c (bit ? -1 : +1) x_c, with outlier columns
//     replaced by q.  The GPU result must match the host's integer sum exactly,
//     through gale_pack and gale_expert_gemv.
//  2. The normalised FWHT is an involution: FWHT(FWHT(x)) == x within 1e-5.
#include <math.h>
#include <string.h>

#include <vector>

#include "common.cuh"

namespace {

constexpr int kR = 16, kC = 1024;

struct Scratch {
    int64_t signs, sblk, srow, idx, q, packed, x, y, status, total;
};

Scratch scratch_layout() {
    using gale::align_up;
    const int k = gale::outliers_per_row(kC);
    Scratch s{};
    int64_t o = 0;
    auto take = [&](int64_t b) { int64_t r = o; o = align_up(o + b, 256); return r; };
    s.signs = take(kR * kC);
    s.sblk = take(kR * (kC / 128) * 2);
    s.srow = take(kR * 2);
    s.idx = take(kR * k * 2);
    s.q = take(kR * k);
    s.packed = take(gale::make_layout(kR, kC).total);
    s.x = take(2 * kC * 4);
    s.y = take(kR * 4);
    s.status = take(4);
    s.total = o;
    return s;
}

}  // namespace

extern "C" size_t gale_selftest_scratch_bytes(void) { return size_t(scratch_layout().total); }

extern "C" int gale_selftest(void* scratch, void* stream) {
    if (!scratch) return GALE_ERR_ARG;
    if (!gale::aligned(scratch, 256)) return GALE_ERR_ALIGN;
    cudaStream_t st = gale::as_stream(stream);
    const Scratch s = scratch_layout();
    char* d = static_cast<char*>(scratch);
    const int k = gale::outliers_per_row(kC);

    std::vector<uint8_t> signs(kR * kC);
    uint32_t lcg = 12345u;
    for (auto& b : signs) {
        lcg = lcg * 1664525u + 1013904223u;
        b = uint8_t(lcg >> 31);
    }
    std::vector<uint16_t> sblk(kR * (kC / 128), 0x3C00), srow(kR, 0x3C00), idx(kR * k);
    std::vector<int8_t> q(kR * k);
    for (int r = 0; r < kR; ++r)
        for (int j = 0; j < k; ++j) {
            idx[r * k + j] = uint16_t(j * 97 + r);
            q[r * k + j] = int8_t((r + 3 * j) % 16 - 8);
        }
    std::vector<float> x(2 * kC);
    for (int c = 0; c < kC; ++c) x[c] = float((c * 7 + 3) % 17 - 8);
    for (int c = 0; c < kC; ++c) x[kC + c] = float((c * 13 + 5) % 31 - 15) * 0.125f;

    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.signs, signs.data(), signs.size(), cudaMemcpyHostToDevice, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.sblk, sblk.data(), sblk.size() * 2, cudaMemcpyHostToDevice, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.srow, srow.data(), srow.size() * 2, cudaMemcpyHostToDevice, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.idx, idx.data(), idx.size() * 2, cudaMemcpyHostToDevice, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.q, q.data(), q.size(), cudaMemcpyHostToDevice, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(d + s.x, x.data(), x.size() * 4, cudaMemcpyHostToDevice, st));
    int rc = gale_pack(reinterpret_cast<uint8_t*>(d + s.signs), reinterpret_cast<uint16_t*>(d + s.sblk),
                       reinterpret_cast<uint16_t*>(d + s.srow), reinterpret_cast<uint16_t*>(d + s.idx),
                       reinterpret_cast<int8_t*>(d + s.q), kR, kC, d + s.packed,
                       reinterpret_cast<int32_t*>(d + s.status), stream);
    if (rc != GALE_OK) return rc;
    gale_matrix W{d + s.packed, kR, kC};
    rc = gale_expert_gemv(&W, nullptr, reinterpret_cast<float*>(d + s.x), 1, reinterpret_cast<float*>(d + s.y),
                          GALE_MODE_PLAIN, stream);
    if (rc != GALE_OK) return rc;
    float* x2 = reinterpret_cast<float*>(d + s.x) + kC;
    rc = gale_fwht1024(x2, GALE_F32, x2, GALE_F32, 1, kC, stream);
    if (rc != GALE_OK) return rc;
    rc = gale_fwht1024(x2, GALE_F32, x2, GALE_F32, 1, kC, stream);
    if (rc != GALE_OK) return rc;
    std::vector<float> y(kR), xr(kC);
    int32_t dev_status = 0;
    GALE_CUDA_TRY(cudaMemcpyAsync(y.data(), d + s.y, kR * 4, cudaMemcpyDeviceToHost, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(xr.data(), x2, kC * 4, cudaMemcpyDeviceToHost, st));
    GALE_CUDA_TRY(cudaMemcpyAsync(&dev_status, d + s.status, 4, cudaMemcpyDeviceToHost, st));
    GALE_CUDA_TRY(cudaStreamSynchronize(st));
    if (dev_status != 0) return GALE_ERR_ARG;
    for (int r = 0; r < kR; ++r) {
        long want = 0;
        for (int c = 0; c < kC; ++c) want += (signs[r * kC + c] ? -1 : 1) * long(x[c]);
        for (int j = 0; j < k; ++j) {
            int c = idx[r * k + j];
            want += (long(q[r * k + j]) - (signs[r * kC + c] ? -1 : 1)) * long(x[c]);
        }
        if (y[r] != float(want)) return GALE_ERR_SELFTEST;
    }
    for (int c = 0; c < kC; ++c)
        if (fabsf(xr[c] - x[kC + c]) > 1e-5f) return GALE_ERR_SELFTEST;
    return GALE_OK;
}

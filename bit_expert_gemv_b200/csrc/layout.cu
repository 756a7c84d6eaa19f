// Host-side entry points with no kernels: status strings, the packed-matrix
// layout and the per-device attribute cache.
#include "common.cuh"

namespace gale {

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace gale

extern "C" const char* gale_status_string(int status) {
    switch (status) {
        case GALE_OK: return "GALE_OK";
        case GALE_ERR_ARG: return "GALE_ERR_ARG: invalid argument or invalid device input";
        case GALE_ERR_ALIGN: return "GALE_ERR_ALIGN: pointer alignment";
        case GALE_ERR_WORKSPACE: return "GALE_ERR_WORKSPACE: workspace missing or too small";
        case GALE_ERR_CUDA: return "GALE_ERR_CUDA: CUDA runtime call or launch failed";
        case GALE_ERR_TIMEOUT: return "GALE_ERR_TIMEOUT: bounded device wait ran out";
        case GALE_ERR_UNSUPPORTED: return "GALE_ERR_UNSUPPORTED: shape or device not supported";
        case GALE_ERR_SELFTEST: return "GALE_ERR_SELFTEST: a self-check result differs from its expected value";
        default: return "GALE: unknown status";
    }
}

extern "C" int gale_pack_layout(int rows, int cols, gale_layout* out) {
    if (!out || rows < 1 || !gale::valid_cols(cols)) return GALE_ERR_ARG;
    gale::Layout L = gale::make_layout(rows, cols);
    out->rows = rows;
    out->cols = cols;
    out->k = L.k;
    out->reserved = 0;
    int64_t r = rows;
    out->offset[0] = L.off_signs; out->size[0] = r * cols / 8;
    out->offset[1] = L.off_sblk;  out->size[1] = r * (cols / gale::kBlock) * 2;
    out->offset[2] = L.off_srow;  out->size[2] = r * 2;
    out->offset[3] = L.off_idx;   out->size[3] = r * L.k * 2;
    out->offset[4] = L.off_q;     out->size[4] = (r * L.k + 1) / 2;
    out->total = L.total;
    return GALE_OK;
}

extern "C" int64_t gale_expert_bytes(int d_model, int d_ff) {
    if (!gale::valid_cols(d_model) || !gale::valid_cols(d_ff)) return 0;
    return 2 * gale::make_layout(d_ff, d_model).total + gale::make_layout(d_model, d_ff).total;
}

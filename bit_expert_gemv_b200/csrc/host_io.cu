// gale_moe_forward_host: the MoE layer with its inputs read from, and its
// result written to, host memory.
//
// A decode step moves little data but pays a fixed cost per transfer: the
// inputs (x, ids, gates) are packed into one caller-owned pinned staging
// buffer and cross to the device in a single copy, and a small result is
// written by the layer kernels straight into the caller's pinned output
// buffer (no separate device-to-host copy).  Larger results go through a
// device buffer and one copy back.
#include <cstring>

#include "common.cuh"
#include "moe.cuh"

namespace {

constexpr size_t kDirectOutBytes = size_t(1) << 20;   // results up to 1 MiB are written in place

inline size_t up256(size_t n) { return (n + 255) & ~size_t(255); }

struct HostLayout {
    size_t x, ids, gates, bytes;   // offsets inside the staging buffer (and its device copy)
};

inline HostLayout host_layout(int B, int K, int d_model) {
    HostLayout h;
    h.x = 0;
    h.ids = up256(size_t(B) * d_model * 2);
    h.gates = h.ids + up256(size_t(B) * K * 4);
    h.bytes = h.gates + up256(size_t(B) * K * 4);
    return h;
}

inline size_t out_bytes(int B, int d_model, int out_dtype) {
    return size_t(B) * d_model * (out_dtype == GALE_F32 ? 4 : 2);
}

// Pinned (page-locked, device-visible) host memory or device memory.
inline bool device_visible(const void* p, bool allow_device) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost || (allow_device && (a.type == cudaMemoryTypeDevice ||
                                                             a.type == cudaMemoryTypeManaged));
}

}  // namespace

extern "C" size_t gale_moe_host_staging_bytes(int B, int K, int d_model) {
    if (B < 0 || K < 1 || K > 16 || d_model < 1) return 0;
    return host_layout(B, K, d_model).bytes;
}

extern "C" size_t gale_moe_host_workspace_size(const gale_layer* layer, int B, int K) {
    const size_t ws = gale_moe_workspace_size(layer, B, K);
    if (ws == 0) return 0;
    // the forward's workspace, the device copy of the staging buffer, a device output buffer
    return up256(ws) + host_layout(B, K, layer->d_model).bytes + up256(out_bytes(B, layer->d_model, GALE_F32));
}

extern "C" int gale_moe_forward_host(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                                     const float* gates, int B, int K, void* out, int out_dtype, int flags,
                                     float eps, void* ws, size_t ws_bytes, void* staging, size_t staging_bytes,
                                     void* stream) {
    using namespace gale;
    int rc = validate_layer(layer);
    if (rc != GALE_OK) return rc;
    if (B < 0 || K < 1 || K > 16 || (out_dtype != GALE_F32 && out_dtype != GALE_BF16)) return GALE_ERR_ARG;
    const size_t need = gale_moe_host_workspace_size(layer, B, K);
    if (need == 0 || !ws || ws_bytes < need) return GALE_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return GALE_ERR_ALIGN;
    const HostLayout hl = host_layout(B, K, layer->d_model);
    if (B == 0) return gale_moe_forward(layer, nullptr, nullptr, nullptr, 0, K, nullptr, out_dtype, flags, eps, ws,
                                        ws_bytes, stream);
    if (!x || !ids || !gates || !out || !staging || staging_bytes < hl.bytes) return GALE_ERR_ARG;
    if (!aligned(staging, 16) || !aligned(out, 4)) return GALE_ERR_ALIGN;
    if (!device_visible(staging, false) || !device_visible(out, true)) return GALE_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    // pack the inputs (host copies), then one copy to the device
    char* sb = static_cast<char*>(staging);
    std::memcpy(sb + hl.x, x, size_t(B) * layer->d_model * 2);
    std::memcpy(sb + hl.ids, ids, size_t(B) * K * 4);
    std::memcpy(sb + hl.gates, gates, size_t(B) * K * 4);
    const size_t fws = up256(gale_moe_workspace_size(layer, B, K));
    char* dev_in = static_cast<char*>(ws) + fws;
    GALE_CUDA_TRY(cudaMemcpyAsync(dev_in, sb, hl.bytes, cudaMemcpyHostToDevice, st));
    const uint16_t* dx = reinterpret_cast<const uint16_t*>(dev_in + hl.x);
    const int32_t* di = reinterpret_cast<const int32_t*>(dev_in + hl.ids);
    const float* dg = reinterpret_cast<const float*>(dev_in + hl.gates);
    const size_t ob = out_bytes(B, layer->d_model, out_dtype);
    if (ob <= kDirectOutBytes) {
        // the kernels write the result into the pinned (device-visible) buffer
        void* dout = nullptr;
        cudaPointerAttributes a{};
        GALE_CUDA_TRY(cudaPointerGetAttributes(&a, out));
        dout = a.devicePointer ? a.devicePointer : out;
        return gale_moe_forward(layer, dx, di, dg, B, K, dout, out_dtype, flags, eps, ws, fws, stream);
    }
    void* dev_out = dev_in + hl.bytes;
    rc = gale_moe_forward(layer, dx, di, dg, B, K, dev_out, out_dtype, flags, eps, ws, fws, stream);
    if (rc != GALE_OK) return rc;
    GALE_CUDA_TRY(cudaMemcpyAsync(out, dev_out, ob, cudaMemcpyDeviceToHost, st));
    return GALE_OK;
}

// gale_moe_forward_noalloc: the MoE layer with its workspace in a fixed
// device array of the library instead of caller-provided memory.
//
// Some callers cannot allocate device memory at the point where they run a
// layer: a plugin that lives inside a host runtime which owns the whole
// device memory pool, or a process that has fixed its device footprint at
// start-up and may not grow it afterwards.  They still own the inputs and
// outputs; only the scratch that gale_moe_forward needs comes from here.
#include <mutex>

#include "common.cuh"
#include "moe.cuh"

namespace {

// File-scope scratch.  Every GPU that loads the library holds this many bytes
// until the process exits.  All calls on one device share it.
__device__ __align__(256) unsigned char g_noalloc_scratch[GALE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  The array's
// name in host code is only a host-side stand-in; the device address comes
// from cudaGetSymbolAddress with that device current.  It is looked up again
// on every call made outside stream capture (a context that was reset and
// created again may place the array elsewhere); a call inside a capture uses
// the address of the last uncaptured call on the device.
int scratch_address(cudaStream_t st, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GALE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GALE_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return GALE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cs == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GALE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    } else if (!g_scratch_addr[dev]) {
        return GALE_ERR_UNSUPPORTED;   // no uncaptured call on this device yet
    }
    *out = g_scratch_addr[dev];
    return GALE_OK;
}

}  // namespace

extern "C" int gale_moe_forward_noalloc(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                                        const float* gates, int B, int K, void* out, int out_dtype, int flags,
                                        float eps, int32_t* status, void* stream) {
    int rc = gale::validate_layer(layer);
    if (rc != GALE_OK) return rc;
    if (B < 0 || K < 1 || K > 16) return GALE_ERR_ARG;
    const size_t need = gale_moe_workspace_size(layer, B, K);
    if (need == 0) return GALE_ERR_ARG;
    if (need > size_t(GALE_NOALLOC_SCRATCH_BYTES)) return GALE_ERR_WORKSPACE;
    if (status && !gale::aligned(status, 4)) return GALE_ERR_ALIGN;
    void* ws = nullptr;
    rc = scratch_address(gale::as_stream(stream), &ws);
    if (rc != GALE_OK) return rc;
    rc = gale_moe_forward(layer, x, ids, gates, B, K, out, out_dtype, flags, eps, ws,
                          size_t(GALE_NOALLOC_SCRATCH_BYTES), stream);
    if (rc != GALE_OK) return rc;
    if (status)
        GALE_CUDA_TRY(cudaMemcpyAsync(status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                                      gale::as_stream(stream)));
    return GALE_OK;
}

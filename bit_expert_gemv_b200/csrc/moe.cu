// gale_moe_forward: one routed-expert layer,
//   y[t] = sum_k gates[t,k] * W2_e H( silu(W1_e H x[t]) * (W3_e H x[t]) ),  e = ids[t,k]
// (SwiGLU experts over GALE 1-bit packed records, top-K routing).
//
// Stages: routing permute -> FWHT(x) -> grouped w1/w3 GEMV + SwiGLU ->
// FWHT(h) -> grouped w2 GEMV -> deterministic gate-weighted combine in fixed
// k order (optionally + residual and RMSNorm).
#include "common.cuh"
#include "gemv_simple.cuh"
#include "moe.cuh"
#include "moe_decode.cuh"
#include "moe_stream.cuh"
#include "moe_prefill.cuh"
#include "route.cuh"

namespace gale {

constexpr int kGWarps = 8;
constexpr int kGRowsPerWarp = 8;
constexpr int kGRowsPerCta = kGWarps * kGRowsPerWarp;

// One or two tokens take the small-batch decode kernel (measured faster there
// than the streaming kernel, whose per-CTA planning and phase hand-off cost
// more than they save at this size).
bool small_batch(const gale_layer& L, int B, int K) { return B >= 1 && B <= 2 && decode_supported(L, B, K); }

MoeWs carve_ws(void* ws, const gale_layer& L, int B, int K) {
    MoeWs w{};
    char* p = static_cast<char*>(ws);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        char* q = p ? p + o : nullptr;
        o = align_up(o + bytes, 256);
        return q;
    };
    const int64_t BK = int64_t(B) * K;
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.counts = reinterpret_cast<int32_t*>(take(4 * int64_t(L.n_experts)));
    w.offsets = reinterpret_cast<int32_t*>(take(4 * (int64_t(L.n_experts) + 1)));
    w.perm = reinterpret_cast<int32_t*>(take(4 * BK));
    w.pos_of_pair = reinterpret_cast<int32_t*>(take(4 * BK));
    w.active = reinterpret_cast<int32_t*>(take(4 * int64_t(L.n_experts)));
    w.n_active = reinterpret_cast<int32_t*>(take(4));
    w.x_rot = reinterpret_cast<float*>(take(4 * int64_t(B) * L.d_model));
    w.h = reinterpret_cast<float*>(take(4 * BK * L.d_ff));
    w.o = reinterpret_cast<float*>(take(4 * BK * L.d_model));
    w.bytes = size_t(o);
    return w;
}

// Grouped GEMV: CTA (row tile, active slot).  The slot's expert e processes
// its pairs in permuted order; w1/w3 read x_rot of the pair's token, w2 reads
// the pair's own rotated hidden row.
template <bool SWIGLU>
__global__ void __launch_bounds__(256) moe_group_gemv_kernel(GroupArgs g) {
    extern __shared__ float xs[];
    const int slot = blockIdx.y;
    if (slot >= *g.n_active) return;
    const int e = g.active[slot];
    const int n_e = g.counts[e];
    const int off = g.offsets[e];
    const char* rec = static_cast<const char*>(g.base) + int64_t(e) * g.expert_stride;
    const MatView a = make_view(rec + g.mat_off_a, g.rows, g.cols);
    const MatView b = make_view(rec + g.mat_off_b, g.rows, g.cols);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cols = g.cols;
    for (int t0 = 0; t0 < n_e; t0 += g.chunk) {
        const int nt = min(g.chunk, n_e - t0);
        __syncthreads();
        for (int i = threadIdx.x; i < nt * cols; i += blockDim.x) {
            const int ti = i / cols, c = i - ti * cols;
            const int64_t src_row = SWIGLU ? int64_t(g.perm[off + t0 + ti] / g.K) : int64_t(off + t0 + ti);
            xs[i] = g.x[src_row * cols + c];
        }
        __syncthreads();
        for (int i = 0; i < kGRowsPerWarp; ++i) {
            const int r = blockIdx.x * kGRowsPerCta + i * kGWarps + warp;
            if (r >= g.rows) break;
            float acc[kSimpleNT];
            row_dot_simple(a, r, xs, nt, acc, lane);
            if (SWIGLU) {
                float acc3[kSimpleNT];
                row_dot_simple(b, r, xs, nt, acc3, lane);
#pragma unroll
                for (int t = 0; t < kSimpleNT; ++t) acc[t] = silu(acc[t]) * acc3[t];
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kSimpleNT; ++t)
                    if (t < nt) g.out[int64_t(off + t0 + t) * g.rows + r] = acc[t];
            }
        }
    }
}

// One CTA per token: y = sum_k gates[t,k] * o[pos(t,k)] in fixed k order,
// then either stored, or v = x + y normalised (RMSNorm, unit weight) to bf16.
// The token's slots and gates are read once into shared memory; each thread
// takes four consecutive columns at a time with all K loads in flight.
__global__ void __launch_bounds__(256) moe_combine_kernel(CombineArgs c) {
    __shared__ int spos[16];
    __shared__ float sg[16];
    __shared__ float red[32];
    const int t = blockIdx.x;
    const int d = c.d_model, n4 = d / 4;
    if (threadIdx.x < c.K) {
        spos[threadIdx.x] = c.pos_of_pair[t * c.K + threadIdx.x];
        sg[threadIdx.x] = c.gates[t * c.K + threadIdx.x];
    }
    __syncthreads();
    float ss = 0.f;
    for (int i4 = threadIdx.x; i4 < n4; i4 += blockDim.x) {
        float4 ov[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            ov[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k < c.K && spos[k] >= 0) ov[k] = __ldcs(reinterpret_cast<const float4*>(c.o + int64_t(spos[k]) * d) + i4);
        }
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (k >= c.K) break;
            const float g = spos[k] >= 0 ? sg[k] : 0.f;
            y.x = fmaf(g, ov[k].x, y.x);
            y.y = fmaf(g, ov[k].y, y.y);
            y.z = fmaf(g, ov[k].z, y.z);
            y.w = fmaf(g, ov[k].w, y.w);
        }
        const int64_t e = int64_t(t) * d + 4 * i4;
        if (c.fuse_norm) {
            // x is only known to be 4-byte aligned: two 32-bit loads
            const uint32_t x01 = *reinterpret_cast<const uint32_t*>(c.x + e);
            const uint32_t x23 = *reinterpret_cast<const uint32_t*>(c.x + e + 2);
            const float4 v = make_float4(bf16_to_f32(uint16_t(x01)) + y.x, bf16_to_f32(uint16_t(x01 >> 16)) + y.y,
                                         bf16_to_f32(uint16_t(x23)) + y.z, bf16_to_f32(uint16_t(x23 >> 16)) + y.w);
            reinterpret_cast<float4*>(c.scratch + int64_t(t) * d)[i4] = v;
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
        } else {
            store_from_f32(c.out, c.out_dtype, e, y.x);
            store_from_f32(c.out, c.out_dtype, e + 1, y.y);
            store_from_f32(c.out, c.out_dtype, e + 2, y.z);
            store_from_f32(c.out, c.out_dtype, e + 3, y.w);
        }
    }
    if (!c.fuse_norm) return;
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        v = warp_sum(v);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float inv = rsqrtf(red[0] / float(d) + c.eps);
    uint16_t* out = static_cast<uint16_t*>(c.out);
    for (int i4 = threadIdx.x; i4 < n4; i4 += blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(c.scratch + int64_t(t) * d)[i4];
        const int64_t e = int64_t(t) * d + 4 * i4;
        out[e] = f32_to_bf16(v.x * inv);
        out[e + 1] = f32_to_bf16(v.y * inv);
        out[e + 2] = f32_to_bf16(v.z * inv);
        out[e + 3] = f32_to_bf16(v.w * inv);
    }
}

int launch_moe_combine(const float* o, const int32_t* pos_of_pair, const float* gates, const uint16_t* x, int B,
                       int K, int d_model, void* out, int out_dtype, bool fuse_norm, float eps, float* scratch,
                       cudaStream_t st) {
    CombineArgs c{};
    c.o = o;
    c.pos_of_pair = pos_of_pair;
    c.gates = gates;
    c.x = x;
    c.K = K;
    c.d_model = d_model;
    c.out = out;
    c.out_dtype = out_dtype;
    c.fuse_norm = fuse_norm;
    c.eps = eps;
    c.scratch = scratch;
    if (K > 16 || d_model % 4 != 0) return GALE_ERR_UNSUPPORTED;
    moe_combine_kernel<<<B, 256, 0, st>>>(c);
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

int validate_layer(const gale_layer* L) {
    if (!L || !L->base || L->n_experts < 1 || L->n_experts > 1024) return GALE_ERR_ARG;
    if (!valid_cols(L->d_model) || !valid_cols(L->d_ff) || L->d_model > 16384 || L->d_ff > 16384)
        return GALE_ERR_ARG;
    const int64_t eb = 2 * make_layout(L->d_ff, L->d_model).total + make_layout(L->d_model, L->d_ff).total;
    if (L->expert_stride < eb || L->expert_stride % 256) return GALE_ERR_ARG;
    if (!aligned(L->base, 256)) return GALE_ERR_ALIGN;
    return GALE_OK;
}

int launch_group_gemv(bool swiglu, GroupArgs g, int max_slots, cudaStream_t st) {
    const int chunk_cap = int((200 * 1024) / (int64_t(g.cols) * 4));
    g.chunk = chunk_cap < 1 ? 1 : (chunk_cap > kSimpleNT ? kSimpleNT : chunk_cap);
    const size_t smem = size_t(g.chunk) * g.cols * sizeof(float);
    dim3 grid((g.rows + kGRowsPerCta - 1) / kGRowsPerCta, max_slots);
    if (swiglu) {
        GALE_CUDA_TRY(cudaFuncSetAttribute(moe_group_gemv_kernel<true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
        moe_group_gemv_kernel<true><<<grid, 256, smem, st>>>(g);
    } else {
        GALE_CUDA_TRY(cudaFuncSetAttribute(moe_group_gemv_kernel<false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
        moe_group_gemv_kernel<false><<<grid, 256, smem, st>>>(g);
    }
    GALE_LAUNCH_CHECK();
    return GALE_OK;
}

}  // namespace gale

extern "C" size_t gale_moe_workspace_size(const gale_layer* layer, int B, int K) {
    if (gale::validate_layer(layer) == GALE_ERR_ARG || B < 0 || K < 1 || K > 16) return 0;
    size_t n = gale::carve_ws(nullptr, *layer, B, K).bytes;
    // each batch takes exactly one path; its workspace also holds the status word
    size_t p = 0;
    if (gale::small_batch(*layer, B, K)) p = gale::carve_decode_ws(nullptr, *layer, B, K).bytes;
    else if (gale::stream_supported(*layer, B, K)) p = gale::carve_stream_ws(nullptr, *layer, B, K).bytes;
    else if (gale::prefill_supported(*layer, B, K)) p = gale::carve_prefill_ws(nullptr, *layer, B, K).bytes;
    return p > n ? p : n;
}

extern "C" int gale_moe_forward(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                                const float* gates, int B, int K, void* out, int out_dtype, int flags,
                                float eps, void* ws, size_t ws_bytes, void* stream) {
    using namespace gale;
    int rc = validate_layer(layer);
    if (rc != GALE_OK) return rc;
    if (B < 0 || K < 1 || K > 16 || K > layer->n_experts) return GALE_ERR_ARG;
    if (flags & ~GALE_FLAG_RESIDUAL_RMSNORM) return GALE_ERR_ARG;
    const bool fuse = flags & GALE_FLAG_RESIDUAL_RMSNORM;
    if (out_dtype != GALE_F32 && out_dtype != GALE_BF16) return GALE_ERR_ARG;
    if (fuse && (out_dtype != GALE_BF16 || !(eps >= 0.f))) return GALE_ERR_ARG;
    if (!ws) return GALE_ERR_WORKSPACE;
    const gale_layer& L = *layer;
    MoeWs w = carve_ws(ws, L, B, K);
    const bool small = small_batch(L, B, K);
    const bool decode = !small && stream_supported(L, B, K);
    const bool prefill = !small && !decode && prefill_supported(L, B, K);
    if (ws_bytes < w.bytes || (small && ws_bytes < carve_decode_ws(nullptr, L, B, K).bytes) ||
        (decode && ws_bytes < carve_stream_ws(nullptr, L, B, K).bytes) ||
        (prefill && ws_bytes < carve_prefill_ws(nullptr, L, B, K).bytes))
        return GALE_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return GALE_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    // the status word (and the small-batch kernel's grid-barrier counters)
    if (!decode || B == 0) GALE_CUDA_TRY(cudaMemsetAsync(w.status, 0, 8 * sizeof(int32_t), st));
    if (B == 0) return GALE_OK;
    if (!x || !ids || !gates || !out) return GALE_ERR_ARG;
    if (!aligned(x, 4) || !aligned(ids, 4) || !aligned(gates, 4) || !aligned(out, 4)) return GALE_ERR_ALIGN;
    const int64_t BK = int64_t(B) * K;
    if (BK > (1 << 24)) return GALE_ERR_UNSUPPORTED;
    // one or two tokens: the small-batch decode kernel
    if (small) return launch_moe_decode(L, x, ids, gates, B, K, out, out_dtype, fuse, eps, ws, st);
    // other decode batches: the streaming kernel (it clears its own status word and counters)
    if (decode) return launch_moe_stream(L, x, ids, gates, B, K, out, out_dtype, fuse, eps, ws, st);
    // larger batches: tcgen05 tensor-core tiles
    if (prefill) return launch_moe_prefill(L, x, ids, gates, B, K, out, out_dtype, fuse, eps, ws, st);

    GALE_CUDA_TRY(cudaMemsetAsync(w.pos_of_pair, 0xFF, size_t(BK) * 4, st));
    RouteArgs ra{};
    ra.ids = ids;
    ra.B = B;
    ra.K = K;
    ra.E = L.n_experts;
    ra.counts = w.counts;
    ra.offsets = w.offsets;
    ra.perm = w.perm;
    ra.pos_of_pair = w.pos_of_pair;
    ra.active = w.active;
    ra.n_active = w.n_active;
    ra.status = w.status;
    rc = launch_route_permute(ra, st);
    if (rc != GALE_OK) return rc;

    rc = gale_fwht1024(x, GALE_BF16, w.x_rot, GALE_F32, B, L.d_model, stream);
    if (rc != GALE_OK) return rc;

    const int64_t w1_bytes = make_layout(L.d_ff, L.d_model).total;
    const int max_slots = int(BK < L.n_experts ? BK : L.n_experts);
    GroupArgs g{};
    g.base = L.base;
    g.expert_stride = L.expert_stride;
    g.counts = w.counts;
    g.offsets = w.offsets;
    g.perm = w.perm;
    g.active = w.active;
    g.n_active = w.n_active;
    g.K = K;
    g.rows = L.d_ff;
    g.cols = L.d_model;
    g.mat_off_a = 0;
    g.mat_off_b = w1_bytes;
    g.x = w.x_rot;
    g.out = w.h;
    rc = launch_group_gemv(true, g, max_slots, st);
    if (rc != GALE_OK) return rc;

    rc = gale_fwht1024(w.h, GALE_F32, w.h, GALE_F32, BK, L.d_ff, stream);
    if (rc != GALE_OK) return rc;

    g.rows = L.d_model;
    g.cols = L.d_ff;
    g.mat_off_a = 2 * w1_bytes;
    g.mat_off_b = 2 * w1_bytes;
    g.x = w.h;
    g.out = w.o;
    rc = launch_group_gemv(false, g, max_slots, st);
    if (rc != GALE_OK) return rc;

    // x_rot is dead by now; reused for v = x + y
    return launch_moe_combine(w.o, w.pos_of_pair, gates, x, B, K, L.d_model, out, out_dtype, fuse, eps, w.x_rot, st);
}

extern "C" size_t gale_moe_chain_workspace_size(const gale_layer* first, int n_layers, int B, int K) {
    if (gale::validate_layer(first) != GALE_OK || n_layers < 1 || n_layers > 4096 || B < 1 || K < 1 || K > 16 ||
        !gale::stream_supported(*first, B, K))
        return 0;
    return gale::carve_stream_ws(nullptr, *first, B, K, n_layers).bytes;
}

extern "C" int gale_moe_chain(const gale_layer* first, int n_layers, int64_t layer_stride, const uint16_t* x0,
                              const int32_t* ids, const float* gates, int B, int K, uint16_t* out, float eps,
                              void* ws, size_t ws_bytes, void* stream) {
    using namespace gale;
    int rc = validate_layer(first);
    if (rc != GALE_OK) return rc;
    const gale_layer& L = *first;
    if (n_layers < 1 || n_layers > 4096 || B < 1 || K < 1 || K > 16 || K > L.n_experts || !(eps >= 0.f))
        return GALE_ERR_ARG;
    if (layer_stride < int64_t(L.n_experts) * L.expert_stride || layer_stride % L.expert_stride)
        return GALE_ERR_ARG;
    if (!stream_supported(L, B, K)) return GALE_ERR_UNSUPPORTED;
    if (!x0 || !ids || !gates || !out) return GALE_ERR_ARG;
    if (!ws || ws_bytes < carve_stream_ws(nullptr, L, B, K, n_layers).bytes) return GALE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(x0, 4) || !aligned(ids, 4) || !aligned(gates, 4) || !aligned(out, 4))
        return GALE_ERR_ALIGN;
    return launch_moe_stream(L, x0, ids, gates, B, K, out, GALE_BF16, true, eps, ws, as_stream(stream), n_layers,
                             layer_stride / L.expert_stride);
}

extern "C" size_t gale_expert_forward_workspace_size(const gale_layer* layer, int B) {
    if (gale::validate_layer(layer) != GALE_OK || B < 1 || !gale::stream_supported(*layer, B, 1)) return 0;
    return gale::carve_stream_ws(nullptr, *layer, B, 1).bytes;
}

extern "C" int gale_expert_forward(const gale_layer* layer, int expert, const float* x, int B, float* out, void* ws,
                                   size_t ws_bytes, void* stream) {
    using namespace gale;
    int rc = validate_layer(layer);
    if (rc != GALE_OK) return rc;
    const gale_layer& L = *layer;
    if (expert < 0 || expert >= L.n_experts || B < 1 || !x || !out) return GALE_ERR_ARG;
    if (!stream_supported(L, B, 1)) return GALE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < carve_stream_ws(nullptr, L, B, 1).bytes) return GALE_ERR_WORKSPACE;
    if (!aligned(ws, 256) || !aligned(x, 4) || !aligned(out, 4)) return GALE_ERR_ALIGN;
    return launch_moe_stream(L, nullptr, nullptr, nullptr, B, 1, out, GALE_F32, false, 0.f, ws, as_stream(stream), 1, 0,
                             x, expert);
}

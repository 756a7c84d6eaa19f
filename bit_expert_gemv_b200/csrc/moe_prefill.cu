// Prefill path of gale_moe_forward (many tokens per expert): the expert
// products are real dense contractions, run on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM).
//
//   route   : stable counting sort of the (token, slot) pairs by expert
//   gather  : x of every pair, in permuted order, rotated (FWHT-1024) to fp16
//   w1/w3   : per (expert, 128-row tile, chunk of <= 256 tokens): the packed
//             signs are expanded to fp16 A tiles +-s_blk (exact) with the
//             outliers patched in (q * s_row, rounded to fp16), in the K-major
//             128-byte-swizzled layout the tensor core reads; the tokens come
//             in by TMA; both products accumulate in TMEM; SwiGLU epilogue
//   rotate  : h -> fp16 FWHT-1024
//   w2      : same tile kernel with one matrix
//   combine : gate-weighted sum in fixed k order (+ residual, RMSNorm)
#include "common.cuh"
#include "fwht.cuh"
#include "moe.cuh"
#include "moe_prefill.cuh"
#include "route.cuh"
#include "tc_prefill.cuh"
#include "tma.cuh"

namespace gale {

namespace {

constexpr int kTcM = 128;
constexpr int kTcK = 64;          // K per stage: one 128-byte row of fp16
constexpr int kTcNRows = 256;     // token rows per chunk
constexpr int kTcStages = 3;
constexpr int kTcThreads = 6 * 32;   // producer, MMA, 4 expander/epilogue warps
constexpr int kPrefetch = 4;      // K-steps of sign words loaded ahead

struct TcJob {
    int e, n0, n;   // expert, first slot of the chunk, tokens in the chunk
};

struct TcArgs {
    const char* base;
    int64_t stride;
    int64_t off_a, off_b;      // byte offsets of the matrices inside a record
    int rows, cols;            // of the streamed matrices
    const TcJob* jobs;
    const int32_t* n_jobs;
    float* out;                // [slots][rows] fp32
    int32_t* status;
};

struct TcSmem {
    int a0, a1, b, bars, misc, stage_bytes, bytes;
};

__host__ __device__ inline TcSmem tc_smem(int nmat) {
    TcSmem s;
    s.a0 = 0;
    s.a1 = kTcM * 128;
    s.b = s.a1 + (nmat == 2 ? kTcM * 128 : 0);
    s.stage_bytes = s.b + kTcNRows * 128;
    s.bars = kTcStages * s.stage_bytes;
    s.misc = s.bars + 8 * (3 * kTcStages + 1);
    s.bytes = int(align_up(s.misc + 64, 1024)) + 1024;
    return s;
}

// The job list: every expert with tokens, split into chunks of <= 256 slots.
__global__ void prefill_jobs_kernel(const int32_t* counts, const int32_t* offsets, int E, TcJob* jobs,
                                    int32_t* n_jobs) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int n = 0;
    for (int e = 0; e < E; ++e)
        for (int t0 = 0; t0 < counts[e]; t0 += kTcNRows) jobs[n++] = TcJob{e, offsets[e] + t0, min(kTcNRows, counts[e] - t0)};
    *n_jobs = n;
}

// x of every pair in permuted order, rotated, as fp16: one warp per (slot, 1024-block).
// Slots past the routed pairs (pairs with an invalid expert id are dropped)
// stay zero.
__global__ void __launch_bounds__(256) gather_rotate_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                                                            const int32_t* __restrict__ n_routed, int K, int d,
                                                            int64_t slots, __half* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
    const int nb = d / 1024;
    if (wid >= slots * nb) return;
    const int64_t s = wid / nb;
    if (s >= *n_routed) return;
    const int blk = int(wid - s * nb);
    const int t = perm[s] / K;
    const uint16_t* src = x + int64_t(t) * d + blk * 1024;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = bf16_to_f32(src[32 * i + lane]);
    fwht1024_warp(v, lane);
    __half* dst = y + s * d + blk * 1024;
#pragma unroll
    for (int i = 0; i < 32; ++i) dst[32 * i + lane] = __float2half_rn(v[i] * (1.0f / 32.0f));
}

// One (expert, 128-row tile, token chunk) job of w1/w3 (NMAT = 2, SwiGLU
// epilogue) or w2 (NMAT = 1).
template <int NMAT>
__global__ void __launch_bounds__(kTcThreads, 1) tc_tile_kernel(const __grid_constant__ CUtensorMap xmap, TcArgs A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(smem_raw), 1024));
    const int job_id = blockIdx.x, mtile = blockIdx.y;
    if (job_id >= *A.n_jobs) return;
    const TcJob job = A.jobs[job_id];
    const TcSmem S = tc_smem(NMAT);
    uint64_t* b_full = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* a_full = b_full + kTcStages;
    uint64_t* mma_done = a_full + kTcStages;
    uint64_t* acc_full = mma_done + kTcStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S.misc);
    int* fail = reinterpret_cast<int*>(smem + S.misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = A.cols / kTcK;
    const int n_mma = (job.n + 15) & ~15;
    const int nbox = (job.n + 63) / 64;
    const uint32_t idesc = umma_idesc_f16(kTcM, n_mma);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(b_full + s, 1);
            mbar_init(a_full + s, 128);
            mbar_init(mma_done + s, 1);
        }
        mbar_init(acc_full, 1);
        *fail = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- producer: token tiles by TMA
        if (lane == 0) {
            int issued = 0;
            for (int ks = 0; ks < nk; ++ks) {
                const int s = ks % kTcStages;
                if (ks >= kTcStages && !mbar_wait(mma_done + s, ((ks / kTcStages) - 1) & 1)) {
                    *fail = 1;
                    break;
                }
                uint8_t* bdst = smem + s * S.stage_bytes + S.b;
                mbar_arrive_expect_tx(b_full + s, uint32_t(nbox * 64 * 128));
                for (int bx = 0; bx < nbox; ++bx)
                    tma_load_3d(bdst + bx * 64 * 128, &xmap, b_full + s, ks * kTcK, job.n0 + bx * 64, 0);
                issued = ks + 1;
            }
            // no copy may still be landing when the CTA exits
            for (int ks = issued - kTcStages < 0 ? 0 : issued - kTcStages; ks < issued; ++ks)
                if (!mbar_wait(b_full + ks % kTcStages, (ks / kTcStages) & 1)) *fail = 1;
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            for (int ks = 0; ks < nk; ++ks) {
                const int s = ks % kTcStages;
                const uint32_t par = (ks / kTcStages) & 1;
                if (!mbar_wait(a_full + s, par) || !mbar_wait(b_full + s, par)) {
                    *fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * S.stage_bytes);
#pragma unroll
                for (int mt = 0; mt < NMAT; ++mt) {
#pragma unroll
                    for (int kk = 0; kk < kTcK / 16; ++kk) {
                        const uint64_t ad = umma_desc_sw128(st + (mt ? S.a1 : S.a0) + kk * 32);
                        const uint64_t bd = umma_desc_sw128(st + S.b + kk * 32);
                        umma_f16(tmem + uint32_t(mt * 256), ad, bd, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                umma_commit(mma_done + s);
            }
            umma_commit(acc_full);
        }
    } else {
        // ---------------- expanders: one weight row per thread
        const int t = threadIdx.x - 64;
        const int row = mtile * kTcM + t;
        const bool valid = row < A.rows;
        const char* rec = A.base + int64_t(job.e) * A.stride;
        MatView mv[NMAT];
#pragma unroll
        for (int mt = 0; mt < NMAT; ++mt) mv[mt] = make_view(rec + (mt ? A.off_b : A.off_a), A.rows, A.cols);
        const int nb = A.cols / 128;
        // next outlier of the row per matrix: its position n and column (cols when none is left)
        int on[NMAT], oc[NMAT];
        float srow[NMAT];
#pragma unroll
        for (int mt = 0; mt < NMAT; ++mt) {
            on[mt] = 0;
            oc[mt] = (valid && mv[mt].k > 0) ? int(mv[mt].idx[int64_t(row) * mv[mt].k]) : A.cols;
            srow[mt] = valid ? __half2float(mv[mt].s_row[row]) : 0.f;
        }
        // sign words and block scale of K-steps ks .. ks + kPrefetch - 1, per matrix
        uint2 wq[NMAT][kPrefetch];
        uint32_t sq[NMAT][kPrefetch];
        auto fetch = [&](int mt, int ks, uint2& w, uint32_t& sc) {
            w = make_uint2(0u, 0u);
            sc = 0u;
            if (valid && ks < nk) {
                w = __ldg(reinterpret_cast<const uint2*>(mv[mt].signs + int64_t(row) * (A.cols / 32)) + ks);
                sc = __ldg(reinterpret_cast<const uint16_t*>(mv[mt].s_blk) + int64_t(row) * nb + (ks >> 1));
            }
        };
#pragma unroll
        for (int mt = 0; mt < NMAT; ++mt)
#pragma unroll
            for (int p = 0; p < kPrefetch; ++p) fetch(mt, p, wq[mt][p], sq[mt][p]);
        bool ok = true;
        for (int ks = 0; ks < nk; ++ks) {
            const int s = ks % kTcStages;
            if (ok && ks >= kTcStages && !mbar_wait(mma_done + s, ((ks / kTcStages) - 1) & 1)) {
                ok = false;
                *fail = 1;
            }
            const int slot = ks % kPrefetch;
#pragma unroll
            for (int mt = 0; mt < NMAT; ++mt) {
                // this K-step's words, then refill the slot kPrefetch steps ahead
                uint2 w = make_uint2(0u, 0u);
                uint32_t sc = 0u;
#pragma unroll
                for (int p = 0; p < kPrefetch; ++p)
                    if (p == slot) {
                        w = wq[mt][p];
                        sc = sq[mt][p];
                        fetch(mt, ks + kPrefetch, wq[mt][p], sq[mt][p]);
                    }
                uint8_t* arow = smem + s * S.stage_bytes + (mt ? S.a1 : S.a0) + t * 128;
                const uint32_t h2 = sc | (sc << 16);
                // 16-byte chunk c holds columns 8c .. 8c+7; a set sign bit negates the fp16 scale
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t byte = ((c < 4 ? w.x : w.y) >> (8 * (c & 3))) & 0xFFu;
                    uint32_t v[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        v[p] = h2 ^ (((byte >> (2 * p)) & 1u) << 15) ^ (((byte >> (2 * p + 1)) & 1u) << 31);
                    *reinterpret_cast<uint4*>(arow + ((c ^ (t & 7)) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
                }
                // outliers of this K-step replace their weights by q * s_row
                const int kend = (ks + 1) * kTcK;
                while (oc[mt] < kend) {
                    const int64_t n = int64_t(row) * mv[mt].k + on[mt];
                    const int c = oc[mt] - ks * kTcK;
                    const __half val = __float2half_rn(float(load_q(mv[mt].q, n)) * srow[mt]);
                    if (c >= 0)   // indices are strictly ascending in a valid record
                        *reinterpret_cast<__half*>(arow + (((c >> 3) ^ (t & 7)) << 4) + (c & 7) * 2) = val;
                    ++on[mt];
                    oc[mt] = on[mt] < mv[mt].k ? int(mv[mt].idx[n + 1]) : A.cols;
                }
            }
            fence_proxy_async();
            mbar_arrive(a_full + s);
        }
        // ---------------- epilogue: TMEM -> registers -> global
        const bool acc_ok = mbar_wait(acc_full, 0);
        ok = __all_sync(0xffffffffu, ok && acc_ok);
        if (!ok) *fail = 1;
        tc_fence_after();
        const int q = warp & 3;   // TMEM lane quarter this warp may read
        const int erow = mtile * kTcM + 32 * q + lane;
        if (ok) {
            for (int col = 0; col < n_mma; col += 16) {
                float v1[16], v3[16];
                tmem_ld16(tmem + (uint32_t(32 * q) << 16) + uint32_t(col), v1);
                if (NMAT == 2) tmem_ld16(tmem + (uint32_t(32 * q) << 16) + uint32_t(256 + col), v3);
                if (erow < A.rows) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int j = col + i;
                        if (j < job.n) {
                            const float y = NMAT == 2 ? silu(v1[i]) * v3[i] : v1[i];
                            A.out[int64_t(job.n0 + j) * A.rows + erow] = y;
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *fail) set_status(A.status, GALE_ERR_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

int act_map(CUtensorMap* m, const void* base, int cols, int64_t rows) {
    // fp16 [rows][cols], boxes of 64 columns x 64 rows, 128-byte swizzle
    return make_map_3d(m, true, base, uint64_t(cols), uint64_t(rows), 1, uint64_t(cols) * 2,
                       uint64_t(cols) * 2 * uint64_t(rows), 64, 64, true);
}

}  // namespace

PrefillWs carve_prefill_ws(void* ws, const gale_layer& L, int B, int K) {
    PrefillWs w{};
    char* p = static_cast<char*>(ws);
    int64_t o = 0;
    auto take = [&](int64_t bytes) {
        char* q = p ? p + o : nullptr;
        o = align_up(o + bytes, 256);
        return q;
    };
    const int64_t P = int64_t(B) * K, dm = L.d_model, df = L.d_ff;
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.counts = reinterpret_cast<int32_t*>(take(4 * int64_t(L.n_experts)));
    w.offsets = reinterpret_cast<int32_t*>(take(4 * (int64_t(L.n_experts) + 1)));
    w.perm = reinterpret_cast<int32_t*>(take(4 * P));
    w.pos_of_pair = reinterpret_cast<int32_t*>(take(4 * P));
    const int64_t max_jobs = L.n_experts + P / kTcNRows + 1;
    w.jobs = take(int64_t(sizeof(TcJob)) * max_jobs);
    w.n_jobs = reinterpret_cast<int32_t*>(take(4));
    w.max_jobs = int(max_jobs);
    w.x16 = reinterpret_cast<__half*>(take(2 * P * dm));
    w.h = reinterpret_cast<float*>(take(4 * P * df));
    w.h16 = reinterpret_cast<__half*>(take(2 * P * df));
    w.o = reinterpret_cast<float*>(take(4 * P * dm));
    w.scratch = reinterpret_cast<float*>(take(4 * int64_t(B) * dm));
    w.bytes = size_t(o);
    return w;
}

bool prefill_supported(const gale_layer& L, int B, int K) {
    return int64_t(B) * K <= (int64_t(1) << 24) && L.d_model <= 16384 && L.d_ff <= 16384;
}

int launch_moe_prefill(const gale_layer& L, const uint16_t* x, const int32_t* ids, const float* gates, int B, int K,
                       void* out, int out_dtype, bool fuse_norm, float eps, void* ws, cudaStream_t st) {
    PrefillWs w = carve_prefill_ws(ws, L, B, K);
    const int64_t P = int64_t(B) * K;
    GALE_CUDA_TRY(cudaMemsetAsync(w.pos_of_pair, 0xFF, size_t(P) * 4, st));
    RouteArgs ra{};
    ra.ids = ids;
    ra.B = B;
    ra.K = K;
    ra.E = L.n_experts;
    ra.counts = w.counts;
    ra.offsets = w.offsets;
    ra.perm = w.perm;
    ra.pos_of_pair = w.pos_of_pair;
    ra.status = w.status;
    int rc = launch_route_permute(ra, st);
    if (rc != GALE_OK) return rc;
    prefill_jobs_kernel<<<1, 32, 0, st>>>(w.counts, w.offsets, L.n_experts, static_cast<TcJob*>(w.jobs), w.n_jobs);
    GALE_LAUNCH_CHECK();
    // permuted, rotated fp16 activations
    GALE_CUDA_TRY(cudaMemsetAsync(w.x16, 0, size_t(P) * L.d_model * 2, st));
    {
        const int64_t warps = P * (L.d_model / 1024);
        gather_rotate_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, st>>>(x, w.perm, w.offsets + L.n_experts, K,
                                                                               L.d_model, P, w.x16);
        GALE_LAUNCH_CHECK();
    }
    const int64_t l1 = make_layout(L.d_ff, L.d_model).total;
    CUtensorMap xm;
    rc = act_map(&xm, w.x16, L.d_model, P);
    if (rc != GALE_OK) return rc;
    TcArgs a{};
    a.base = static_cast<const char*>(L.base);
    a.stride = L.expert_stride;
    a.jobs = static_cast<const TcJob*>(w.jobs);
    a.n_jobs = w.n_jobs;
    a.status = w.status;
    // w1 / w3 + SwiGLU
    a.off_a = 0;
    a.off_b = l1;
    a.rows = L.d_ff;
    a.cols = L.d_model;
    a.out = w.h;
    {
        const TcSmem S = tc_smem(2);
        rc = ensure_smem(reinterpret_cast<const void*>(tc_tile_kernel<2>), S.bytes);
        if (rc != GALE_OK) return rc;
        dim3 grid(w.max_jobs, (L.d_ff + kTcM - 1) / kTcM);
        tc_tile_kernel<2><<<grid, kTcThreads, S.bytes, st>>>(xm, a);
        GALE_LAUNCH_CHECK();
    }
    // rotate h
    rc = gale_fwht1024(w.h, GALE_F32, w.h16, GALE_F16, P, L.d_ff, st);
    if (rc != GALE_OK) return rc;
    CUtensorMap hm;
    rc = act_map(&hm, w.h16, L.d_ff, P);
    if (rc != GALE_OK) return rc;
    // w2
    a.off_a = 2 * l1;
    a.off_b = 2 * l1;
    a.rows = L.d_model;
    a.cols = L.d_ff;
    a.out = w.o;
    {
        const TcSmem S = tc_smem(1);
        rc = ensure_smem(reinterpret_cast<const void*>(tc_tile_kernel<1>), S.bytes);
        if (rc != GALE_OK) return rc;
        dim3 grid(w.max_jobs, (L.d_model + kTcM - 1) / kTcM);
        tc_tile_kernel<1><<<grid, kTcThreads, S.bytes, st>>>(hm, a);
        GALE_LAUNCH_CHECK();
    }
    return launch_moe_combine(w.o, w.pos_of_pair, gates, x, B, K, L.d_model, out, out_dtype, fuse_norm, eps,
                              w.scratch, st);
}

}  // namespace gale

/*
 * gale.h -- C ABI of libgale, the sm_100a (B200) implementation of the
 * decode-time GALE 1-bit routed-expert forward.
 *
 * The format (DeepSeek-V4-Flash -- GALE 1-bit experts, "What is in the pack",
 * routed-experts row; the same on the DeepSeek-V4-Pro-671B-GALE-1bit-v4 card,
 * weights table): every expert matrix W [rows x cols] is stored in the domain
 * rotated by a blocked FWHT-1024 along its input dimension (cols), as one sign
 * bit per weight, one fp16 scale per 128-weight block along the row, and 1 %
 * of the columns of every row as int4 outliers with a per-row fp16 scale.
 * The outlier value replaces the signed weight at its column.
 *
 * Conventions shared by every entry point
 *  - C linkage, no exceptions, no exit().  Every call returns an int status:
 *    GALE_OK (0) or a negative GALE_ERR_* code.
 *  - All memory is owned by the caller.  Pointers named "device" must point
 *    to CUDA device memory of the current device; nothing is allocated or
 *    freed by the library, which keeps only a per-device attribute cache.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream unless stated; launch
 *    failures return GALE_ERR_CUDA.  Errors found on the device (bad expert
 *    ids, unsorted outlier columns) are written to a caller-provided int32
 *    status word in device memory, which the caller reads after the stream
 *    has been synchronised.  The library never traps a kernel.
 *  - Dtype codes: GALE_F32, GALE_BF16, GALE_F16.  All multi-byte values are
 *    little-endian.
 */
#ifndef GALE_H
#define GALE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define GALE_OK               0
#define GALE_ERR_ARG         -1   /* invalid argument or device-detected invalid input */
#define GALE_ERR_ALIGN       -2   /* a pointer lacks the alignment the call needs */
#define GALE_ERR_WORKSPACE   -3   /* workspace missing or too small */
#define GALE_ERR_CUDA        -4   /* a CUDA runtime call or launch failed */
#define GALE_ERR_TIMEOUT     -5   /* a bounded device-side wait ran out */
#define GALE_ERR_UNSUPPORTED -6   /* shape or device not supported */
#define GALE_ERR_SELFTEST    -7   /* gale_selftest: a GPU result differs from the expected value */

/* element types */
#define GALE_F32  0
#define GALE_BF16 1
#define GALE_F16  2

/* gale_expert_gemv modes */
#define GALE_MODE_PLAIN  0        /* y = Q(W) x_rot */
#define GALE_MODE_SWIGLU 1        /* y = silu(Q(W) x_rot) * (Q(W3) x_rot) */

/* gale_moe_forward flags */
#define GALE_FLAG_RESIDUAL_RMSNORM 1  /* out = bf16(RMSNorm(x + y)), unit weight */

/* Human-readable name of a status code (static string, never NULL). */
const char* gale_status_string(int status);

/* ---------------------------------------------------------------------------
 * Packed-matrix layout.
 *
 * A packed matrix of `rows` x `cols` weights (cols a multiple of 1024, which
 * is also a multiple of the 128-weight scale block) holds five sections, each
 * starting on a 256-byte boundary (the manifest of the pack records "sections"
 * per matrix: DeepSeek-V4-Flash -- GALE 1-bit experts, "Files"):
 *   0 signs : rows*cols/8 bytes of uint32 words, row-major; column c of row r
 *             is bit (c % 32) of word r*(cols/32) + c/32; a set bit means -1.
 *   1 s_blk : fp16 [rows][cols/128], the scale of weights 128b..128b+127.
 *   2 s_row : fp16 [rows], the outlier scale of each row.
 *   3 idx   : uint16 [rows][k], outlier columns, strictly ascending per row.
 *   4 q     : int4 two's complement; value j of row r is nibble n = r*k + j,
 *             stored in byte n/2, low nibble first.
 * k = nearest integer to cols/100 (41 for 4096 columns, 20 for 2048): the
 * count that reproduces the card's 1.329 bits/weight and 46.0 GB.  Sign bits
 * under outlier columns are stored and ignored.  An expert record is
 * w1 || w3 || w2 (w1, w3: [d_ff x d_model], w2: [d_model x d_ff]), with no
 * padding between matrices.
 * ------------------------------------------------------------------------- */
typedef struct {
    int32_t rows;
    int32_t cols;
    int32_t k;            /* outliers per row */
    int32_t reserved;
    int64_t offset[5];    /* byte offset of each section from the record start */
    int64_t size[5];      /* byte size of each section (without padding) */
    int64_t total;        /* bytes of the whole matrix record (256-aligned) */
} gale_layout;

/* Fills *out for a rows x cols matrix.  Host only, no CUDA call.
 * Errors: GALE_ERR_ARG if out is NULL, rows < 1, cols < 1024,
 * cols % 1024 != 0 or cols > 65536 (idx is uint16). */
int gale_pack_layout(int rows, int cols, gale_layout* out);

/* Bytes of one expert record w1 || w3 || w2, or 0 on invalid sizes. */
int64_t gale_expert_bytes(int d_model, int d_ff);

/* Packs a matrix from canonical unpacked device arrays into `dst` (device,
 * gale_layout.total bytes, 16-byte aligned; padding bytes are zeroed):
 *   signs uint8 [rows][cols] (0 = +1, nonzero = -1), s_blk fp16 bits
 *   [rows][cols/128], s_row fp16 bits [rows], idx uint16 [rows][k],
 *   q int8 [rows][k] in [-8, 7].
 * `status` (device int32) is set to 0 by the call, then to GALE_ERR_ARG by
 * the kernel if any row's idx is not strictly ascending and < cols, or a q
 * value is out of range; the bytes of such rows are then unspecified. */
int gale_pack(const uint8_t* signs, const uint16_t* s_blk, const uint16_t* s_row,
              const uint16_t* idx, const int8_t* q, int rows, int cols,
              void* dst, int32_t* status, void* stream);

/* Dense dequantisation Q(W_rot) of a packed matrix (device) into
 * dense fp32 [rows][cols] (device): sign * s_blk, then outliers replaced by
 * q * s_row.  Every value is exact in fp32.  Reads idx without validation:
 * pass only records produced by gale_pack with status 0. */
int gale_unpack(const void* packed, int rows, int cols, float* dense, void* stream);

/* ---------------------------------------------------------------------------
 * Blocked FWHT-1024 (the rotation; DeepSeek-V4-Pro-671B-GALE-1bit-v4 card,
 * knobs paragraph, butterfly Walsh-Hadamard transform).
 * y[r, 1024b + i] = (1/32) * sum_j H[i, j] * x[r, 1024b + j], H the Sylvester
 * Hadamard matrix of order 1024 in natural order (H[i,j] = (-1)^popcount(i&j)).
 * x: device [rows][cols] of x_dtype; y: device [rows][cols] of y_dtype
 * (GALE_F32, GALE_BF16 or GALE_F16; the sums are taken in fp32 and rounded
 * to y_dtype once).  y may alias x when the dtypes are equal.
 * Errors: GALE_ERR_ARG for cols % 1024 != 0, rows < 0, bad dtypes;
 * GALE_ERR_ALIGN for pointers not 4-byte aligned.  rows == 0 is a no-op.
 * ------------------------------------------------------------------------- */
int gale_fwht1024(const void* x, int x_dtype, void* y, int y_dtype, int64_t rows, int cols,
                  void* stream);

/* ---------------------------------------------------------------------------
 * One packed matrix (or a SwiGLU w1/w3 pair) times rotated activations
 * (DeepSeek-V4-Pro-671B-GALE-1bit-v4 card, knobs paragraph: the direct GEMV
 * straight from the packed record, signs, block scales and int4 outliers
 * decoded in registers).
 * ------------------------------------------------------------------------- */
typedef struct {
    const void* packed;   /* device, 16-byte aligned record */
    int32_t rows;
    int32_t cols;
} gale_matrix;

/* x_rot: device fp32 [ntok][W.cols], already rotated (gale_fwht1024).
 * y: device fp32 [ntok][W.rows].
 * mode GALE_MODE_PLAIN : y = Q(W) x_rot (W3 must be NULL).
 * mode GALE_MODE_SWIGLU: y = silu(Q(W) x_rot) * (Q(W3) x_rot), W3 of the
 *                        same shape as W.
 * 1 <= ntok <= 64.  Accumulation is fp32.
 * Errors: GALE_ERR_ARG (shapes, mode, ntok), GALE_ERR_ALIGN. */
int gale_expert_gemv(const gale_matrix* W, const gale_matrix* W3, const float* x_rot,
                     int ntok, float* y, int mode, void* stream);

/* ---------------------------------------------------------------------------
 * Routing permute: groups the B*K (token, slot) pairs by expert, stable in
 * pair order (pair index p = t*K + k).
 *   ids    : device int32 [B][K], expert ids in [0, E), distinct within a token
 *   counts : device int32 [E]      pairs per expert
 *   offsets: device int32 [E + 1]  exclusive prefix sum of counts
 *   perm   : device int32 [B*K]    pair indices sorted by (expert, p)
 *   status : device int32, set to 0 by the call, GALE_ERR_ARG if an id is out
 *            of range or repeated within a token (such pairs are dropped).
 * 1 <= K <= 16, 1 <= E <= 1024, B >= 0.  Bit-exact and deterministic.
 * ------------------------------------------------------------------------- */
int gale_route_permute(const int32_t* ids, int B, int K, int E, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* status, void* stream);

/* The same permute spread over many CTAs, for large batches (the form above
 * runs in one CTA on one SM): identical arguments, results (bit for bit),
 * status and errors, plus
 *   scratch       : device, 4-byte aligned, at least
 *                   gale_route_permute_scratch_bytes(B, K, E) bytes; needs no
 *                   initialisation and holds nothing after the call
 *   scratch_bytes : its size; GALE_ERR_WORKSPACE if too small.
 * Three kernel launches: per-range expert counts (ranges of 256 pairs), a
 * scan in (expert, range) order, placement. */
size_t gale_route_permute_scratch_bytes(int B, int K, int E);   /* 0 on invalid sizes */
int gale_route_permute_grid(const int32_t* ids, int B, int K, int E, int32_t* counts,
                            int32_t* offsets, int32_t* perm, int32_t* status, void* scratch,
                            size_t scratch_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Router: the top-K experts of every token and their gates (the cards' "top-6
 * of 256 experts" per token; the gates are the softmax over the K selected
 * logits, as the benchmark configuration normalises them).
 *   logits : device fp32 [B][E]
 *   ids    : device int32 [B][K], experts by descending logit; on equal logits
 *            the lower expert index comes first; NaN logits rank as -inf
 *   gates  : device fp32 [B][K], exp(l_k - l_max) / sum over the K picks (fp32)
 * 1 <= K <= 16, K <= E <= 1024, B >= 0 (0 is a no-op).  One launch, one warp
 * per token; the outputs feed gale_moe_forward directly.
 * Errors: GALE_ERR_ARG (sizes, NULL pointers), GALE_ERR_ALIGN.
 * ------------------------------------------------------------------------- */
int gale_route_topk(const float* logits, int B, int E, int K, int32_t* ids, float* gates, void* stream);

/* ---------------------------------------------------------------------------
 * One routed-expert MoE layer.
 * ------------------------------------------------------------------------- */
typedef struct {
    const void* base;       /* device; expert e's record at base + e*expert_stride */
    int64_t expert_stride;  /* bytes, >= gale_expert_bytes(d_model, d_ff), multiple of 256 */
    int32_t n_experts;      /* E, 1..1024 */
    int32_t d_model;        /* hidden size, multiple of 1024 */
    int32_t d_ff;           /* expert intermediate size, multiple of 1024 */
    int32_t reserved;
} gale_layer;

/* Workspace bytes gale_moe_forward needs for B tokens and top-K routing. */
size_t gale_moe_workspace_size(const gale_layer* layer, int B, int K);

/* y[t] = sum_{k<K} gates[t,k] * expert_{ids[t,k]}(x[t]), where
 * expert_e(x) = Q(W2_e) H( silu(Q(W1_e) H x) * (Q(W3_e) H x) ) with H the
 * blocked FWHT-1024 (SwiGLU expert, top-K routed experts of the layer; the
 * card's "43 layers x 256 experts", "experts touched per token 258 (43 x 6)").
 * The K contributions are summed in fixed k order (deterministic, no atomics).
 *   x     : device bf16 bits [B][d_model]
 *   ids   : device int32 [B][K];   gates : device fp32 [B][K]
 *   out   : device [B][d_model] of out_dtype (GALE_F32 or GALE_BF16)
 *   flags : 0, or GALE_FLAG_RESIDUAL_RMSNORM: out = bf16(v / sqrt(mean(v^2) + eps))
 *           with v = x + y (post-norm residual step of an expert-only layer
 *           chain; out_dtype must be GALE_BF16).
 *   ws    : device workspace of at least gale_moe_workspace_size() bytes,
 *           256-byte aligned.  Its first int32 is the device status word:
 *           the call resets it to 0; kernels set GALE_ERR_ARG (bad ids) or
 *           GALE_ERR_TIMEOUT (a bounded wait ran out).  Read it after the
 *           stream is synchronised.  Calls sharing one workspace must not
 *           overlap on the device.
 * Tokens per expert choose the kernel: decode batches stream the packed
 * signs through the fused GEMV; prefill-sized groups use the tensor-core
 * tile path.  Both compute the same function.
 * Errors: GALE_ERR_ARG, GALE_ERR_ALIGN, GALE_ERR_WORKSPACE, GALE_ERR_CUDA. */
int gale_moe_forward(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                     const float* gates, int B, int K, void* out, int out_dtype, int flags,
                     float eps, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * gale_moe_forward without caller-provided workspace.  This is an interface
 * addition of this library and has no counterpart on the GALE cards.
 *
 * For callers that cannot allocate device memory where they run a layer:
 * for example a plugin inside a host runtime that owns the device memory pool,
 * or a process that fixed its device footprint at start-up.  The caller still
 * owns x, ids, gates, out and status; the scratch comes from one file-scope
 * device array of GALE_NOALLOC_SCRATCH_BYTES (4 MiB) inside the library,
 * which every GPU that loads the library holds until the process exits.
 *
 * Same computation, arguments and errors as gale_moe_forward, except:
 *  - no ws / ws_bytes; a call whose workspace (gale_moe_workspace_size)
 *    exceeds GALE_NOALLOC_SCRATCH_BYTES returns GALE_ERR_WORKSPACE;
 *  - status: optional device int32; when non-NULL the call ends by copying
 *    the device status word there (same codes as gale_moe_forward's);
 *  - the library allocates and frees nothing (no cudaMalloc, no cudaFree);
 *  - every call made outside stream capture looks the array's device
 *    address up again with the calling device current (so the address stays
 *    right after a cudaDeviceReset or any other re-creation of the primary
 *    context); a call made while its stream is being captured uses the
 *    address of the last uncaptured call on that device, so make at least
 *    one call on the device before capturing, and again after a reset;
 *  - all calls on a device share the one array and it keeps the previous
 *    call's contents (each call clears what must start at zero): calls that
 *    overlap on the GPU, from any stream or thread, race and give undefined
 *    results.  Serialise them.
 * ------------------------------------------------------------------------- */
#define GALE_NOALLOC_SCRATCH_BYTES (4u << 20)

int gale_moe_forward_noalloc(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                             const float* gates, int B, int K, void* out, int out_dtype, int flags,
                             float eps, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * gale_moe_forward with the inputs and the result in host memory.  An
 * interface addition of this library, with no counterpart on the GALE cards:
 * a decode step moves a few kilobytes but pays a fixed cost per transfer, so
 * the inputs cross in one copy and a small result is written in place.
 *
 * Same computation, flags and errors as gale_moe_forward, except:
 *  - x, ids, gates: host memory of any kind (the call copies them, with the
 *    CPU, into `staging`, then moves `staging` to the device in one copy);
 *  - staging: pinned host memory (cudaHostAlloc / cudaMallocHost), 16-byte
 *    aligned, at least gale_moe_host_staging_bytes(B, K, d_model) bytes,
 *    owned by the caller; it must not be written again until the stream has
 *    passed this call;
 *  - out: pinned host memory (or device memory) of out_dtype [B][d_model].
 *    A result of up to 1 MiB is written there by the layer's kernels; a
 *    larger one goes through the workspace and one device-to-host copy.  The
 *    result is complete once the stream has passed this call;
 *  - ws: device workspace of at least gale_moe_host_workspace_size() bytes
 *    (the status word is its first int32, as for gale_moe_forward).
 * Pageable staging or out returns GALE_ERR_ARG.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
size_t gale_moe_host_staging_bytes(int B, int K, int d_model);
size_t gale_moe_host_workspace_size(const gale_layer* layer, int B, int K);
int gale_moe_forward_host(const gale_layer* layer, const uint16_t* x, const int32_t* ids,
                          const float* gates, int B, int K, void* out, int out_dtype, int flags,
                          float eps, void* ws, size_t ws_bytes, void* staging, size_t staging_bytes,
                          void* stream);

/* ---------------------------------------------------------------------------
 * One expert's SwiGLU forward in one launch (the single-expert configuration
 * of the GALE cards' format table: w1/w3 [d_ff x d_model], w2 [d_model x
 * d_ff], fp32 activations):
 *   out[t] = W2 H( silu(W1 H x[t]) * (W3 H x[t]) )      (expert `expert` of layer)
 *   x   : device fp32 [B][d_model]        out : device fp32 [B][d_model]
 *   ws  : device, 256-byte aligned, gale_expert_forward_workspace_size()
 *         bytes; its first int32 is the status word
 * The batches of the streaming decode kernel (B <= 384, d_model <= 4096,
 * d_ff <= 2048), else GALE_ERR_UNSUPPORTED.  gale_expert_gemv is the
 * one-matrix call.  One launch, asynchronous on `stream`; the workspace and
 * out must not be in use by another call on another stream.
 * Errors: GALE_ERR_ARG (layer descriptor, expert outside [0, n_experts),
 * B < 1, NULL x or out), GALE_ERR_UNSUPPORTED (above), GALE_ERR_WORKSPACE,
 * GALE_ERR_ALIGN (ws not 256-byte, x or out not 4-byte aligned),
 * GALE_ERR_CUDA; on the device, GALE_ERR_TIMEOUT in the status word if a
 * bounded wait ran out.
 * ------------------------------------------------------------------------- */
size_t gale_expert_forward_workspace_size(const gale_layer* layer, int B);
int gale_expert_forward(const gale_layer* layer, int expert, const float* x, int B, float* out, void* ws,
                        size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * A stack of layers in one launch (decode): for l = 0 .. n_layers-1,
 *   x_{l+1} = bf16( RMSNorm( x_l + MoE_l(x_l) ) )   (unit weight, eps)
 * with MoE_l the layer of gale_moe_forward on ids[l], gates[l]; out = x_L.
 * The DeepSeek-V4-Pro-671B-GALE-1bit-v4 card's A100 paragraph names the
 * batch-1 floor: expert unpacks plus about 200 small kernel launches per
 * layer; here a whole stack is one persistent cooperative kernel.  Each layer
 * starts once every token's output of the previous one is written (a
 * counter per layer, bounded wait), and the weight ring streams on across
 * the layers.
 *   first        : layer 0; layer l's expert e is record l * (layer_stride /
 *                  first->expert_stride) + e of the records starting at
 *                  first->base (every layer the same shape and record size;
 *                  layer_stride a multiple of expert_stride, at least
 *                  n_experts * expert_stride)
 *   x0           : device bf16 [B][d_model]
 *   ids, gates   : device int32 / fp32 [n_layers][B][K] (as gale_moe_forward)
 *   out          : device bf16 [B][d_model], x_L
 *   ws           : device, 256-byte aligned, gale_moe_chain_workspace_size()
 *                  bytes; its first int32 is the status word (as for
 *                  gale_moe_forward)
 * 1 <= n_layers <= 4096; the batches of the streaming decode kernel
 * (B * K <= 384, d_model <= 4096, d_ff <= 2048), else GALE_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------- */
size_t gale_moe_chain_workspace_size(const gale_layer* first, int n_layers, int B, int K);
int gale_moe_chain(const gale_layer* first, int n_layers, int64_t layer_stride, const uint16_t* x0,
                   const int32_t* ids, const float* gates, int B, int K, uint16_t* out, float eps, void* ws,
                   size_t ws_bytes, void* stream);

/* Failure-path testing hook; an interface addition of this library with no
 * counterpart on the GALE cards.  Applies to later gale_moe_forward calls of
 * this process that take the streaming decode kernel (3 to 64 tokens):
 *   wait_limit_ns : bound of every device-side wait of the kernel, in ns
 *                   (0 restores the default of 2 s);
 *   withhold_cta  : a CTA index whose finished h tiles are never counted
 *                   (-1: none), so that the phase-2 waits of the CTAs that
 *                   need those tiles run out: the call then reports
 *                   GALE_ERR_TIMEOUT in its status word, every CTA drains its
 *                   copies and returns, and the output is unspecified.
 * Process-wide and not thread-safe; meant for tests of the failure path. */
int gale_debug_set_failure(uint64_t wait_limit_ns, int withhold_cta);

/* ---------------------------------------------------------------------------
 * Encoder: a dense fp32 matrix -> one packed record (the layout above), the
 * plain encoder of the DeepSeek-V4-Pro-671B-GALE-1bit-v4 card ("the v3 pack
 * rounded each weight to its sign"; the v4 error-feedback sign choice needs
 * real activations and is not this call).  Readings, in the pages' order:
 *   rotation : W_rot = W H, i.e. a blocked FWHT-1024 of every row, in fp64,
 *              butterfly stages h = 1, 2, ..., 512 (a + b lower, a - b upper),
 *              then times 1/32;
 *   signs    : bit 1 where W_rot < 0 (every column, outliers included);
 *   outliers : the k columns of largest |W_rot| (the lower column first on
 *              equal magnitudes), stored ascending; s_row = fp16(max|W_rot|/7)
 *              and q = clamp(rint(W_rot / s_row), -7, 7) in fp64 (0 if s_row
 *              is 0);
 *   s_blk    : fp16 of the mean |W_rot| over the block's columns that are not
 *              outliers (the least-squares scale of their signs), summed in
 *              column order in fp64; 0 for a block of outliers only.
 *   w   : device fp32 [rows][cols], 4-byte aligned
 *   dst : device, gale_layout.total bytes, 16-byte aligned (fully written;
 *         padding zero)
 * 1024 <= cols <= 16384, cols % 1024 == 0.  One launch (one CTA per row) after
 * a memset of dst.  Errors: GALE_ERR_ARG, GALE_ERR_ALIGN, GALE_ERR_UNSUPPORTED
 * (cols > 16384: the row is held in shared memory in fp64).
 * ------------------------------------------------------------------------- */
int gale_encode(const float* w, int rows, int cols, void* dst, void* stream);

/* ---------------------------------------------------------------------------
 * 4-bit non-expert weights (W4, g128).  The DeepSeek-V4-Pro-671B-GALE-1bit-v4
 * card (paragraph under the weights table) keeps attention and shared-expert
 * weights as symmetric int4 per 128-block with fp16 scales; the
 * DeepSeek-V4-Flash card ("What is in the pack", non-expert row) keeps them
 * 4-bit in VRAM.  Readings: codes q in [-7, 7]; per (row, 128-column block)
 * s = fp16(amax / 7) (fp32 division, round to nearest even) and
 * q = clamp(rint(w / s), -7, 7) in fp32 with ties to even (q = 0 when s = 0).
 * Layout of one [rows x cols] matrix (cols % 128 == 0):
 *   q at q_offset = 0 : [rows][cols/2] bytes, two's complement nibbles, the
 *                       low nibble holding the even column
 *   s at s_offset     : fp16 [rows][cols/128], 256-byte aligned
 *   total             : 256-byte aligned.
 * ------------------------------------------------------------------------- */
typedef struct {
    int64_t rows, cols;
    int64_t q_offset, q_bytes;
    int64_t s_offset, s_bytes;
    int64_t total;
} gale_w4_layout_t;

/* Host only.  Errors: GALE_ERR_ARG (NULL out, rows < 1, cols < 128 or not a
 * multiple of 128). */
int gale_w4_layout(int64_t rows, int64_t cols, gale_w4_layout_t* out);

/* Quantizes a dense fp32 matrix into the layout above (bit-exact with the
 * readings: the same fp32 decisions).
 *   w      : device fp32 [rows][cols], 16-byte aligned
 *   packed : device, gale_w4_layout(...).total bytes, 256-byte aligned; owned
 *            by the caller, fully written (padding bytes excepted)
 * One launch, one warp per (row, block).  Errors: GALE_ERR_ARG, GALE_ERR_ALIGN. */
int gale_w4_quantize(const float* w, int64_t rows, int64_t cols, void* packed, void* stream);

/* y = x W^T for 1..8 tokens (decode):
 *   y[t][r] = sum_c s[r][c/128] q[r][c] x[t][c]
 *   packed : device, the layout above, 256-byte aligned
 *   x      : device bf16 bits [B][cols]
 *   y      : device fp32 [B][rows] (overwritten)
 *   ws     : device, 256-byte aligned, gale_w4_workspace_size(rows, cols, B)
 *            bytes (256); its first int32 is a sticky status word: the caller
 *            sets it to 0 once, the call never clears it and writes
 *            GALE_ERR_TIMEOUT there if a bounded wait inside the kernel ran
 *            out (results are then undefined).
 * rows % 16 == 0, cols % 1024 == 0, 1 <= B <= 8, and the activation digits
 * 6 ceil(B/2) (cols + 16) bytes plus two ring stages within 227 KB of shared
 * memory (GALE_ERR_UNSUPPORTED beyond: cols <= 8192 at 7-8 tokens, 11264 at
 * 5-6, 16384 at 3-4, 34816 at 1-2).  Activations are held in fixed point per
 * 1024 columns (21 bits, three int8 digits, built inside the kernel) and
 * multiplied on the int8 tensor cores with exact int32 sums; scales and sums
 * in fp32.  One launch: a persistent CTA per SM streams its 16-row tiles by
 * bulk copies through a ring of shared-memory stages, reading every weight
 * byte once for all B tokens.
 * Errors: GALE_ERR_ARG (shape, NULL), GALE_ERR_ALIGN, GALE_ERR_WORKSPACE,
 * GALE_ERR_UNSUPPORTED (shared memory, above). */
size_t gale_w4_workspace_size(int64_t rows, int64_t cols, int B);   /* host only; 0 on invalid or
                                                                        unsupported sizes */
int gale_w4_gemv(const void* packed, int64_t rows, int64_t cols, const uint16_t* x, int B, float* y, void* ws,
                 size_t ws_bytes, void* stream);

/* Built-in parity self-check on tiny shapes (the card's "optional fast paths
 * verify themselves at startup" -- without any fallback).  Synchronous:
 * allocates nothing itself but needs `scratch` of gale_selftest_scratch_bytes()
 * device bytes.  Returns GALE_OK when the GPU results match the host-side
 * expectations built into the library, GALE_ERR_SELFTEST when one differs,
 * and the usual codes for launch or argument failures. */
size_t gale_selftest_scratch_bytes(void);
int gale_selftest(void* scratch, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GALE_H */

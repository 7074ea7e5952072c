/*
 * wq.h -- C ABI of the B200 (sm_100a) library for 4-bit per-group weight
 * quantization and the W4A16 decode linear.
 *
 * The problem, as the quantization pages state it:
 *   - a linear layer computes Y = X W^T with W: [out_features, in_features]
 *     = [N][K], and per-group quantization cuts each row of W into groups of
 *     G consecutive input channels ("大模型量化全景解析", section
 *     粒度和矩阵维度的关系);
 *   - weight-only quantization stores Q(W) plus scale/zero metadata and
 *     computes Y_hat = X dequant(Q(W))^T (same page, section
 *     公式补课：从一层 Linear 看量化到底改了什么); the 4-bit weights are
 *     dequantized inside the matmul kernel and multiplied with 16-bit
 *     activations ("3.6 量化(Quantization)", section 仅权重 vs 权重 + 激活);
 *   - the uniform quantizer is q = clamp(round(w/s) + z, qmin, qmax),
 *     w_hat = s (q - z); symmetric: z = 0, s = max|w| / 7, q in [-7, 7];
 *     asymmetric: s = (max - min) / 15, z = round(-min / s), q in [0, 15]
 *     ("3.6 量化(Quantization)", section 对称与非对称量化; "后训练量化（PTQ,
 *     Post-Training Quantization）", section 基础量化公式; "量化" compendium,
 *     section 量化方程);
 *   - the AWQ variant scales input channels before quantizing, W' = W diag(s),
 *     and undoes it on the activations, Y = X diag(s)^-1 quant(W')^T
 *     ("后训练量化（PTQ, Post-Training Quantization）", section AWQ, steps 3-5;
 *     "3.6 量化(Quantization)", section AWQ).
 *
 * Conventions shared by every call:
 *   - every pointer argument is a DEVICE pointer owned by the caller; the
 *     library allocates, frees and synchronizes nothing (except
 *     wq_last_device_status, which synchronizes the given stream);
 *   - every compute call only enqueues work on `stream` and returns at once;
 *   - arguments are validated synchronously, before anything is enqueued; a
 *     call that returns an error has enqueued nothing;
 *   - all matrices are dense and row-major; N, K are the output / input
 *     dimensions of the linear, M the number of activation rows;
 *   - pointers must be 16-byte aligned (WQ_ERR_MISALIGNED), except d_status
 *     (4-byte aligned);
 *   - group_size must be WQ_GROUP_SIZE and K a multiple of it
 *     (WQ_ERR_UNSUPPORTED_SHAPE); N and K are at most WQ_MAX_DIM;
 *   - the functions are thread-safe; the only state the library keeps is one
 *     device error word per GPU, read by wq_last_device_status.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream type (identical to cudaStream_t / CUstream); NULL is the
 * legacy default stream. */
typedef struct CUstream_st* wq_stream_t;

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,        /* NULL where a buffer is required, bad flag, buffer too small */
    WQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 128 != 0, group_size != 128, M out of range, dims too large */
    WQ_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
    WQ_ERR_WORKSPACE_TOO_SMALL = 4,
    WQ_ERR_NONFINITE = 5,          /* reported through d_status only (see wq_quantize_rtn) */
    WQ_ERR_TIMEOUT = 6,            /* a bounded wait inside a kernel gave up */
    WQ_ERR_CUDA = 7                /* the CUDA runtime reported an error (launch or stream) */
} wq_status;

#define WQ_GROUP_SIZE 128
#define WQ_MAX_DIM (1 << 20)
#define WQ_LAYOUT_TILED 1

/* Human-readable name of a status code; never NULL. */
const char* wq_status_string(int status);

/* ABI version of this header (bumped on any incompatible change). */
int wq_abi_version(void);
#define WQ_ABI_VERSION 1

/*
 * wq_quantize_rtn -- per-group round-to-nearest 4-bit quantization plus
 * canonical packing ("3.6 量化(Quantization)", sections 对称与非对称量化 and
 * 粒度; "后训练量化（PTQ, Post-Training Quantization）", section 基础量化公式).
 *
 *   W          bf16 [N][K]: the weight, row n = output channel.
 *   awq_scale  fp32 [K] or NULL: AWQ per-input-channel scale s; when given,
 *              w' = fp32(W[n][k]) * s[k] (one rounded fp32 product) is
 *              quantized instead of W.
 *   group_size must be 128; groups are 128 consecutive k of one row.
 *   symmetric  1: z = 0, s = max|w|/7, q = clamp(rne(w/s16), -7, 7), stored
 *              as q + 8 (1..15);  0: s = (max-min)/15, z = rne(-min/s16),
 *              q = clamp(rne(w/s16) + z, 0, 15), stored as q.
 *   qweight    uint32 [N][K/8] out: element k = 8j + i of row n is nibble i
 *              (bits [4i, 4i+4)) of qweight[n][j].
 *   scales     fp16 [N][K/128] out: s16 = fp16_rne(max(range, 1e-8) / qden),
 *              range and division in fp32; an s16 that rounds to 0 becomes
 *              2^-24.  The codes are computed with this stored s16.
 *   zeros      fp16 [N][K/128] out when symmetric == 0 (must be NULL when
 *              symmetric == 1): z16 = fp16(rne(-min / s16)), an integer
 *              (stored as +0 when zero); the codes use this stored z16.
 *   d_status   int32 on device, or NULL: set to the number of non-finite
 *              groups (a NaN/Inf input after the AWQ product, or an fp16
 *              scale or zero that overflows).  Such a group is written as
 *              nibbles 0 with scale (and zero) 0x7E00 (fp16 NaN), so a linear
 *              that reads it yields NaN.  0 means every group is finite.
 *   Rounding is round-half-to-even throughout; divisions are IEEE fp32.
 *   Returns WQ_OK once enqueued.
 */
wq_status wq_quantize_rtn(const void* W, const float* awq_scale, int N, int K, int group_size,
                          int symmetric, uint32_t* qweight, void* scales, void* zeros,
                          int* d_status, wq_stream_t stream);

/*
 * wq_packed_bytes -- size in bytes of the kernel layout `layout` for an
 * N x K weight; 0 if the arguments are invalid.
 *
 * Layout WQ_LAYOUT_TILED: the weight is cut into tiles of 128 rows x one
 * K-slab of 4 groups (512 inputs; the last slab may hold fewer groups).
 * Tiles are stored slab by slab and, within a slab, row-tile by row-tile;
 * every full tile has the same size, so tile (s, b) starts at
 * s * NB * full_tile + b * tile_bytes(s) with NB = ceil(N/128).  A tile holds
 * first the codes (row r: its qweight words for the slab's gs groups, gs*64
 * bytes at offset r*gs*64), then the metadata (entry (r, g) at offset
 * 128*gs*64 + (r*gs + g) * mb): mb = 2, the fp16 scale, when symmetric;
 * mb = 4, the fp16 scale in the low and the fp16 zero in the high half of a
 * little-endian uint32, when asymmetric.  Each code word is the canonical
 * word with its nibbles interleaved: nibble slot t holds canonical nibble 2t
 * (t < 4) or 2(t-4)+1 (t >= 4), so one mask 0x000F000F after a shift by 4t
 * isolates the adjacent inputs 2t and 2t+1.  Rows past N are zero.
 */
size_t wq_packed_bytes(int N, int K, int group_size, int symmetric, int layout);

/*
 * wq_pack_layout -- permute the canonical (qweight, scales, zeros) produced
 * by wq_quantize_rtn into kernel layout `layout` (see wq_packed_bytes).  The
 * same bytes, moved; nothing is recomputed.  packed_bytes is the size of
 * `packed` and must be >= wq_packed_bytes(...) (else WQ_ERR_INVALID_ARG).
 * `zeros` must be NULL iff symmetric.
 */
wq_status wq_pack_layout(const uint32_t* qweight, const void* scales, const void* zeros, int N,
                         int K, int group_size, int symmetric, int layout, void* packed,
                         size_t packed_bytes, wq_stream_t stream);

/*
 * wq_workspace_bytes -- workspace needed by wq_gemv_w4a16 for M = 1..8
 * (0 when that call needs none), and by wq_gemm_w4a16 for M = 9 ..
 * WQ_GEMM_MAX_M (the only entry point for those M); 0 for other M or invalid
 * sizes.
 * wq_gemm_workspace_bytes -- workspace needed by wq_gemm_w4a16,
 * M = 1..WQ_GEMM_MAX_M.
 * A workspace holds completion counters and split-K partial sums; the GEMM's
 * also holds the per-group sums of x, so every GEMM call needs one, and for
 * the shapes of the GEMV's tensor-core kernel (M = 2..8, K a multiple of 512)
 * it also holds the activation operand prepared once per 512-input slab, so
 * every such GEMV call needs one too.  The first WQ_WORKSPACE_COUNTER_BYTES bytes hold
 * the counters: they must be zero before the first call that uses a
 * workspace (allocate it zero-filled), and every call that completes leaves
 * them zero again, so one workspace serves any number of later calls of any
 * size.  Calls that share a workspace must not run concurrently.
 */
#define WQ_WORKSPACE_COUNTER_BYTES 262144
size_t wq_workspace_bytes(int M, int N, int K);
size_t wq_gemm_workspace_bytes(int M, int N, int K);

/*
 * wq_gemv_w4a16 -- the W4A16 decode linear for M = 1..8 activation rows
 * (dequantization in registers, fp32 accumulation):
 *
 *   y[m][n] = sum_g s16[n][g] * sum_{k in g} x'[m][k] * (q[n][k] - z[n][g])
 *
 * where x' is the activation as the kernel multiplies it.  Let
 * u[m][k] = x[m][k] (bf16, exact in fp32), or, when inv_act_scale is given,
 * u[m][k] = fp32(x[m][k]) * inv_act_scale[k] (the AWQ fold, inv_act_scale =
 * 1/s, one rounded fp32 product).
 *   - The integer paths: M = 2..8 with K a multiple of 512 (int8 tensor
 *     cores, tcgen05.mma kind::i8), and M <= 4 otherwise (CUDA cores,
 *     dp4a), both with or without inv_act_scale.  Each
 *     64-input chunk of a row of u is rounded to 16-bit fixed point,
 *     x' = rn(u * 2^e) * 2^-e with e chosen so that the chunk's largest |u|
 *     lies in [2^14, 2^15) (a bf16 value there, and any value with at most
 *     15 - (its exponent gap to the largest) significant bits, stays exact;
 *     every other is within 2^-15 of the chunk's largest |u|).  The codes
 *     times these integers are summed exactly in int32, so the error in y is
 *     at most 2^-15 * sum_k |w_hat[n][k]| * max|u| over k's chunk.  A chunk
 *     holding a NaN or an infinity makes every output of its row NaN.  Both
 *     integer kernels give the same per-chunk integers and differ only in
 *     the order of the fp32 additions of the chunks' contributions.
 *   - otherwise (M = 5..8 with K not a multiple of 512) x' = u, multiplied
 *     in fp32 on the CUDA cores.
 *   x        bf16 [M][K];      inv_act_scale fp32 [K] or NULL;
 *   packed   the weight in kernel layout `layout` (from wq_pack_layout);
 *   y        fp32 [M][N] out;
 *   workspace, ws_bytes: see wq_workspace_bytes (WQ_ERR_WORKSPACE_TOO_SMALL
 *            if smaller; may be NULL when wq_workspace_bytes returns 0).
 * The result does not depend on the GPU's scheduling: partial sums are
 * combined in a fixed order.
 */
wq_status wq_gemv_w4a16(const void* x, const float* inv_act_scale, const void* packed, int M,
                        int N, int K, int group_size, int symmetric, int layout, float* y,
                        void* workspace, size_t ws_bytes, wq_stream_t stream);

/*
 * wq_gemm_w4a16 -- the same linear for M = 1..WQ_GEMM_MAX_M activation rows
 * on the tensor cores (tcgen05).  Three kernels:
 *   - M <= 16 with K a multiple of 512 (decode batches): the int8 kernel of
 *     wq_gemv_w4a16's integer path (codes times the 16-bit fixed-point
 *     activations of each 64-input chunk, exact int32 sums, same rounding
 *     and error bound as described there);
 *   - otherwise M <= 64: per group, the weights are dequantized into tensor
 *     memory as bf16 tiles holding the exact integers 128 + q, multiplied
 *     with x (zero-padded to 16, 32, 48 or 64 rows) with fp32 accumulation,
 *     and the group's exact contribution s16 * (D - (128 + z) * sum_k x[m][k])
 *     is added in fp32;
 *   - M > 64 (prefill, "大模型量化全景解析", section 八: compute-bound): the
 *     same bf16 arithmetic in tiles of 128 weight rows x 128 activation rows,
 *     the dequantized weights in shared memory, the running sums in tensor
 *     memory.
 * Arguments as wq_gemv_w4a16; inv_act_scale must be NULL
 * (WQ_ERR_INVALID_ARG otherwise: the bf16 tensor-core operand cannot hold
 * x * inv_act_scale exactly).
 */
#define WQ_GEMM_MAX_M 65536
wq_status wq_gemm_w4a16(const void* x, const float* inv_act_scale, const void* packed, int M,
                        int N, int K, int group_size, int symmetric, int layout, float* y,
                        void* workspace, size_t ws_bytes, wq_stream_t stream);

/*
 * wq_gptq_quantize -- GPTQ: per-group 4-bit quantization in which the input
 * columns are quantized one at a time in natural order and each column's
 * rounding error is fed back into the columns not yet quantized, weighted by
 * the inverse Hessian of the layer's calibration inputs, to minimize
 * ||X W^T - X W_hat^T||^2 ("3.6 量化(Quantization)", section GPTQ: objective,
 * H = 2 X X^T over the calibration inputs, update
 * W[:, F] -= e_j / [H^-1]_jj [H^-1]_{j,F}; "推理优化中“用精度换性能“的核心技术：量化",
 * section 四.2: columns in natural order with per-column error feedback;
 * "大模型量化全景解析", section 六.2: damping of the Hessian).
 *
 *   W          bf16 [N][K]: the weight, row n = output channel.
 *   X          bf16 [T][K]: T calibration input rows of the layer.
 *   damp       H = 2 X^T X + damp * mean(diag(2 X^T X)) * I (0.01 is the
 *              usual choice); must be >= 0.
 *   qweight, scales, zeros: out, exactly the format of wq_quantize_rtn
 *              (so wq_pack_layout and both linears take it unchanged); zeros
 *              must be NULL iff symmetric.
 *   workspace  device scratch of wq_gptq_workspace_bytes(T, N, K) bytes,
 *              256-byte aligned, owned by the caller (its contents on entry
 *              do not matter): about 8 (K^2 + T K + N K) bytes.
 *   d_status   int32 on device, or NULL: 0 when all went well; bit 0: a
 *              group met a non-finite weight (written as nibbles 0 with
 *              scale and zero 0x7E00, like wq_quantize_rtn); bit 1: the
 *              damped Hessian was not positive definite (a Cholesky pivot
 *              <= 0; the codes are then not meaningful).
 * Arithmetic: fp64 throughout, except that a group's scale and zero come
 * from the RTN rules (fp32 range, IEEE fp32 divisions, fp16 RNE) applied to
 * its 128 current weights rounded to fp32 when its first column is
 * quantized; codes q = clamp(rint(w / s16) + z16) on the fp64 current
 * weights.  The restricted inverses are taken from one Cholesky
 * factorization of H with its index order reversed (H = R R^T, R upper); in
 * exact arithmetic this is the same update.
 * Limits: K <= WQ_GPTQ_MAX_K, 1 <= T <= WQ_GPTQ_MAX_T
 * (WQ_ERR_UNSUPPORTED_SHAPE).  Enqueues about 4 K / 64 kernels on `stream`.
 */
#define WQ_GPTQ_MAX_K 32768
#define WQ_GPTQ_MAX_T 65536
size_t wq_gptq_workspace_bytes(int T, int N, int K);
wq_status wq_gptq_quantize(const void* W, const void* X, int T, int N, int K, int group_size,
                           int symmetric, double damp, uint32_t* qweight, void* scales,
                           void* zeros, void* workspace, size_t ws_bytes, int* d_status,
                           wq_stream_t stream);

/*
 * wq_awq_search -- the AWQ scale search: for alpha = i / n_grid, i = 0..n_grid,
 * scale the input channels by s = s_X^alpha, quantize W diag(s) with per-group
 * RTN (exactly wq_quantize_rtn with awq_scale = s) and measure the layer's
 * output error on the calibration inputs X with the activations divided by
 * s; pick the alpha with the smallest error ("3.6 量化(Quantization)",
 * section AWQ: s = s_X^alpha with s_X the mean activation magnitude per input
 * channel, alpha searched over [0, 1] per layer on calibration data,
 * y = sum_j quant(s_j w_j) x_j / s_j; "后训练量化（PTQ, Post-Training
 * Quantization）", section AWQ).
 *
 *   W          bf16 [N][K] weight;  X  bf16 [T][K] calibration inputs.
 *   s_X,j      max(mean_t |X[t][j]|, 1e-8) in fp64.
 *   s          s_X^alpha divided by its geometric mean (so prod_j s_j = 1),
 *              computed in fp64 and rounded to fp32 (the quantizer's input).
 *   losses     fp64 [n_grid + 1] out (device, 16-byte aligned):
 *              ||X W^T - (X diag(s)^-1) dequant(Q(W diag(s)))^T||_F^2 in fp64
 *              for every alpha, summed in a fixed order.
 *   best       int32 out (device): the first index of the smallest loss.
 *   scale_out  fp32 [K] out (device): s of the chosen alpha, ready for
 *              wq_quantize_rtn(awq_scale = scale_out) and, as 1/s, for the
 *              linears' inv_act_scale.
 *   workspace  device scratch of wq_awq_search_workspace_bytes(T, N, K, n_grid)
 *              bytes, 256-byte aligned, owned by the caller: about
 *              8 (N K + T K + T N) + N K / 2 bytes.
 * Limits: 1 <= T <= WQ_AWQ_MAX_T (WQ_ERR_UNSUPPORTED_SHAPE),
 * 1 <= n_grid <= WQ_AWQ_MAX_GRID (WQ_ERR_INVALID_ARG).  Non-finite weights or
 * scales give NaN losses.  Enqueues about 6 (n_grid + 1) kernels on `stream`.
 */
#define WQ_AWQ_MAX_T 65536
#define WQ_AWQ_MAX_GRID 1000
size_t wq_awq_search_workspace_bytes(int T, int N, int K, int n_grid);
wq_status wq_awq_search(const void* W, const void* X, int T, int N, int K, int group_size,
                        int symmetric, int n_grid, double* losses, float* scale_out, int* best,
                        void* workspace, size_t ws_bytes, wq_stream_t stream);

/*
 * NVFP4: block-scaled 4-bit floating point, E2M1 elements in blocks of 16
 * consecutive inputs with one E4M3 scale per block and one fp32 scale per
 * tensor ("3.6 量化(Quantization)", section 数值格式: E2M1 magnitudes 0, 0.5,
 * 1, 1.5, 2, 3, 4, 6; E4M3 with largest value 448; 16 E2M1 elements share one
 * E4M3 scale plus one fp32 scale per tensor; section 实例演算: 4.5 bits per
 * element).
 *
 * wq_nvfp4_quantize -- A bf16 [R][C] (C a multiple of 128) ->
 *   codes         uint8 [R][C/2]: two E2M1 codes per byte, element 2i in the
 *                 low nibble (bit 3 of a code is the sign);
 *   block_scales  uint8 [R][C/16]: E4M3 codes;
 *   tensor_scale  fp32 [1] (device): S = max(amax(A), 1e-8) / (6 * 448).
 * Each step is one correctly rounded fp32 operation: sb = E4M3(amax_block /
 * fl(6 S)) (round to nearest even, saturating at 448; a scale that rounds to
 * 0 becomes the smallest subnormal 2^-9); q = E2M1(a / fl(E4M3(sb) S))
 * (nearest magnitude, ties to the even code, saturating at 6, sign kept);
 * a_hat = E2M1(q) E4M3(sb) S.  d_status (int32 on device, or NULL): the number
 * of non-finite inputs (they are left out of amax; their codes are undefined).
 *
 * wq_nvfp4_packed_bytes / wq_nvfp4_pack_layout -- the weight layout the
 * linear reads: the codes unchanged (N*K/2 bytes), then the block scales in
 * the tensor cores' scale layout: for each tile of 128 rows t and each 64
 * inputs kb, a 512-byte block at ((t * K/64) + kb) * 512 holding the 4 scales
 * of row 128 t + 32 m1 + m0 at bytes m0 * 16 + m1 * 4 + (0..3) (rows past N
 * are 0).
 *
 * wq_nvfp4_linear -- y fp32 [M][N] = dequant(x_q) dequant(W)^T, both operands
 * NVFP4 (the FP4 tensor-core form): x bf16 [M][K] is quantized like the
 * weights (its own tensor scale), then the block-scaled FP4 tensor cores
 * (tcgen05.mma kind::mxf4nvf4, block scales in tensor memory) accumulate in
 * fp32, and the tensor scales are applied once per output.
 *   packed          the weight from wq_nvfp4_pack_layout;
 *   w_tensor_scale  fp32 [1] on device: the weight's S from wq_nvfp4_quantize;
 *   workspace       wq_nvfp4_linear_workspace_bytes(M, N, K) bytes, 256-byte
 *                   aligned (the quantized activations and split-K partials).
 * M = 1..WQ_NVFP4_MAX_M.
 */
#define WQ_NVFP4_MAX_M 128
wq_status wq_nvfp4_quantize(const void* A, int R, int C, uint8_t* codes, uint8_t* block_scales,
                            float* tensor_scale, int* d_status, wq_stream_t stream);
size_t wq_nvfp4_packed_bytes(int N, int K);
wq_status wq_nvfp4_pack_layout(const uint8_t* codes, const uint8_t* block_scales, int N, int K,
                               void* packed, size_t packed_bytes, wq_stream_t stream);
size_t wq_nvfp4_linear_workspace_bytes(int M, int N, int K);
wq_status wq_nvfp4_linear(const void* x, const void* packed, const float* w_tensor_scale, int M,
                          int N, int K, float* y, void* workspace, size_t ws_bytes,
                          wq_stream_t stream);

/*
 * wq_last_device_status -- synchronize `stream`, then report and clear the
 * device error word of the current GPU: WQ_ERR_TIMEOUT if a kernel's bounded
 * wait gave up since the last call (its outputs are then undefined),
 * WQ_ERR_CUDA if the stream reports a CUDA error, else WQ_OK.  The error word
 * is shared by all streams of the GPU.
 */
wq_status wq_last_device_status(wq_stream_t stream);

/*
 * wq_gemv_w4a16_static -- wq_gemv_w4a16 without a workspace argument, for
 * callers that cannot allocate device memory (a custom-op hook or plugin whose
 * host forbids or owns all device allocations, or a captured region with a
 * fixed memory pool).  The quantization pages have no counterpart: this is a
 * deployment convenience of this library.
 *
 * Same arguments, semantics and result as wq_gemv_w4a16, minus workspace and
 * ws_bytes.  The split-K scratch lives in one static device array of
 * WQ_STATIC_SCRATCH_BYTES inside the library (held by every GPU that loads the
 * library until the process exits); shapes with wq_workspace_bytes(M, N, K)
 * above that are refused with WQ_ERR_WORKSPACE_TOO_SMALL.  Nothing is
 * allocated or freed: each call clears the counters it uses with an
 * asynchronous memset on `stream` and launches the GEMV kernel.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls share the one array: calls that may overlap on the GPU (on
 *     different streams, or from different threads without ordering) race
 *     and may return wrong results.  Order them on one stream.
 */
#define WQ_STATIC_SCRATCH_BYTES (8u << 20)
wq_status wq_gemv_w4a16_static(const void* x, const float* inv_act_scale, const void* packed,
                               int M, int N, int K, int group_size, int symmetric, int layout,
                               float* y, wq_stream_t stream);

/*
 * wq_debug_set_wait_limit_ns -- test hook, not part of the stable ABI: the
 * time a kernel's bounded wait (on its shared-memory pipeline barriers) gives
 * before it records WQ_ERR_TIMEOUT and returns; default 2 s, 0 is treated as
 * 1 ns.  A tiny limit makes any wait that is not already satisfied give up at
 * once, which exercises the timeout path without stalling the GPU.  Affects
 * calls enqueued afterwards, from any thread.
 */
void wq_debug_set_wait_limit_ns(unsigned long long ns);

/*
 * wq_debug_gemm_force_fold -- test hook, not part of the stable ABI: 1 makes
 * wq_gemm_w4a16 use its many-row kernel (M > 64) for every M, so both kernels
 * can be checked and timed on the same shapes; 0 restores the choice by M.
 * Affects calls enqueued afterwards, from any thread.
 */
void wq_debug_gemm_force_fold(int on);

/*
 * wq_debug_gemv_force_cuda_cores -- test hook, not part of the stable ABI: 1
 * makes wq_gemv_w4a16 (and wq_gemv_w4a16_static) use the CUDA-core kernel for
 * every shape, and wq_gemm_w4a16 its bf16 tensor-core kernels, so they and
 * the int8 tensor-core decode kernel can be checked and timed on the same
 * shapes; 0 restores the default choice.  Affects calls enqueued afterwards,
 * from any thread.
 */
void wq_debug_gemv_force_cuda_cores(int on);

/*
 * wq_debug_gemv_split -- test hook, not part of the stable ABI: how
 * wq_gemv_w4a16 would split an M x N x K linear (awq != 0: with the
 * activation factor) over a GPU with num_sms SMs holding ctas_per_sm of its
 * CTAs each.  Writes the number of 128 x 512 tiles, the teams per CTA and the
 * CTAs of the grid; team t of the grid's teams T owns tiles
 * [t * tiles / T, (t + 1) * tiles / T).  For the shapes of the tensor-core
 * decode kernel (M = 2..8, K a multiple of 512, not forced onto the CUDA
 * cores) that is one team per CTA and min(tiles, num_sms) CTAs.  Host arithmetic only (no device
 * call, usable without a GPU).  WQ_ERR_INVALID_ARG for M outside 1..8, N < 1,
 * K not a positive multiple of 128, num_sms or ctas_per_sm < 1, or a null
 * output pointer.
 */
wq_status wq_debug_gemv_split(int M, int N, int K, int awq, int num_sms, int ctas_per_sm,
                              long long* tiles, int* teams, long long* grid);

/*
 * wq_stream_read_probe -- measurement helper with no counterpart on the
 * quantization pages: read `bytes` bytes of device memory at `buf` once, with
 * 16-byte streaming loads from every SM, and write their 32-bit XOR checksum
 * to *out (device pointer, 4-byte aligned; the call zeroes it first).  Timing
 * it gives the read-only HBM rate of this GPU, the ceiling for the
 * weight-streaming linears above (which read their weights once and write
 * almost nothing).  buf 16-byte aligned, bytes a positive multiple of 16
 * (WQ_ERR_INVALID_ARG / WQ_ERR_MISALIGNED otherwise).  Asynchronous on
 * `stream`.
 */
wq_status wq_stream_read_probe(const void* buf, size_t bytes, uint32_t* out, wq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */

/*
 * w4.h -- C ABI of the B200 (sm_100a) group-wise 4-bit weight-only library.
 *
 * The packed weight format is the LoopQ storage contract (page "loopq/packed_weight.py",
 * class PackedLoopQWeight and its validate / _dequantize_validated / pack_weight):
 *
 *   W is [N, K]: N rows (output features), K columns (input features, "width").
 *   codes  uint8  [N, ceil(K/2)], row-major, contiguous. Byte j of a row holds column 2j in
 *          its LOW nibble and column 2j+1 in its HIGH nibble ("even_column_low"). For an odd K
 *          the unused high nibble of the last byte is zero.
 *   values signed two's-complement nibbles: a nibble v >= 8 stands for v - 16.
 *          Format v1 forbids the nibble 8 (the narrow range [-7, 7]); v2 allows it (-8).
 *   scales float32 [N, ceil(K/32)], row-major, finite and > 0: column k of row n is
 *          dequantized as fp32(value * scales[n][k/32]); the last group covers only the
 *          columns that exist.
 *
 * The asymmetric sub-channel variant (page "keras/src/layers/core/dense.py", int4 diff:
 * _int4_build's kernel_scale / kernel_zero / g_idx and _int4_call's dequantize-with-zero)
 * uses UNSIGNED nibbles u in [0, 15], a per-(row, group) zero point z (int8 holding [0, 15])
 * and a column-to-group map g_idx: w[n][k] = fp32((u - z[n][g]) * s[n][g]) with g = g_idx[k].
 * Scales and zeros are stored [N, n_groups] (rows = output features, as the packed codes).
 *
 * Conventions for every entry point:
 *   - Every array pointer is DEVICE memory owned by the caller. The library keeps no pointer
 *     after a call returns and allocates no device memory; scratch memory, where a call needs
 *     it, comes in through (workspace, workspace_bytes).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Calls that must read a result back (validation) synchronize that stream and
 *     say so.
 *   - Host-side checks (NULL pointers, sizes, dtype codes, alignment of the workspace) are
 *     done before anything is enqueued and returned synchronously; nothing is enqueued on
 *     an error.
 *   - The hot calls (w4_dequantize, w4_linear, w4_linear_asym_gidx) do NOT check the content
 *     of the codes and scales: the owner validates once before use (LoopQ's
 *     _dequantize_validated fast path). w4_validate / w4_validate_asym do that check.
 *   - Sizes are int64_t; N, K, M >= 1. K <= 2^24, N and M <= 2^31 - 1.
 *   - A CUDA launch error is returned as W4_ERR_CUDA; w4_last_cuda_error() gives its code.
 */
#ifndef W4_H_
#define W4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (no CUDA header is needed to include this file). */
typedef struct CUstream_st *w4_stream_t;

typedef enum {
  W4_OK = 0,
  W4_ERR_NULL = 1,          /* a required pointer is NULL                                  */
  W4_ERR_SHAPE = 2,         /* a size is <= 0 or above its limit, or sizes do not agree    */
  W4_ERR_DTYPE = 3,         /* unknown w4_dtype, or one the call does not offer            */
  W4_ERR_NONFINITE = 4,     /* W holds NaN or +-Inf (pack_weight: "weight must be finite") */
  W4_ERR_SCALE = 5,         /* a scale is not finite or not > 0 (validate)                 */
  W4_ERR_HIGH_NIBBLE = 6,   /* odd K and a nonzero unused high nibble (validate)           */
  W4_ERR_RESERVED_CODE = 7, /* format v1 and a nibble equal to 8 (validate)                */
  W4_ERR_VERSION = 8,       /* format_version not in {1, 2} (validate)                     */
  W4_ERR_GIDX = 9,          /* a g_idx entry outside [0, n_groups), or a bad perm          */
  W4_ERR_ZERO = 10,         /* a zero point outside [0, 15]                                */
  W4_ERR_UNSUPPORTED = 11,  /* a valid request this build does not serve                   */
  W4_ERR_WORKSPACE = 12,    /* workspace too small or not 256-byte aligned                 */
  W4_ERR_TIMEOUT = 13,      /* a bounded device-side wait expired (see w4_device_error)    */
  W4_ERR_CUDA = 14          /* a CUDA runtime/driver call failed (see w4_last_cuda_error)  */
} w4_status;

typedef enum { W4_BF16 = 0, W4_F16 = 1, W4_F32 = 2, W4_F64 = 3 } w4_dtype;

/*
 * w4_quantize_rtn -- round-to-nearest symmetric group-32 quantization and packing.
 * Page "loopq/packed_weight.py", pack_weight (checks and packing order); the rounding is
 * round-half-to-even and the clip follows page "gemma/peft/_quantization_utils.py",
 * uniform_quantize; the range is the narrow [-7, 7] that format v1 requires (validate).
 * For each row n and group g (columns 32g .. min(32g+32, K)-1):
 *     amax = max |W|;  s = max(fl32(amax / 7), 2^-126);  q = clamp(rne(fl32(W / s)), -7, 7)
 *     scales[n][g] = s; codes packed as in the format above (odd K: high pad nibble = 0).
 *   W        float32 [N, K] row-major, read only.
 *   codes    out, uint8 [N, ceil(K/2)];  scales  out, float32 [N, ceil(K/32)].
 *   d_status optional device int32: set to W4_ERR_NONFINITE if W holds NaN/Inf, left
 *            unchanged otherwise (the caller zeroes it). If NULL, the call synchronizes
 *            `stream` and returns W4_ERR_NONFINITE itself, using one status word inside the
 *            library that every NULL-d_status call (this one, w4_quantize_rtn_channel,
 *            w4_lora_merge) shares: such calls must not overlap on the GPU (from several
 *            host threads or streams at once) -- pass d_status when they may. Outputs are
 *            unspecified for a non-finite W. The results are bit-identical to the
 *            definition above (IEEE divide, no flush-to-zero).
 */
w4_status w4_quantize_rtn(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                          int32_t *d_status, w4_stream_t stream);

/*
 * w4_dequantize -- dense weight from the packed format.
 * Page "loopq/packed_weight.py", _dequantize_validated: values * repeat_interleave(scales,
 * 32)[:, :K] in fp32, then .to(output dtype): round-to-nearest-even to bf16/f16, exact
 * widening to f64. Bit-identical to that definition.
 *   format_version 1 or 2 (only checked for range here; content is not validated).
 *   out  [N, K] row-major of `out_dtype` (W4_BF16, W4_F16, W4_F32 or W4_F64).
 */
w4_status w4_dequantize(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                        int format_version, w4_dtype out_dtype, void *out, w4_stream_t stream);

/*
 * w4_linear -- y = x . dequant(W)^T + bias, the dequantize-fused weight-only linear.
 * Page "paddlenlp/quantization/quantization_linear.py", quant_weight_forward
 * (weight_only_linear(x, weight, bias, weight_scale, weight_dtype, group_size)); page
 * "keras/src/layers/core/dense.py", _int4_call (dequantize, matmul, add bias).
 *   x     bf16 [M, K] row-major (activations are not quantized: weight-only, A16).
 *   bias  optional fp32 [N] (NULL = none), added in fp32 before the final rounding.
 *   y     out [M, N] row-major, W4_BF16 or W4_F32 (others: W4_ERR_DTYPE).
 * Products and sums are formed in fp32 from the exact codes; where the tensor cores consume
 * the weight, each weight enters as bf16(fp32(value * scale)). The result satisfies
 *     |y - y_exact| <= 4e-3 * sum_k |x[m][k] * w[n][k]| + 1e-6 per element.
 * The kernel is chosen by M (decode GEMV for small M, tensor-core GEMM for larger M) and
 * by the alignment of the rows; every shape is served. workspace may be NULL when
 * w4_linear_workspace_bytes(...) returns 0; otherwise it must hold that many bytes and be
 * 256-byte aligned. Calls sharing one workspace must not overlap in time.
 */
w4_status w4_linear(const void *x, int64_t M, const uint8_t *codes, const float *scales,
                    int64_t N, int64_t K, const float *bias, void *y, w4_dtype y_dtype,
                    void *workspace, size_t workspace_bytes, w4_stream_t stream);

/* Workspace bytes w4_linear needs for this shape (0 = none). */
size_t w4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Workspace bytes w4_linear_asym_gidx uses for this shape when its codes are prepared
 * (perm given): the activations are gathered through perm into the workspace once per call
 * (M * K bf16, rounded up to 256 bytes) for the tensor-core GEMM (larger M) and for the decode
 * kernel (K a multiple of 128). A call given less (or no) workspace still succeeds on a
 * slower kernel. */
size_t w4_linear_asym_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t n_groups);

/*
 * w4_asym_prepare -- one-time act-order preparation of an asymmetric weight.
 * Sorts the columns by group (stable: columns of one group keep their order) and writes
 *   perm       out, int32 [K]: perm[j] = original column placed at sorted position j;
 *   codes_out  out, uint8 [N, ceil(K/2)]: the unsigned nibbles reordered, column j of
 *              codes_out = column perm[j] of codes_in (pad nibble zero).
 * The result is the same weight with relabelled columns; w4_linear_asym_gidx given `perm`
 * and `codes_out` gathers x through perm and reads each group's columns contiguously.
 * g_idx entries outside [0, n_groups) give W4_ERR_GIDX (this call synchronizes `stream`).
 */
w4_status w4_asym_prepare(const uint8_t *codes_in, const int32_t *g_idx, int64_t N, int64_t K,
                          int64_t n_groups, uint8_t *codes_out, int32_t *perm,
                          w4_stream_t stream);

/*
 * w4_linear_asym_gidx -- y = x . dequant_asym(W)^T + bias with act-order g_idx.
 * Page "keras/src/layers/core/dense.py", _int4_call sub-channel branch
 * (dequantize_with_sz_map(kernel, kernel_scale, kernel_zero, g_idx), matmul, bias) and
 * page "max/graph/quantization.py", QuantizationConfig (sym=False, desc_act=True).
 *   codes    uint8 [N, ceil(K/2)] unsigned nibbles. If perm == NULL they are in original
 *            column order; if perm != NULL they are the codes_out of w4_asym_prepare.
 *   scales   float32 [N, n_groups]; zeros int8 [N, n_groups] in [0, 15];
 *   g_idx    int32 [K]: group of ORIGINAL column k;  perm  int32 [K] or NULL.
 *   x, bias, y, y_dtype: as w4_linear; the same tolerance holds.
 *   workspace  NULL or 256-byte aligned device memory of w4_linear_asym_workspace_bytes(...)
 *              bytes (W4_ERR_WORKSPACE if misaligned); calls sharing it must not overlap.
 */
w4_status w4_linear_asym_gidx(const void *x, int64_t M, const uint8_t *codes,
                              const float *scales, const int8_t *zeros, const int32_t *g_idx,
                              const int32_t *perm, int64_t N, int64_t K, int64_t n_groups,
                              const float *bias, void *y, w4_dtype y_dtype, void *workspace,
                              size_t workspace_bytes, w4_stream_t stream);

/*
 * w4_linear_asym_gidx_noalloc -- w4_linear_asym_gidx for callers that cannot allocate.
 * The source pages have no counterpart to this call; it exists for host code that may not
 * allocate device memory when it calls the linear -- for example a program whose framework
 * owns every device allocation through its own pool, or a serving process that must not call
 * cudaMalloc after start-up (it synchronizes the device and can fail on a fragmented heap).
 * Arguments and results are those of w4_linear_asym_gidx without (workspace,
 * workspace_bytes): the scratch memory lives in one fixed 16 MiB array inside the library,
 * present on every GPU that loads the library until the process exits.
 *   - The call allocates nothing (no cudaMalloc / cudaFree, no allocating library routine).
 *   - The limit is M * K * 2 bytes (the activations gathered in bf16) <= 16 MiB, whichever
 *     kernel serves the shape: M = 2048 at K = 4096 is exactly 16 MiB and is accepted;
 *     M = 2049 or M = 4096 at K = 4096 return W4_ERR_SHAPE.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress); the first call on a device also loads the library's device
 *     code there, so make that first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents (each call overwrites
 *     what it reads, so nothing needs clearing). Calls that overlap on the GPU -- on
 *     different streams, or concurrently from several host threads -- race on it.
 */
w4_status w4_linear_asym_gidx_noalloc(const void *x, int64_t M, const uint8_t *codes,
                                      const float *scales, const int8_t *zeros,
                                      const int32_t *g_idx, const int32_t *perm, int64_t N,
                                      int64_t K, int64_t n_groups, const float *bias, void *y,
                                      w4_dtype y_dtype, w4_stream_t stream);

/*
 * w4_validate -- the LoopQ content checks (page "loopq/packed_weight.py", validate) on a
 * device-resident packed weight, reported in the page's order: W4_ERR_VERSION (format not
 * 1 or 2), W4_ERR_SCALE, W4_ERR_HIGH_NIBBLE, W4_ERR_RESERVED_CODE (v1 only). Shape and
 * dtype are the caller's contract. Synchronizes `stream`. The flags live in one word inside
 * the library shared by w4_validate and w4_validate_asym: calls must not overlap on the GPU.
 */
w4_status w4_validate(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                      int format_version, w4_stream_t stream);

/*
 * w4_validate_asym -- checks for the asymmetric variant: W4_ERR_SCALE, W4_ERR_HIGH_NIBBLE
 * (odd K), W4_ERR_ZERO (zero point outside [0, 15]), W4_ERR_GIDX (g_idx outside
 * [0, n_groups)). Synchronizes `stream`.
 */
w4_status w4_validate_asym(const uint8_t *codes, const float *scales, const int8_t *zeros,
                           const int32_t *g_idx, int64_t N, int64_t K, int64_t n_groups,
                           w4_stream_t stream);

/*
 * Per-channel symmetric int4: one fp32 scale per output row. Keras page
 * (keras/src/layers/core/dense.py, int4 diff), quantize's per-channel branch:
 * AbsMaxQuantizer(axis=0, value_range=(-8, 7)) and kernel_scale of shape (units,); the
 * quantizer's body is not on the page. Reading, the rule of w4_quantize_rtn over a whole
 * row and the Keras range: for each row n
 *     amax = max |W[n][:]|;  s = max(fl32(amax / 7), 2^-126);  q = clamp(rne(fl32(W / s)), -8, 7)
 * with the codes packed as in the format above (they lie in [-7, 7], valid for v1).
 * Only the scale layout differs from the group-32 format: w4_expand_channel_scales writes
 * the row's scale into every group, after which w4_dequantize, w4_linear,
 * w4_linear_backward_x and w4_validate serve the weight unchanged (keep the expanded array,
 * as a model keeps its parameters; expanding costs one small kernel).
 *
 * w4_quantize_rtn_channel -- W float32 [N, K] -> codes uint8 [N, ceil(K/2)], scales float32
 *   [N]; d_status as w4_quantize_rtn (NULL: synchronize and return W4_ERR_NONFINITE for a
 *   non-finite W). Bit-identical to the definition above.
 * w4_expand_channel_scales -- scales float32 [N] -> scales_out float32 [N, ceil(K/32)].
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE, W4_ERR_NONFINITE (quantize), W4_ERR_CUDA.
 */
w4_status w4_quantize_rtn_channel(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                  int32_t *d_status, w4_stream_t stream);
w4_status w4_expand_channel_scales(const float *scales, int64_t N, int64_t K, float *scales_out,
                                   w4_stream_t stream);

/*
 * w4_linear_channel -- the linear y = x . dequant(W)^T + bias for a per-channel weight: codes
 * as w4_linear, scales float32 [N] (one per row). The dequantized weight is q * s[n]; the
 * result agrees with w4_linear on the expanded scales within the linear tolerance (here the
 * row's sum of code * x is scaled once instead of each group's).
 *   M <= 16, K a multiple of 128, 16-byte aligned x and codes: a decode kernel that streams
 *   the codes and one scale per row (0.5 bytes per weight instead of 0.625 with expanded
 *   scales), no workspace.
 *   Other calls: the scales are expanded into `workspace` (w4_linear_channel_workspace_bytes:
 *   N * ceil(K/32) floats, 256-byte aligned) and the group-32 linear runs; W4_ERR_WORKSPACE if
 *   it is missing or too small.
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE, W4_ERR_DTYPE (y bf16 or f32), W4_ERR_WORKSPACE, W4_ERR_CUDA.
 */
size_t w4_linear_channel_workspace_bytes(int64_t M, int64_t N, int64_t K);
w4_status w4_linear_channel(const void *x, int64_t M, const uint8_t *codes, const float *scales, int64_t N,
                            int64_t K, const float *bias, void *y, w4_dtype y_dtype, void *workspace,
                            size_t workspace_bytes, w4_stream_t stream);

/*
 * w4_lora_merge -- merge a LoRA update into a packed weight and re-quantize it.
 * Keras page (keras/src/layers/core/dense.py, int4 diff), Dense's merged-kernel helper:
 * dequantize the kernel, add (lora_alpha / lora_rank) * matmul(lora_kernel_a, lora_kernel_b)
 * in the float domain, re-quantize, pack. With W stored [N, K]:
 *     w  = fp32(value * scale)                        (as w4_dequantize, f32)
 *     t  = 0; for j = 0 .. rank-1: t = fl32(t + fl32(lora_b_t[n][j] * lora_a_t[j][k]))
 *     w' = fl32(w + fl32(alpha_over_rank * t))
 * each step rounded in this order (no fused multiply-add), then the RTN rule of
 * w4_quantize_rtn on w' -> codes_out, scales_out. Bit-identical to that definition.
 *   lora_b_t  float32 [N, rank] (Keras lora_kernel_b transposed); lora_a_t float32 [rank, K]
 *             (lora_kernel_a transposed); both may be NULL when rank == 0.
 *   codes_out, scales_out  as w4_quantize_rtn's outputs; they may be codes and scales
 *             themselves (in place).
 *   d_status  as w4_quantize_rtn (a non-finite merged weight).
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE (sizes, rank < 0 or > 65536), W4_ERR_NONFINITE,
 * W4_ERR_CUDA.
 */
w4_status w4_lora_merge(const uint8_t *codes, const float *scales, int64_t N, int64_t K, const float *lora_b_t,
                        const float *lora_a_t, int64_t rank, float alpha_over_rank, uint8_t *codes_out,
                        float *scales_out, int32_t *d_status, w4_stream_t stream);

/*
 * w4_linear_backward_x -- input gradient of w4_linear: dx = dy . dequant(W).
 * Keras page (keras/src/layers/core/dense.py, int4 diff), _int4_call's grad_fn:
 * inputs_grad = matmul(upstream, transpose(float_kernel)); PaddleNLP page
 * (paddlenlp/quantization/quantization_linear.py), QuantizationLinearFunc.backward:
 * input_grad = matmul(grad_output, qdq_weight.T). With W stored [N, K] as above:
 *     dx[m][k] = sum_n dy[m][n] * fp32(value[n][k] * scales[n][k/32]),
 * fp32 accumulation: |dx - dx_ref| <= 4e-3 * sum_n |dy w| + 1e-6 per element.
 *   dy   bf16 [M, N] row-major (the upstream gradient).   codes, scales: as w4_linear.
 *   dx   [M, K] row-major, bf16 or float32 (dx_dtype), written.
 *   workspace  w4_linear_backward_x_workspace_bytes(M, N, K) bytes, 256-byte aligned (0:
 *        none needed); the rows are split over CTAs and the splits added in a fixed order,
 *        so results are deterministic.
 * K a multiple of 8 with 4-byte aligned codes and scales runs the streaming kernel; other
 * shapes a plain kernel.
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE, W4_ERR_DTYPE (dx_dtype not bf16 / f32),
 * W4_ERR_WORKSPACE, W4_ERR_CUDA.
 */
size_t w4_linear_backward_x_workspace_bytes(int64_t M, int64_t N, int64_t K);
w4_status w4_linear_backward_x(const void *dy, int64_t M, const uint8_t *codes, const float *scales, int64_t N,
                               int64_t K, void *dx, w4_dtype dx_dtype, void *workspace, size_t workspace_bytes,
                               w4_stream_t stream);

/*
 * GGUF Q4_0 blocks. Page "max/python/max/graph/quantization.py" (Modular MAX),
 * QuantizationEncoding.Q4_0 and its block parameters: a block encodes 32 consecutive
 * elements in 2 + 32/2 = 18 bytes, the scale d and then the 4-bit codes. Readings (the page
 * gives only the sizes and the field order): d is IEEE binary16, little-endian, in bytes
 * 0-1; code byte j (bytes 2 + j, j < 16) holds element j in its LOW nibble and element
 * j + 16 in its HIGH nibble; an element's value is fp32(d * (code - 8)) (exact).
 *   blocks  uint8 [N, K/32, 18], row-major: a row's K/32 blocks are consecutive, rows are
 *           consecutive (row n starts at byte n * K/32 * 18). K must be a multiple of 32.
 * The content is not checked: a non-finite d makes its block's elements NaN or infinite,
 * as the definition gives.
 */

/*
 * w4_dequantize_q4_0 -- dense [N, K] weight of out_dtype (bf16 / f16 / f32 / f64) from Q4_0
 * blocks: fp32(d * (code - 8)), then round to nearest even (bf16, f16; f16 overflows to
 * infinity past 65504) or widen exactly (f64). Bit-identical to that definition.
 *   out  [N, K] row-major, written.
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE (sizes, K not a multiple of 32), W4_ERR_DTYPE,
 * W4_ERR_CUDA.
 */
w4_status w4_dequantize_q4_0(const uint8_t *blocks, int64_t N, int64_t K, w4_dtype out_dtype, void *out,
                             w4_stream_t stream);

/*
 * w4_linear_q4_0 -- y = x . dequant(W)^T (+ bias) for Q4_0 blocks, fp32 accumulation:
 * |y - y_ref| <= 4e-3 * sum_k |x w| + 1e-6 per element (y_ref the exact sum of x times the
 * fp32 dequantized weight, plus the bias).
 *   x     bf16 [M, K] row-major.    bias  optional float32 [N].
 *   y     [M, N] row-major, bf16 or float32 (y_dtype), written.
 * M = 1 with K a multiple of 256 and 16-byte aligned x and blocks runs the TMA-fed
 * tensor-core decode GEMV (launched like w4_linear's decode kernel: programmatic dependent
 * launch, and w4_set_weight_prefetch applies); every other shape a plain kernel.
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE, W4_ERR_DTYPE (y_dtype not bf16 / f32), W4_ERR_CUDA.
 */
w4_status w4_linear_q4_0(const void *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K,
                         const float *bias, void *y, w4_dtype y_dtype, w4_stream_t stream);

/*
 * w4_q4_0_to_group32 -- re-lay Q4_0 blocks out as this library's packed group-32 format, once
 * per weight (at load time). MAX page (max/python/max/graph/quantization.py),
 * QuantizationEncoding.Q4_0: a block is 32 consecutive columns of a row with one scale, and
 * its value d * (c - 8) is scale * code with
 *     scales[n][g] = fp32(d[n][g])                 (binary16 widened exactly)
 *     code of column k = c[n][k] - 8 in [-8, 7]    (a two's-complement nibble; -8 is the
 *                                                   format-v2 code, accepted by every call)
 * so w4_linear, w4_dequantize, w4_linear_backward_x ... on (codes, scales) see exactly the
 * dequantized weights of the blocks: fp32(scale * code) = fp32(d * (c - 8)), both exact.
 * Any binary16 d is carried over (negative, zero, subnormal; a non-finite d becomes a
 * non-finite scale, which w4_validate reports).
 *   blocks  uint8 [N, K/32, 18] (device), K a multiple of 32; not modified.
 *   codes   uint8 [N, K/2] (device, caller-owned, written); scales float32 [N, K/32]
 *           (device, caller-owned, written). Neither may overlap the blocks.
 * Errors: W4_ERR_NULL, W4_ERR_SHAPE (sizes, K not a multiple of 32), W4_ERR_CUDA.
 */
w4_status w4_q4_0_to_group32(const uint8_t *blocks, int64_t N, int64_t K, uint8_t *codes, float *scales,
                             w4_stream_t stream);

/*
 * w4_set_weight_prefetch -- launch policy of the decode linear (process-wide; default 0).
 * The source pages have no counterpart to this call: it only decides when a kernel starts.
 * The M = 1 decode kernel is launched with CUDA programmatic dependent launch: it may begin
 * while the previous kernel of its stream is still running, and it reads x (and bias) and
 * writes y only after that kernel has completed and its writes are visible. With enable = 1
 * it also starts streaming codes and scales at once, hiding its ramp-up behind the previous
 * kernel in a chain of decode linears.
 * Contract while enabled: the codes and scales of a decode call must already be complete
 * when the chain of overlapping kernels before it began -- write them earlier and separate
 * the two by a stream synchronization, an event, or any kernel launched without
 * programmatic serialization (every other kernel of this library is). Weights written by a
 * kernel that may still be running may be read stale. Returns the previous setting.
 */
int w4_set_weight_prefetch(int enable);

/* Error word written by bounded device-side waits (W4_OK if none expired). Reading it
 * synchronizes the device and clears it. */
w4_status w4_device_error(void);

/*
 * w4_selftest_wait_timeout -- diagnostic with no counterpart on the source pages: launches one
 * CTA on `stream` that waits, through the same bounded wait every kernel of the library uses,
 * on a barrier nothing arrives on, with a limit of `limit_ns` nanoseconds (1 .. 1e9). The wait
 * expires and records W4_ERR_TIMEOUT in the error word that w4_device_error() reads, exactly
 * as an expired wait in a real kernel would; no copy or MMA is in flight and the CUDA context
 * stays usable. Returns W4_ERR_SHAPE for a limit outside the range, else the launch status.
 */
w4_status w4_selftest_wait_timeout(uint64_t limit_ns, w4_stream_t stream);

/* The cudaError_t of the last call that returned W4_ERR_CUDA (0 if none). */
int w4_last_cuda_error(void);

/* Static description of a status code. */
const char *w4_status_string(w4_status status);

/* Library ABI version (major * 100 + minor). */
int w4_version(void);

/*
 * w4_last_linear_kernel -- name of the kernel family that the calling thread's last
 * w4_linear / w4_linear_asym_gidx / w4_linear_asym_gidx_noalloc call launched: "gemv_tma",
 * "gather_x+gemv_tma", "gemv_rows", "gemv_mma", "gemv", "gemm_tc", "gather_x+gemm_tc" or
 * "linear_generic"; w4_linear_channel reports "gemv_tma_channel" or, after expanding the
 * scales, the group-32 kernel it ran ("none" before the first call on the thread). A static string owned by the
 * library; set only when a call got as far as launching. For tests and profiling: the choice
 * depends on M, the shape, the alignment of the arrays and the workspace (no counterpart on
 * the source pages).
 */
const char *w4_last_linear_kernel(void);

#ifdef __cplusplus
}
#endif

#endif /* W4_H_ */

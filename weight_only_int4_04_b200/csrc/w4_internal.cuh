// Internal declarations and device helpers shared by the kernels of libw4.
// Target: sm_100a only. Nothing here is part of the C ABI (see include/w4.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "w4.h"

namespace w4i {

// ---------------------------------------------------------------------------
// Launch parameter blocks
// ---------------------------------------------------------------------------

struct LinearParams {
  const __nv_bfloat16 *x;  // [M, K]
  const uint8_t *codes;    // [N, P], P = ceil(K/2)
  const float *scales;     // sym: [N, ceil(K/32)]; asym: [N, n_groups]
  const int8_t *zeros;     // asym only: [N, n_groups]
  const int32_t *g_idx;    // asym only: [K], group of ORIGINAL column
  const int32_t *perm;     // asym only, may be null: sorted position -> original column
  const float *bias;       // [N] or null
  void *y;                 // [M, N]
  int64_t M, N, K;
  int n_groups;            // asym only
  int y_dtype;             // W4_BF16 or W4_F32
  int asym;                // 0 = symmetric signed codes, 1 = asymmetric unsigned codes
  int channel;             // symmetric only: 1 = one scale per row, scales [N] (per-channel)
};

// Each launcher enqueues on `stream` and returns the launch error (cudaSuccess or not).
cudaError_t launch_quantize_rtn(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                int32_t *status, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                              int out_dtype, void *out, cudaStream_t stream);
cudaError_t launch_validate(const uint8_t *codes, const float *scales, const int8_t *zeros,
                            const int32_t *g_idx, int64_t N, int64_t K, int64_t n_groups,
                            int format_version, int asym, uint32_t *flags, cudaStream_t stream);
cudaError_t launch_reorder_codes(const uint8_t *codes_in, const int32_t *perm, int64_t N, int64_t K,
                                 uint8_t *codes_out, cudaStream_t stream);
cudaError_t launch_linear_generic(const LinearParams &p, cudaStream_t stream);
// Decode GEMV (CUDA cores). Returns cudaErrorNotSupported when the shape/alignment does not
// fit this kernel (the caller then picks another).
cudaError_t launch_gemv(const LinearParams &p, cudaStream_t stream);
bool gemv_supports(const LinearParams &p);
// Register-streaming decode GEMV (M = 1): every lane prefetches its own code rows.
cudaError_t launch_gemv_rows(const LinearParams &p, cudaStream_t stream);
bool gemv_rows_supports(const LinearParams &p);
// Small-M linear (M <= 16) on register-fed tensor cores (mma.sync), streaming rows through a
// bulk-copy slot ring; the main decode path.
cudaError_t launch_gemv_mma(const LinearParams &p, int32_t *err, cudaStream_t stream);
bool gemv_mma_supports(const LinearParams &p);
// Decode GEMV / small-M linear (M <= 16, symmetric codes, K a multiple of 128, 16-byte
// aligned arrays, activations that fit in shared memory) on register-fed tensor cores with
// a TMA stage ring; launched with programmatic stream serialization. `prefetch` lets it
// stream codes and scales before the previous kernel of the stream has finished (x and y
// are touched only after it has).
// Act-order: `x_sorted` (or null) holds x already gathered through perm (launch_gather_x).
cudaError_t launch_gemv_tma(const LinearParams &p, bool prefetch, const __nv_bfloat16 *x_sorted, int32_t *err,
                            cudaStream_t stream);
// xg[m][j] = x[m][perm[j]] for the act-order kernels (K % 8 == 0, 16-byte aligned xg).
cudaError_t launch_gather_x(const __nv_bfloat16 *x, const int32_t *perm, int64_t M, int64_t K, __nv_bfloat16 *xg,
                            cudaStream_t stream);
bool gemv_tma_supports(const LinearParams &p);
// Act-order: true when launch_gemv_tma gathers x through perm itself (one activation row of
// moderate length); otherwise the caller passes x_sorted.
bool gemv_tma_gathers_x(const LinearParams &p);
// Tensor-core GEMM (tcgen05, TMA, TMEM) for larger M, aligned rows. The asymmetric
// act-order variant gathers x through perm into `workspace` (gemm_tc_asym_workspace bytes).
cudaError_t launch_gemm_tc(const LinearParams &p, int32_t *err, cudaStream_t stream, void *workspace);
bool gemm_tc_supports(const LinearParams &p);
size_t gemm_tc_asym_workspace(int64_t M, int64_t K);

// GGUF Q4_0 blocks (uint8 [N, K/32, 18]): the linear (M = 1 with K a multiple of 256 and
// 16-byte aligned x and blocks on the TMA-fed tensor-core GEMV, anything else on a plain
// kernel) and the dequantization to a dense [N, K] array of out_dtype.
cudaError_t launch_q4_0_linear(const __nv_bfloat16 *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K,
                               const float *bias, void *y, int y_dtype, bool prefetch, int32_t *err,
                               cudaStream_t stream);
bool q4_0_gemv_supports(const void *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K, int y_dtype);
cudaError_t launch_q4_0_to_group32(const uint8_t *blocks, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                   cudaStream_t stream);
cudaError_t launch_q4_0_dequantize(const uint8_t *blocks, int64_t N, int64_t K, int out_dtype, void *out,
                                   cudaStream_t stream);

// Input gradient dx = dy . dequant(W) (symmetric group-32 codes). The fast kernel needs K a
// multiple of 8 and 4-byte aligned codes and scales, and, when it splits the rows over
// CTAs, linear_backward_x_workspace(M, N, K) bytes of workspace; otherwise a plain kernel.
size_t linear_backward_x_workspace(int64_t M, int64_t N, int64_t K);
cudaError_t launch_linear_backward_x(const __nv_bfloat16 *dy, int64_t M, const uint8_t *codes, const float *scales,
                                     int64_t N, int64_t K, void *dx, int dx_dtype, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream);

// Per-channel symmetric int4 (one scale per row): RTN quantize + pack, and the expansion of
// the [N] scales to the group layout [N, ceil(K/32)] the other kernels read.
cudaError_t launch_quantize_rtn_channel(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                        int32_t *status, cudaStream_t stream);
cudaError_t launch_expand_channel_scales(const float *scales, int64_t N, int64_t K, float *out,
                                         cudaStream_t stream);

// LoRA merge: codes/scales + alpha_over_rank * lora_b_t . lora_a_t, re-quantized (RTN
// group-32) into codes_out/scales_out (which may be the inputs). status as quantize.
cudaError_t launch_lora_merge(const uint8_t *codes, const float *scales, const float *lora_b_t,
                              const float *lora_a_t, int64_t N, int64_t K, int64_t r, float alpha_over_rank,
                              uint8_t *codes_out, float *scales_out, int32_t *status, cudaStream_t stream);

// Diagnostic: one CTA waits, with the library's bounded wait and a limit of limit_ns, on a
// barrier that nothing arrives on, so the wait expires and records W4_ERR_TIMEOUT in `err`.
// No copy or MMA is in flight; the kernel returns normally.
cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *err, cudaStream_t stream);

// Validation flag bits (w4_validate reports them in the page's order).
enum : uint32_t {
  FLAG_SCALE = 1u << 0,
  FLAG_HIGH_NIBBLE = 1u << 1,
  FLAG_RESERVED = 1u << 2,
  FLAG_ZERO = 1u << 3,
  FLAG_GIDX = 1u << 4,
};

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------

// (a & b) ^ c in one LOP3.
__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// bf16x2 a - b computed as fma(a, 1, -b) (fma.rn.bf16x2, a native sm_80+ instruction;
// exact for the small integers it is used on).
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(0x3F803F80u), "r"(b ^ 0x80008000u));
  return d;
}

// Nibble pair -> bf16x2 with the integer 128 + (n ^ xmask) in each half.
// The low nibble of each 16-bit half of `w` lands in the low mantissa bits of the bf16
// 128.0 (0x4300), whose ulp is 1, so the result is the exact integer. xor 8 turns a
// two's-complement nibble n into n_signed + 8.
// Signed codes: 0x43084308 gives 136 + q; unsigned codes: 0x43004300 gives 128 + u.
__device__ __forceinline__ uint32_t nib_pair_bf16(uint32_t w, uint32_t magic) {
  return lop3_and_xor(w, 0x000F000Fu, magic);
}

// fp32 acc += bf16 a * bf16 b for both halves of two bf16x2 registers (mixed-precision
// FMA: the bf16 x small-integer product is exact, one fp32 rounding per step).
__device__ __forceinline__ float fma2_bf16_f32(uint32_t a2, uint32_t b2, float acc) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a2), "r"(b2));
  return acc;
}

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace w4i

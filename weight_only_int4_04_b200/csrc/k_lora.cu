// LoRA merge into a packed weight (Keras page, keras/src/layers/core/dense.py int4 diff,
// Dense's merged-kernel helper: dequantize, add (lora_alpha / lora_rank) * A . B in the
// float domain, re-quantize, pack). Layout [N, K]: delta[n][k] = c * sum_j b[n][j] * a[j][k]
// with b = B^T [N, r], a = A^T [r, K], c = alpha / rank. Reading of the arithmetic (fp32,
// every step rounded, in this order, so the new codes depend on the inputs alone):
//     w = fl32(q * s);  t = 0; for j: t = fl32(t + fl32(b[n][j] * a[j][k]));  w' = fl32(w + fl32(c * t))
// then the RTN group-32 rule of w4_quantize_rtn on w'. The products and sums use the
// rounded-intrinsic forms (__fmul_rn / __fadd_rn): never contracted into FMAs.
//   * lora_merge_kernel: as quantize_rtn_kernel, eight lanes per 32-column group and four
//     columns per lane; each lane dequantizes its columns, adds the update, and the eight
//     lanes reduce the group's amax by shuffles. A code byte belongs to one group, so the
//     output may overwrite the input.
#include <cfloat>

#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int kLoraThreads = 256;

__global__ void __launch_bounds__(kLoraThreads) lora_merge_kernel(const uint8_t *codes, const float *scales,
                                                                  const float *__restrict__ b,
                                                                  const float *__restrict__ a, int64_t N, int64_t K,
                                                                  int64_t r, float c, uint8_t *codes_out,
                                                                  float *scales_out, int32_t *__restrict__ status) {
  const int64_t G = (K + 31) / 32;
  const int64_t P = (K + 1) / 2;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int64_t tasks = N * G;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warp_stride = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  // a warp owns four consecutive (row, group) tasks per trip; the trip count is warp-uniform
  // so every lane reaches the shuffles (lanes past the end carry zeros and store nothing)
  for (int64_t wb = warp_id * 4; wb < tasks; wb += warp_stride * 4) {
    const int64_t t = wb + (lane >> 3);
    const bool active = t < tasks;
    const int64_t n = active ? t / G : 0, g = active ? t % G : 0;
    const int64_t c0 = 32 * g + 4 * sub;
    float w[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (active) {
      const float s = scales[n * G + g];
      const uint8_t *crow = codes + n * P;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int64_t j = 0; j < r; ++j) {
        const float bj = b[n * r + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (c0 + i < K) acc[i] = __fadd_rn(acc[i], __fmul_rn(bj, a[j * K + c0 + i]));
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t col = c0 + i;
        if (col < K) {
          const uint32_t byte = crow[col >> 1];
          const int u = static_cast<int>((col & 1) ? (byte >> 4) : (byte & 15u));
          const float deq = __fmul_rn(static_cast<float>(u >= 8 ? u - 16 : u), s);
          w[i] = __fadd_rn(deq, __fmul_rn(c, acc[i]));
          bad |= !isfinite(w[i]);
        }
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(w[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float s2 = fmaxf(__fdiv_rn(amax, 7.0f), FLT_MIN);
    uint32_t nib[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = __float2int_rn(__fdiv_rn(w[i], s2));  // round half to even
      q = q < -7 ? -7 : (q > 7 ? 7 : q);
      nib[i] = (c0 + i < K) ? (static_cast<uint32_t>(q) & 15u) : 0u;  // pad nibble = 0
    }
    // the output may alias the input: a lane writes only the two code bytes it read itself,
    // and the group's scale, read by its eight lanes before the shuffles, is written after
    if (!active) continue;
    uint8_t *orow = codes_out + n * P;
    const int64_t jb = c0 / 2;
    if (jb < P) orow[jb] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
    if (jb + 1 < P) orow[jb + 1] = static_cast<uint8_t>(nib[2] | (nib[3] << 4));
    if (sub == 0) scales_out[n * G + g] = s2;
  }
  if (bad) *status = W4_ERR_NONFINITE;
}

}  // namespace

cudaError_t launch_lora_merge(const uint8_t *codes, const float *scales, const float *lora_b_t,
                              const float *lora_a_t, int64_t N, int64_t K, int64_t r, float alpha_over_rank,
                              uint8_t *codes_out, float *scales_out, int32_t *status, cudaStream_t stream) {
  const int64_t groups = N * ((K + 31) / 32);
  int64_t blocks = (groups + (kLoraThreads / 8) - 1) / (kLoraThreads / 8);
  if (blocks > 148LL * 8 * 4) blocks = 148LL * 8 * 4;
  if (blocks < 1) blocks = 1;
  lora_merge_kernel<<<static_cast<unsigned>(blocks), kLoraThreads, 0, stream>>>(
      codes, scales, lora_b_t, lora_a_t, N, K, r, alpha_over_rank, codes_out, scales_out, status);
  return cudaGetLastError();
}

}  // namespace w4i

// Per-channel symmetric int4: one fp32 scale per output row (Keras page, keras/src/layers/
// core/dense.py int4 diff, quantize's per-channel branch: AbsMaxQuantizer(axis=0,
// value_range=(-8, 7)), kernel_scale of shape (units,)). Reading: per row n
//     s_n = max(fl32(amax_n / 7), 2^-126),  q = clamp(rne(fl32(w / s_n)), -8, 7),
// the scale multiplying the code as in the packed group-32 format. Only the scale layout
// differs from that format, so a per-channel weight is served by the group-32 kernels once
// its scales are expanded to one per 32-column group (expand_channel_scales_kernel).
//   * quantize_rtn_channel_kernel: one CTA per row (grid-stride over rows): the row's amax
//     (block reduction of max |w|, non-finite flag), then every byte of the packed row.
//   * expand_channel_scales_kernel: scales_out[n][g] = scales[n].
#include <cfloat>

#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int kChThreads = 256;

__global__ void __launch_bounds__(kChThreads) quantize_rtn_channel_kernel(const float *__restrict__ W, int64_t N,
                                                                          int64_t K, uint8_t *__restrict__ codes,
                                                                          float *__restrict__ scales,
                                                                          int32_t *__restrict__ status) {
  __shared__ float part[kChThreads / 32];
  const int64_t P = (K + 1) / 2;
  bool bad = false;
  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const float *row = W + n * K;
    float amax = 0.0f;
    for (int64_t k = threadIdx.x; k < K; k += kChThreads) {
      const float v = row[k];
      bad |= !isfinite(v);
      amax = fmaxf(amax, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = part[0];
#pragma unroll
    for (int w = 1; w < kChThreads / 32; ++w) amax = fmaxf(amax, part[w]);
    __syncthreads();  // part is rewritten by the next row
    const float s = fmaxf(__fdiv_rn(amax, 7.0f), FLT_MIN);  // IEEE round-to-nearest divide
    if (threadIdx.x == 0) scales[n] = s;
    for (int64_t j = threadIdx.x; j < P; j += kChThreads) {
      uint32_t nib[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k = 2 * j + h;
        int q = 0;
        if (k < K) {
          q = __float2int_rn(__fdiv_rn(row[k], s));  // round half to even
          q = q < -8 ? -8 : (q > 7 ? 7 : q);
        }
        nib[h] = static_cast<uint32_t>(q) & 15u;  // the pad nibble of an odd row stays 0
      }
      codes[n * P + j] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
    }
  }
  if (bad) *status = W4_ERR_NONFINITE;
}

__global__ void __launch_bounds__(256) expand_channel_scales_kernel(const float *__restrict__ scales, int64_t N,
                                                                    int64_t G, float *__restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < N * G) out[i] = scales[i / G];
}

}  // namespace

cudaError_t launch_quantize_rtn_channel(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                        int32_t *status, cudaStream_t stream) {
  const int64_t grid = N < 148LL * 16 ? N : 148LL * 16;
  quantize_rtn_channel_kernel<<<static_cast<unsigned>(grid), kChThreads, 0, stream>>>(W, N, K, codes, scales,
                                                                                     status);
  return cudaGetLastError();
}

cudaError_t launch_expand_channel_scales(const float *scales, int64_t N, int64_t K, float *out,
                                         cudaStream_t stream) {
  const int64_t G = (K + 31) / 32, total = N * G;
  if ((total + 255) / 256 > 0x7fffffffLL) return cudaErrorInvalidValue;
  expand_channel_scales_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(scales, N, G, out);
  return cudaGetLastError();
}

}  // namespace w4i

// Generic fused dequantize + linear on CUDA cores: serves every shape and alignment (odd
// widths, ragged groups, unaligned rows, unsorted act-order maps). The fast kernels take
// the aligned shapes; this one is the path for the rest.
//
// y[m][n] = sum_k x[m][k] * w[n][k] + b[n], with w[n][k] the exact fp32 dequantized weight:
//   symmetric : fp32(v * s[n][k/32]),               v the signed nibble
//   asymmetric: fp32((u - z[n][g]) * s[n][g]),      g = g_idx[col], u the unsigned nibble
// (page "loopq/packed_weight.py", _dequantize_validated; page "keras/src/layers/core/
// dense.py", _int4_call). Accumulation in fp32, bias added before the output rounding.
#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int BM = 64, BN = 64, BK = 32, kThreads = 256;

__global__ void __launch_bounds__(kThreads) linear_generic_kernel(LinearParams p) {
  __shared__ float xs[BK][BM + 1];
  __shared__ float ws[BK][BN + 1];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t K = p.K, M = p.M, N = p.N;
  const int64_t P = (K + 1) / 2;
  const int64_t G = p.asym ? p.n_groups : (K + 31) / 32;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int64_t k0 = 0; k0 < K; k0 += BK) {
    // x tile [BM x BK] -> xs[k][m]; in act-order mode with a perm, sorted column k reads
    // the activation of original column perm[k].
#pragma unroll
    for (int i = 0; i < (BM * BK) / kThreads; ++i) {
      const int e = tid + i * kThreads;
      const int mm = e / BK, kk = e % BK;
      const int64_t m = m0 + mm, k = k0 + kk;
      float v = 0.0f;
      if (m < M && k < K) {
        const int64_t col = (p.asym && p.perm) ? p.perm[k] : k;
        v = __bfloat162float(p.x[m * K + col]);
      }
      xs[kk][mm] = v;
    }
    // weight tile [BN x BK] -> ws[k][n], dequantized to exact fp32
#pragma unroll
    for (int i = 0; i < (BN * BK) / kThreads; ++i) {
      const int e = tid + i * kThreads;
      const int nn = e / BK, kk = e % BK;
      const int64_t n = n0 + nn, k = k0 + kk;
      float w = 0.0f;
      if (n < N && k < K) {
        const uint32_t byte = p.codes[n * P + k / 2];
        const int nib = static_cast<int>((k & 1) ? (byte >> 4) : (byte & 15u));
        if (!p.asym) {
          const int v = nib >= 8 ? nib - 16 : nib;
          w = __fmul_rn(static_cast<float>(v), p.scales[n * G + k / 32]);
        } else {
          const int64_t col = p.perm ? p.perm[k] : k;
          const int64_t g = p.g_idx[col];
          w = __fmul_rn(static_cast<float>(nib - static_cast<int>(p.zeros[n * G + g])), p.scales[n * G + g]);
        }
      }
      ws[kk][nn] = w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (p.bias) v += p.bias[n];
      if (p.y_dtype == W4_F32) {
        static_cast<float *>(p.y)[m * N + n] = v;
      } else {
        static_cast<__nv_bfloat16 *>(p.y)[m * N + n] = __float2bfloat16_rn(v);
      }
    }
  }
}

}  // namespace

cudaError_t launch_linear_generic(const LinearParams &p, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((p.N + BN - 1) / BN), static_cast<unsigned>((p.M + BM - 1) / BM));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  linear_generic_kernel<<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace w4i

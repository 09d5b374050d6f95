// Input gradient of the linear: dx[m, k] = sum_n dy[m, n] * w[n, k], w = fp32(q * s) the
// dequantized weight (Keras page, _int4_call's grad_fn: matmul(upstream, transpose(kernel));
// PaddleNLP page, QuantizationLinearFunc.backward: matmul(grad_output, qdq_weight.T); the
// weight here is stored [N, K], rows = output features).
//
// The contraction runs over the rows of the packed weight, so the code bytes pair columns
// along k, not along the contracted axis: the kernel streams the weight row by row on CUDA
// cores instead of feeding tensor-core fragments.
//   * bwd_x_kernel<TM> (K a multiple of 8, 4-byte aligned codes and scales): CTA (tile,
//     split, token chunk) owns 256 columns, a contiguous slice of rows and TM <= 8 upstream
//     rows. Its eight warps take the slice's rows in turn; lane l holds code word l of the
//     tile (8 consecutive columns, one group) for four rows at a time (coalesced 128-byte
//     row segments, read once, L1 bypassed). Each nibble becomes the exact float q through
//     the fp32 mantissa (lop3 into 2^23 + (q + 8), minus 2^23 + 8); the coefficient
//     dy[m, n] * s[n, g] is formed once per (row, token) and every weight costs one FFMA per
//     token. The warps' sums meet in shared memory in a fixed order; when the rows are split
//     over several CTAs each writes its partial sums to the workspace and
//     bwd_x_reduce_kernel adds the splits in a fixed order (deterministic results).
//   * bwd_x_plain_kernel: any K, one thread per (token, column), rows in order.
#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int kBwdTile = 256;   // columns per CTA (32 code words)
constexpr int kBwdWarps = 8;
constexpr int kBwdTargetCtas = 592;  // four per SM on a 148-SM part; sets the row split
constexpr int kBwdStageRows = 1024;  // rows whose upstream gradient is staged in shared memory at once
constexpr int64_t kBwdMinRows = 64;  // rows per split at least

__device__ __forceinline__ uint32_t ld_stream_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// read-only scale load, kept in program order with the code loads (issued together up front)
__device__ __forceinline__ float ld_scale(const float *p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float nibble_float(uint32_t w, int j) {
  // 0x4B000000 | (nibble ^ 8) = 2^23 + q + 8 exactly; subtracting 2^23 + 8 leaves q
  return __uint_as_float(lop3_and_xor(w >> (4 * j), 0xFu, 0x4B000008u)) - 8388616.0f;
}

__device__ __forceinline__ void store_out(void *out, int dtype, int64_t i, float v) {
  if (dtype == W4_F32)
    static_cast<float *>(out)[i] = v;
  else
    static_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(v);
}

template <int TM>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_x_kernel(const __nv_bfloat16 *__restrict__ dy,
                                                               const uint8_t *__restrict__ codes,
                                                               const float *__restrict__ scales,
                                                               float *__restrict__ part, void *dx, int dx_dtype,
                                                               int64_t M, int64_t N, int64_t K, int64_t rows_per_split,
                                                               int splits) {
  __shared__ __align__(16) float red[kBwdWarps][kBwdTile];
  __shared__ __align__(16) float sdy[kBwdStageRows * TM];  // [row][token], fp32
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = static_cast<int>(blockIdx.x), split = static_cast<int>(blockIdx.y);
  const int64_t m0 = static_cast<int64_t>(blockIdx.z) * TM;
  const int64_t P4 = K / 8;  // code words per row
  const int64_t G = (K + 31) / 32;
  const int64_t word = static_cast<int64_t>(tile) * 32 + lane;
  const bool active = word < P4;
  const int64_t grp = word >> 2;  // 4 words = 32 columns per group
  const int64_t n0 = static_cast<int64_t>(split) * rows_per_split;
  const int64_t n1 = (n0 + rows_per_split < N) ? n0 + rows_per_split : N;
  const uint32_t *cw = reinterpret_cast<const uint32_t *>(codes);

  float acc[TM][8];
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[m][j] = 0.0f;

  // rows in flight per warp: enough bytes outstanding to cover the memory latency
  constexpr int kRowsAhead = TM == 1 ? 16 : (TM == 8 ? 4 : 8);
  for (int64_t c0 = n0; c0 < n1; c0 += kBwdStageRows) {
    const int64_t c1 = (c0 + kBwdStageRows < n1) ? c0 + kBwdStageRows : n1;
    // the upstream gradient of these rows, once per CTA: sdy[(n - c0) * TM + m] = dy[m0 + m][n]
#pragma unroll
    for (int m = 0; m < TM; ++m)
      for (int64_t n = c0 + threadIdx.x; n < c1; n += blockDim.x)
        sdy[(n - c0) * TM + m] = (m0 + m < M) ? __bfloat162float(dy[(m0 + m) * N + n]) : 0.0f;
    __syncthreads();
    for (int64_t nb = c0 + warp; nb < c1; nb += kRowsAhead * kBwdWarps) {
      uint32_t w[kRowsAhead];
      float s[kRowsAhead];
#pragma unroll
      for (int r = 0; r < kRowsAhead; ++r) {
        const int64_t n = nb + r * kBwdWarps;
        const bool ok = n < c1 && active;
        w[r] = ok ? ld_stream_u32(cw + n * P4 + word) : 0u;
        s[r] = ok ? ld_scale(scales + n * G + grp) : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < kRowsAhead; ++r) {
        const int64_t n = nb + r * kBwdWarps;
        const int64_t ln = (n < c1 ? n : c0) - c0;  // rows past the range carry s = 0
        float coef[TM];
#pragma unroll
        for (int m = 0; m < TM; ++m) coef[m] = sdy[ln * TM + m] * s[r];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float q = nibble_float(w[r], j);
#pragma unroll
          for (int m = 0; m < TM; ++m) acc[m][j] = fmaf(coef[m], q, acc[m][j]);
        }
      }
    }
    __syncthreads();
  }

  // the warps' column sums meet in shared memory, added in warp order
  const int64_t k = static_cast<int64_t>(tile) * kBwdTile + threadIdx.x;
#pragma unroll
  for (int m = 0; m < TM; ++m) {
    float4 *rw = reinterpret_cast<float4 *>(&red[warp][lane * 8]);
    rw[0] = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
    rw[1] = make_float4(acc[m][4], acc[m][5], acc[m][6], acc[m][7]);
    __syncthreads();
    float v = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < kBwdWarps; ++w2) v += red[w2][threadIdx.x];
    if (k < K && m0 + m < M) {
      if (splits == 1)
        store_out(dx, dx_dtype, (m0 + m) * K + k, v);
      else
        part[(static_cast<int64_t>(split) * M + m0 + m) * K + k] = v;
    }
    __syncthreads();
  }
}

// One upstream row (M = 1), K a multiple of 32, 16-byte aligned codes: lane l streams the 16
// code bytes of group l of a 1024-column tile per row (4x the bytes per load of the word
// kernel), one scale per row; otherwise as bwd_x_kernel<1>.
constexpr int kBwdWideTile = 1024;

__device__ __forceinline__ uint4 ld_stream_u128(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(32 * kBwdWarps) bwd_x_wide_kernel(const __nv_bfloat16 *__restrict__ dy,
                                                                    const uint8_t *__restrict__ codes,
                                                                    const float *__restrict__ scales,
                                                                    float *__restrict__ part, void *dx, int dx_dtype,
                                                                    int64_t N, int64_t K, int64_t rows_per_split,
                                                                    int splits) {
  __shared__ __align__(16) float red[kBwdWarps][kBwdWideTile];
  __shared__ float sdy[kBwdStageRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = static_cast<int>(blockIdx.x), split = static_cast<int>(blockIdx.y);
  const int64_t G = K / 32;  // groups = 16-byte code chunks per row
  const int64_t grp = static_cast<int64_t>(tile) * 32 + lane;
  const bool active = grp < G;
  const int64_t n0 = static_cast<int64_t>(split) * rows_per_split;
  const int64_t n1 = (n0 + rows_per_split < N) ? n0 + rows_per_split : N;
  const uint4 *c4 = reinterpret_cast<const uint4 *>(codes);

  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
  constexpr int kRowsAhead = 4;
  for (int64_t c0 = n0; c0 < n1; c0 += kBwdStageRows) {
    const int64_t c1 = (c0 + kBwdStageRows < n1) ? c0 + kBwdStageRows : n1;
    for (int64_t n = c0 + threadIdx.x; n < c1; n += blockDim.x) sdy[n - c0] = __bfloat162float(dy[n]);
    __syncthreads();
    for (int64_t nb = c0 + warp; nb < c1; nb += kRowsAhead * kBwdWarps) {
      uint4 w[kRowsAhead];
      float s[kRowsAhead];
#pragma unroll
      for (int r = 0; r < kRowsAhead; ++r) {
        const int64_t n = nb + r * kBwdWarps;
        const bool ok = n < c1 && active;
        w[r] = ok ? ld_stream_u128(c4 + n * G + grp) : make_uint4(0u, 0u, 0u, 0u);
        s[r] = ok ? ld_scale(scales + n * G + grp) : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < kRowsAhead; ++r) {
        const int64_t n = nb + r * kBwdWarps;
        const float coef = sdy[(n < c1 ? n : c0) - c0] * s[r];
        const uint32_t ww[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[8 * q + j] = fmaf(coef, nibble_float(ww[q], j), acc[8 * q + j]);
      }
    }
    __syncthreads();
  }
  float4 *rw = reinterpret_cast<float4 *>(&red[warp][lane * 32]);
#pragma unroll
  for (int q = 0; q < 8; ++q) rw[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
  __syncthreads();
  for (int c = threadIdx.x; c < kBwdWideTile; c += blockDim.x) {
    float v = 0.0f;
#pragma unroll
    for (int w2 = 0; w2 < kBwdWarps; ++w2) v += red[w2][c];
    const int64_t k = static_cast<int64_t>(tile) * kBwdWideTile + c;
    if (k < K) {
      if (splits == 1)
        store_out(dx, dx_dtype, k, v);
      else
        part[static_cast<int64_t>(split) * K + k] = v;
    }
  }
}

__global__ void __launch_bounds__(256) bwd_x_reduce_kernel(const float *__restrict__ part, void *dx, int dx_dtype,
                                                           int64_t MK, int splits) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= MK) return;
  float v = 0.0f;
  for (int sp = 0; sp < splits; ++sp) v += __ldcg(part + sp * MK + i);
  store_out(dx, dx_dtype, i, v);
}

__global__ void __launch_bounds__(256) bwd_x_plain_kernel(const __nv_bfloat16 *__restrict__ dy,
                                                          const uint8_t *__restrict__ codes,
                                                          const float *__restrict__ scales, void *dx, int dx_dtype,
                                                          int64_t M, int64_t N, int64_t K) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= M * K) return;
  const int64_t m = i / K, k = i % K;
  const int64_t P = (K + 1) / 2, G = (K + 31) / 32;
  float v = 0.0f;
  for (int64_t n = 0; n < N; ++n) {
    const uint32_t byte = codes[n * P + k / 2];
    const int u = static_cast<int>((k & 1) ? (byte >> 4) : (byte & 15u));
    const float wv = __fmul_rn(static_cast<float>(u >= 8 ? u - 16 : u), scales[n * G + k / 32]);
    v = fmaf(__bfloat162float(dy[m * N + n]), wv, v);
  }
  store_out(dx, dx_dtype, i, v);
}

bool bwd_fast(const uint8_t *codes, const float *scales, int64_t K) {
  return K % 8 == 0 && (reinterpret_cast<uintptr_t>(codes) | reinterpret_cast<uintptr_t>(scales)) % 4 == 0;
}

int bwd_tm(int64_t M) { return M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8)); }

// Row splits for the fast kernel: enough CTAs for the whole GPU, at least kBwdMinRows rows
// each. A function of the sizes only (the workspace query must not depend on the device).
bool bwd_wide(int64_t M, int64_t K) { return M == 1 && K % 32 == 0; }

int64_t bwd_splits(int64_t M, int64_t N, int64_t K) {
  const int64_t tiles = bwd_wide(M, K) ? (K + kBwdWideTile - 1) / kBwdWideTile : (K + kBwdTile - 1) / kBwdTile;
  const int64_t chunks = (M + bwd_tm(M) - 1) / bwd_tm(M);
  const int64_t by_gpu = (kBwdTargetCtas + tiles * chunks - 1) / (tiles * chunks);
  const int64_t by_rows = (N + kBwdMinRows - 1) / kBwdMinRows;
  int64_t s = by_gpu < by_rows ? by_gpu : by_rows;
  if (s < 1) s = 1;
  if (s > 65535) s = 65535;
  return s;
}

template <int TM>
cudaError_t launch_tm(const __nv_bfloat16 *dy, const uint8_t *codes, const float *scales, float *part, void *dx,
                      int dx_dtype, int64_t M, int64_t N, int64_t K, int64_t splits, cudaStream_t stream) {
  const int64_t tiles = (K + kBwdTile - 1) / kBwdTile;
  const int64_t chunks = (M + TM - 1) / TM;
  const int64_t rows = (N + splits - 1) / splits;
  if (tiles > 0x7fffffffLL || chunks > 65535) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(splits), static_cast<unsigned>(chunks));
  bwd_x_kernel<TM><<<grid, 32 * kBwdWarps, 0, stream>>>(dy, codes, scales, part, dx, dx_dtype, M, N, K, rows,
                                                        static_cast<int>(splits));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t MK = M * K;
  bwd_x_reduce_kernel<<<static_cast<unsigned>((MK + 255) / 256), 256, 0, stream>>>(part, dx, dx_dtype, MK,
                                                                                  static_cast<int>(splits));
  return cudaGetLastError();
}

}  // namespace

size_t linear_backward_x_workspace(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || K % 8 != 0) return 0;
  const int64_t s = bwd_splits(M, N, K);
  return s > 1 ? static_cast<size_t>(s) * static_cast<size_t>(M) * static_cast<size_t>(K) * sizeof(float) : 0;
}

cudaError_t launch_linear_backward_x(const __nv_bfloat16 *dy, int64_t M, const uint8_t *codes, const float *scales,
                                     int64_t N, int64_t K, void *dx, int dx_dtype, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream) {
  const size_t need = linear_backward_x_workspace(M, N, K);
  const bool chunks_fit = (M + bwd_tm(M) - 1) / bwd_tm(M) <= 65535;  // grid z of the streaming kernel
  if (bwd_fast(codes, scales, K) && chunks_fit && (need == 0 || (workspace != nullptr && workspace_bytes >= need))) {
    const int64_t splits = need == 0 ? 1 : bwd_splits(M, N, K);
    float *part = static_cast<float *>(workspace);
    if (bwd_wide(M, K) && reinterpret_cast<uintptr_t>(codes) % 16 == 0) {
      const int64_t tiles = (K + kBwdWideTile - 1) / kBwdWideTile;
      const int64_t rows = (N + splits - 1) / splits;
      const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(splits), 1u);
      bwd_x_wide_kernel<<<grid, 32 * kBwdWarps, 0, stream>>>(dy, codes, scales, part, dx, dx_dtype, N, K, rows,
                                                             static_cast<int>(splits));
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess || splits == 1) return e;
      bwd_x_reduce_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, stream>>>(part, dx, dx_dtype, K,
                                                                                     static_cast<int>(splits));
      return cudaGetLastError();
    }
    switch (bwd_tm(M)) {
      case 1: return launch_tm<1>(dy, codes, scales, part, dx, dx_dtype, M, N, K, splits, stream);
      case 2: return launch_tm<2>(dy, codes, scales, part, dx, dx_dtype, M, N, K, splits, stream);
      case 4: return launch_tm<4>(dy, codes, scales, part, dx, dx_dtype, M, N, K, splits, stream);
      default: return launch_tm<8>(dy, codes, scales, part, dx, dx_dtype, M, N, K, splits, stream);
    }
  }
  const int64_t MK = M * K;
  if ((MK + 255) / 256 > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_x_plain_kernel<<<static_cast<unsigned>((MK + 255) / 256), 256, 0, stream>>>(dy, codes, scales, dx, dx_dtype,
                                                                                 M, N, K);
  return cudaGetLastError();
}

}  // namespace w4i

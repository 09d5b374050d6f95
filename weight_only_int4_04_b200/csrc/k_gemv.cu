// Decode GEMV on CUDA cores: y[m][n] = sum_k x[m][k] * w[n][k] + b[n] for M <= 4.
//
// The weight stream is the whole cost (0.625 byte per weight), so the kernel is built
// around it:
//   * One CTA owns RB = 8 rows and all of K. Warp w takes the 1024-column slices
//     w, w + nwarps, ...; lane l of a slice owns the 32-column chunk that equals exactly
//     one scale group and 16 code bytes, so every code load is a coalesced 128-bit
//     load (512 contiguous bytes per warp instruction) and every scale load is 128
//     contiguous bytes. All RB rows' loads are issued before any math (16 B x 8 in flight
//     per lane).
//   * Nibbles become bf16x2 pairs with one LOP3 each (the magic-exponent trick: the nibble
//     drops into the mantissa of 128.0, whose ulp is 1) and one exact bf16x2 subtract;
//     the activations are permuted once per chunk with PRMT so their pairs line up.
//   * Products use the sm_100 mixed-precision FMA (bf16 x bf16 + fp32): the product of a
//     bf16 activation and a 4-bit integer is exact, so each step rounds once in fp32.
//     The scale of the group multiplies the fp32 partial (one FFMA per row and group).
//   * Per-lane partials of 8 rows are reduced across the warp with a transposing
//     butterfly (9 shuffles per lane for 8 rows), then across warps through shared memory
//     in a fixed order, so results are deterministic. No global scratch memory.
// Symmetric (signed nibbles, 32-column groups) and asymmetric act-order (unsigned nibbles
// minus a zero point, codes sorted by w4_asym_prepare, x gathered through perm) variants.
#include "w4_dot.cuh"

namespace w4i {

namespace {

constexpr int RB = 8;            // rows per CTA
constexpr int kMaxWarps = 16;    // 1024-column slices handled concurrently per CTA

// Slow per-column fallback for an act-order chunk whose 32 sorted columns span two groups.
template <int MT>
__device__ float dot_chunk_mixed(const LinearParams &p, int64_t n, int64_t col0, const uint4 cw,
                                 const uint32_t (&xp)[MT][16], int m) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
  float acc = 0.0f;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int64_t col = col0 + 8 * t + e;
      if (col >= p.K) continue;
      const int u = static_cast<int>((words[t] >> (4 * e)) & 15u);
      const int64_t g = p.g_idx[p.perm[col]];
      const float w = __fmul_rn(static_cast<float>(u - p.zeros[n * p.n_groups + g]),
                                p.scales[n * p.n_groups + g]);
      // xp pair index for column e of word t: pairs (0,4) (1,5) (2,6) (3,7)
      const uint32_t pair = xp[m][4 * t + (e & 3)];
      const float xv = __uint_as_float((e < 4 ? (pair & 0xFFFFu) : (pair >> 16)) << 16);
      acc = fmaf(xv, w, acc);
    }
  }
  return acc;
}

template <int MT, bool ASYM>
__global__ void __launch_bounds__(kMaxWarps * 32) gemv_kernel(const LinearParams p, int x_vec) {
  __shared__ float red[kMaxWarps][RB][MT];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * RB;
  const int64_t K = p.K, N = p.N, M = p.M;
  const int64_t C = (K + 31) / 32;      // 32-column chunks per row
  const int64_t P = (K + 1) / 2;        // code bytes per row (multiple of 16 here)
  const int64_t SG = ASYM ? p.n_groups : C;  // scale columns per row

  float part[RB][MT];
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) part[r][m] = 0.0f;

  for (int64_t cb = static_cast<int64_t>(warp) * 32; cb < C; cb += static_cast<int64_t>(nwarps) * 32) {
    const int64_t c = cb + lane;
    const bool active = c < C;
    // Issue every weight load of the RB rows first.
    uint4 cw[RB];
    float sc[RB];
    uint32_t zoff[RB];
    int64_t g = 0;
    bool mixed = false;
    if (ASYM && active) {
      const int64_t last = (32 * c + 31 < K) ? 32 * c + 31 : K - 1;
      g = __ldg(p.g_idx + __ldg(p.perm + 32 * c));
      mixed = g != __ldg(p.g_idx + __ldg(p.perm + last));
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const int64_t n = n0 + r;
      const bool ok = active && n < N;
      cw[r] = ok ? ld_stream_v4(p.codes + n * P + 16 * c) : make_uint4(0u, 0u, 0u, 0u);
      if (!ASYM) {
        sc[r] = ok ? __ldg(p.scales + n * SG + c) : 0.0f;
        zoff[r] = 0x43084308u;
      } else {
        sc[r] = ok ? __ldg(p.scales + n * SG + g) : 0.0f;
        const uint32_t z = ok ? static_cast<uint32_t>(static_cast<uint8_t>(__ldg(p.zeros + n * SG + g))) : 0u;
        zoff[r] = (0x4300u | z) * 0x00010001u;
      }
    }
    uint32_t xp[MT][16];
    load_x_chunk<MT>(p.x, M, K, 32 * c, x_vec != 0, ASYM ? p.perm : nullptr, xp);
    if (!active) continue;  // partials stay zero; every lane still reaches the reduction
#pragma unroll
    for (int r = 0; r < RB; ++r) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float acc;
        if (ASYM && mixed) {
          acc = (n0 + r < N) ? dot_chunk_mixed<MT>(p, n0 + r, 32 * c, cw[r], xp, m) : 0.0f;
          part[r][m] += acc;
        } else {
          acc = dot_chunk(cw[r], xp[m], ASYM ? 0x43004300u : 0x43084308u, zoff[r], 0.0f);
          part[r][m] = fmaf(acc, sc[r], part[r][m]);
        }
      }
    }
  }

#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float v[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) v[r] = part[r][m];
    const float s = reduce_rows8(v, lane);
    if ((lane & 3) == 0) red[warp][(lane >> 2) & 7][m] = s;
  }
  __syncthreads();
  if (threadIdx.x < RB * MT) {
    const int r = threadIdx.x / MT, m = threadIdx.x % MT;
    const int64_t n = n0 + r;
    if (n < N && m < M) {
      float v = 0.0f;
      for (int w = 0; w < nwarps; ++w) v += red[w][r][m];
      if (p.bias) v += __ldg(p.bias + n);
      if (p.y_dtype == W4_F32) {
        static_cast<float *>(p.y)[m * N + n] = v;
      } else {
        static_cast<__nv_bfloat16 *>(p.y)[m * N + n] = __float2bfloat16_rn(v);
      }
    }
  }
}

template <int MT>
cudaError_t launch_mt(const LinearParams &p, cudaStream_t stream) {
  const int64_t C = (p.K + 31) / 32;
  int64_t nwarps = (C + 31) / 32;
  if (nwarps > kMaxWarps) nwarps = kMaxWarps;
  const int64_t blocks = (p.N + RB - 1) / RB;
  const int x_vec = (p.K % 8 == 0) && (reinterpret_cast<uintptr_t>(p.x) % 16 == 0);
  if (p.asym) {
    gemv_kernel<MT, true><<<static_cast<unsigned>(blocks), static_cast<unsigned>(nwarps * 32), 0, stream>>>(p, x_vec);
  } else {
    gemv_kernel<MT, false><<<static_cast<unsigned>(blocks), static_cast<unsigned>(nwarps * 32), 0, stream>>>(p, x_vec);
  }
  return cudaGetLastError();
}

}  // namespace

bool gemv_supports(const LinearParams &p) {
  const int64_t P = (p.K + 1) / 2;
  if (p.M < 1 || p.M > 4) return false;
  if (P % 16 != 0) return false;
  if (reinterpret_cast<uintptr_t>(p.codes) % 16 != 0) return false;
  if (p.asym && p.perm == nullptr) return false;
  if ((p.N + RB - 1) / RB > 0x7fffffffLL) return false;
  return true;
}

cudaError_t launch_gemv(const LinearParams &p, cudaStream_t stream) {
  if (!gemv_supports(p)) return cudaErrorNotSupported;
  switch (p.M) {
    case 1: return launch_mt<1>(p, stream);
    case 2: return launch_mt<2>(p, stream);
    case 3: return launch_mt<3>(p, stream);
    default: return launch_mt<4>(p, stream);
  }
}

}  // namespace w4i

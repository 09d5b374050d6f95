// Standalone element-wise kernels: RTN quantize + pack, dequantize, content validation and
// the act-order column reorder. All of them are HBM-bound streams: coalesced loads and
// stores, no shared memory, grids sized in multiples of the SM count.
#include <cfloat>

#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int kThreads = 256;

int sm_count() {
  static int counts[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    counts[dev] = n;
  }
  return counts[dev];
}

int grid_for(int64_t work_items, int items_per_block) {
  // Enough blocks to cover the work, capped at a multiple of 148 SMs x 8 resident blocks;
  // the kernels are grid-stride loops.
  int64_t blocks = (work_items + items_per_block - 1) / items_per_block;
  const int64_t cap = 148LL * 8 * 4;
  if (blocks > cap) blocks = cap;
  return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// ---------------------------------------------------------------------------
// RTN quantize + pack (page "loopq/packed_weight.py", pack_weight; rounding and clip of
// page "gemma/peft/_quantization_utils.py", uniform_quantize).
// Eight lanes cooperate on one group of 32 columns, four columns per lane, so one warp
// instruction reads four consecutive groups (512 contiguous bytes of W). A lane's (row,
// group) advances by a fixed step per trip of the grid-stride loop (no division inside it).
//
// The code is rne(fl32(w / s)) clamped to [-7, 7], s = max(fl32(amax / 7), 2^-126), formed
// without a division per element: |w / s| <= 7 / (1 - 2^-24) because |w| <= amax and
// s >= amax / 7 rounded down by at most half an ulp (or s = 2^-126 > amax / 7), so the clamp
// never acts. y = rcp.approx(s) is within one ulp of 1 / s (the PTX ISA's bound for
// rcp.approx.f32; s and 1 / s are normal), so x = fl32(w * y) is within 1.51 * 2^-21 of
// w / s and fl32(w / s) within 2^-22 of it (|w / s| < 8): both round to the same integer
// unless x is within 2^-20 of a half-integer; a lane whose four values come within 2^-18 of
// one takes the IEEE quotients instead. Adding 1.5 * 2^23 rounds to an integer, half to even,
// and leaves its two's-complement nibble in the low bits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t rtn_nibble(float w, float y, bool &near) {
  const float x = __fmul_rn(w, y);
  const float xm = __fadd_rn(x, 12582912.0f);
  near |= fabsf(__fsub_rn(x, __fsub_rn(xm, 12582912.0f))) > 0.5f - 0x1p-18f;
  return __float_as_uint(xm) & 15u;
}

__device__ __forceinline__ float rcp_approx(float s) {
  float y;
  asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(s));
  return y;
}

// max that returns NaN when either input is NaN, so one test of the amax covers the values
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ uint32_t rtn_nibble_exact(float w, float s) {
  return __float_as_uint(__fadd_rn(__fdiv_rn(w, s), 12582912.0f)) & 15u;
}

__global__ void __launch_bounds__(kThreads) quantize_rtn_kernel(const float *__restrict__ W,
                                                                int64_t N, int64_t K,
                                                                uint8_t *__restrict__ codes,
                                                                float *__restrict__ scales,
                                                                int32_t *__restrict__ status,
                                                                int vec_ok) {
  const int64_t G = (K + 31) / 32;
  const int64_t P = (K + 1) / 2;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int64_t tasks = N * G;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t step = ((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) * 4;  // tasks per trip
  const int64_t dn = step / G, dg = step % G;
  // this lane's task t = n * G + g (past the end on the last trips: then unused)
  int64_t t = warp_id * 4 + (lane >> 3);
  int64_t n = t / G, g = t % G;
  bool bad = false;
  // A warp owns four consecutive tasks per trip; the trip count is warp-uniform so every
  // lane reaches the shuffles below (lanes past the end work on zeros and store nothing).
  for (int64_t wb = warp_id * 4; wb < tasks; wb += step) {
    const bool active = t < tasks;
    const int64_t na = active ? n : 0, ga = active ? g : 0;
    const int64_t c0 = 32 * ga + 4 * sub;
    const float *row = W + na * K;
    float w[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (!active) {
    } else if (vec_ok && c0 + 3 < K) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(row + c0));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = (c0 + i < K) ? row[c0 + i] : 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = max_nan(amax, fabsf(w[i]));
    bad |= !(amax <= FLT_MAX);  // a NaN or an infinity among this lane's values
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    // s = max(fl32(amax / 7), FLT_MIN): IEEE round-to-nearest divide.
    const float s = fmaxf(__fdiv_rn(amax, 7.0f), FLT_MIN);
    const float y = rcp_approx(s);
    bool near = false;
    uint32_t nib[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) nib[i] = rtn_nibble(w[i], y, near);
    if (near) {  // rare: a value close to a half-integer takes the exact quotient
#pragma unroll
      for (int i = 0; i < 4; ++i) nib[i] = rtn_nibble_exact(w[i], s);
    }
    // columns past K: pad nibble 0
    const int64_t left = K - c0;
    const uint32_t colmask = left >= 4 ? 0xFFFFu : (left <= 0 ? 0u : (1u << (4 * left)) - 1u);
    const uint32_t w16 = (nib[0] | (nib[1] << 4) | (nib[2] << 8) | (nib[3] << 12)) & colmask;
    const uint8_t b0 = static_cast<uint8_t>(w16);
    const uint8_t b1 = static_cast<uint8_t>(w16 >> 8);
    // advance this lane's task by one trip: t + step = (n + dn) G + (g + dg), one carry at most
    t += step;
    n += dn;
    g += dg;
    if (g >= G) {
      g -= G;
      ++n;
    }
    if (!active) continue;
    uint8_t *crow = codes + na * P;
    const int64_t j = c0 / 2;
    if (j < P) crow[j] = b0;
    if (j + 1 < P) crow[j + 1] = b1;
    if (sub == 0) scales[na * G + ga] = s;
  }
  if (bad) *status = W4_ERR_NONFINITE;
}

// ---------------------------------------------------------------------------
// Dequantize (page "loopq/packed_weight.py", _dequantize_validated): fp32 value * scale,
// then round-to-nearest-even into the output dtype (f64: exact widening).
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T convert_out(float v);
template <>
__device__ __forceinline__ __nv_bfloat16 convert_out<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ __half convert_out<__half>(float v) {
  return __float2half_rn(v);
}
template <>
__device__ __forceinline__ float convert_out<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ double convert_out<double>(float v) {
  return static_cast<double>(v);
}

__device__ __forceinline__ float signed_nibble(uint32_t byte, int hi) {
  const int n = hi ? static_cast<int>(byte >> 4) : static_cast<int>(byte & 15u);
  return static_cast<float>(n >= 8 ? n - 16 : n);
}

// Vector path: K % 8 == 0, so a row holds whole 4-byte code words and each word expands to
// 8 consecutive outputs (16 bytes for bf16/f16). One thread per code word.
template <typename T>
__global__ void __launch_bounds__(kThreads) dequant_vec_kernel(const uint8_t *__restrict__ codes,
                                                               const float *__restrict__ scales,
                                                               int64_t N, int64_t K,
                                                               T *__restrict__ out) {
  const int64_t words_per_row = K / 8;
  const int64_t G = (K + 31) / 32;
  const int64_t total = N * words_per_row;
  const uint32_t *cw = reinterpret_cast<const uint32_t *>(codes);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t n, q;
    if (total <= 0xffffffffLL) {  // 32-bit divide when the index fits (the common case)
      const uint32_t i32 = static_cast<uint32_t>(i), wpr = static_cast<uint32_t>(words_per_row);
      n = i32 / wpr;
      q = i32 - static_cast<uint32_t>(n) * wpr;
    } else {
      n = i / words_per_row;
      q = i % words_per_row;
    }
    const uint32_t w = __ldcs(cw + i);
    const float s = __ldg(scales + n * G + q / 4);
    __align__(16) T v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      // nibble n -> the float 2^23 + (n ^ 8), minus 2^23 + 8: the exact signed code
      const float val = __uint_as_float(lop3_and_xor(w >> (4 * e), 0xFu, 0x4B000008u)) - 8388616.0f;
      v[e] = convert_out<T>(__fmul_rn(val, s));
    }
    T *dst = out + n * K + q * 8;
    constexpr int kVecs = (8 * sizeof(T)) / 16;
#pragma unroll
    for (int j = 0; j < kVecs; ++j) {
      __stcs(reinterpret_cast<uint4 *>(dst) + j, reinterpret_cast<const uint4 *>(v)[j]);
    }
  }
}

// Generic path: any K (odd widths, partial groups, unaligned rows). One thread per code byte.
template <typename T>
__global__ void __launch_bounds__(kThreads) dequant_generic_kernel(const uint8_t *__restrict__ codes,
                                                                   const float *__restrict__ scales,
                                                                   int64_t N, int64_t K,
                                                                   T *__restrict__ out) {
  const int64_t P = (K + 1) / 2;
  const int64_t G = (K + 31) / 32;
  const int64_t total = N * P;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / P, j = i % P;
    const uint32_t b = codes[i];
    const int64_t k0 = 2 * j;
    const float s = scales[n * G + k0 / 32];
    out[n * K + k0] = convert_out<T>(__fmul_rn(signed_nibble(b, 0), s));
    if (k0 + 1 < K) out[n * K + k0 + 1] = convert_out<T>(__fmul_rn(signed_nibble(b, 1), s));
  }
}

// Tile path for widths that are not a multiple of 8 (rows of up to kTileCodeBytes of codes):
// a CTA owns rows r0 .. r0 + R - 1, whose output is the contiguous flat range
// [r0 K, (r0 + R) K). Their codes (a contiguous byte range) and scales are copied into
// shared memory with 16-byte loads; then each thread computes 16-byte aligned chunks of the
// flat output range straight from shared memory (a chunk may span a row end) and stores
// them whole; the elements before the first and after the last chunk boundary are stored
// singly.
constexpr int kTileCodeBytes = 8 * 1024;

template <typename T>
__global__ void __launch_bounds__(kThreads) dequant_tile_kernel(const uint8_t *__restrict__ codes,
                                                                const float *__restrict__ scales,
                                                                int64_t N, int64_t K, int rows_per_tile,
                                                                T *__restrict__ out) {
  constexpr int kV = 16 / sizeof(T);  // elements per 16-byte chunk
  extern __shared__ __align__(16) uint8_t dq_smem[];
  const int64_t P = (K + 1) / 2;
  const int64_t G = (K + 31) / 32;
  const int64_t total_code_bytes = N * P;
  const int code_cap = static_cast<int>((rows_per_tile * P + 31) / 16 * 16);  // bytes of the code tile
  uint8_t *ct = dq_smem;                                                       // codes, from a 16-byte boundary
  float *st = reinterpret_cast<float *>(dq_smem + code_cap);                  // scales [R][G]
  for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_tile; r0 < N;
       r0 += static_cast<int64_t>(gridDim.x) * rows_per_tile) {
    const int rows = static_cast<int>((N - r0) < rows_per_tile ? (N - r0) : rows_per_tile);
    // codes: bytes [b0, b1) of the flat code array, fetched as aligned 16-byte words from
    // the word holding b0 (bytes before b0 land in ct[0 .. lead))
    const int64_t b0 = r0 * P, b1 = b0 + rows * P;
    const int64_t w0 = b0 / 16, w1 = (b1 + 15) / 16;
    const int lead = static_cast<int>(b0 - 16 * w0);
    const uint4 *cw = reinterpret_cast<const uint4 *>(codes);
    for (int64_t wi = w0 + threadIdx.x; wi < w1; wi += blockDim.x) {
      uint4 v;
      if (16 * (wi + 1) <= total_code_bytes) {
        v = __ldcs(cw + wi);
      } else {  // the array's last word, partly past its end
        __align__(16) uint8_t tmp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) tmp[i] = (16 * wi + i < total_code_bytes) ? codes[16 * wi + i] : 0;
        v = *reinterpret_cast<const uint4 *>(tmp);
      }
      reinterpret_cast<uint4 *>(ct)[wi - w0] = v;
    }
    for (int64_t i = threadIdx.x; i < rows * G; i += blockDim.x) st[i] = __ldg(scales + r0 * G + i);
    __syncthreads();
    const int64_t f0 = r0 * K, f1 = f0 + rows * K;  // flat output range
    auto value = [&](int64_t e) -> T {               // e: element index inside the tile
      const int64_t i = e / K, k = e - i * K;
      const uint32_t b = ct[lead + i * P + (k >> 1)];
      return convert_out<T>(__fmul_rn(signed_nibble(b, static_cast<int>(k & 1)), st[i * G + (k >> 5)]));
    };
    const int64_t a0 = (f0 + kV - 1) / kV * kV, a1 = f1 / kV * kV;  // chunk boundaries inside
    if (a1 > a0) {
      const uint32_t K32 = static_cast<uint32_t>(K), P32 = static_cast<uint32_t>(P), G32 = static_cast<uint32_t>(G);
      for (int64_t c = threadIdx.x; c < (a1 - a0) / kV; c += blockDim.x) {
        const uint32_t e0 = static_cast<uint32_t>(a0 - f0 + c * kV);  // below R * K < 2^31
        const uint32_t i = e0 / K32, k0 = e0 - i * K32;
        __align__(16) T v[kV];
        if (k0 + kV <= K32) {
          // the chunk lies in one row: its kV / 2 + 1 code bytes from one 8-byte window of
          // shared memory, shifted so that bit 0 holds column k0
          const uint32_t b = lead + i * P32 + (k0 >> 1);
          const uint32_t* wp = reinterpret_cast<const uint32_t *>(ct + (b & ~3u));
          uint64_t win = (static_cast<uint64_t>(wp[1]) << 32) | wp[0];
          win >>= 8 * (b & 3u) + 4 * (k0 & 1u);
          const float *srow = st + i * G32;
          const float s0 = srow[k0 >> 5], s1 = srow[(k0 + kV - 1) >> 5];
#pragma unroll
          for (int u = 0; u < kV; ++u) {
            // nibble n of column k0 + u -> the float 2^23 + (n ^ 8), minus 2^23 + 8: exact q
            const uint32_t bits = lop3_and_xor(static_cast<uint32_t>(win >> (4 * u)), 0xFu, 0x4B000008u);
            const float q = __uint_as_float(bits) - 8388616.0f;
            const float sc = ((k0 + u) >> 5) != (k0 >> 5) ? s1 : s0;
            v[u] = convert_out<T>(__fmul_rn(q, sc));
          }
        } else {
          int64_t ii = i, k = k0;
#pragma unroll
          for (int u = 0; u < kV; ++u) {
            const uint32_t bb = ct[lead + ii * P + (k >> 1)];
            v[u] = convert_out<T>(__fmul_rn(signed_nibble(bb, static_cast<int>(k & 1)), st[ii * G + (k >> 5)]));
            if (++k == K) {
              k = 0;
              ++ii;
            }
          }
        }
        __stcs(reinterpret_cast<uint4 *>(out + f0 + e0), *reinterpret_cast<const uint4 *>(v));
      }
      if (threadIdx.x < a0 - f0) out[f0 + threadIdx.x] = value(threadIdx.x);
      if (threadIdx.x < f1 - a1) out[a1 + threadIdx.x] = value(a1 - f0 + threadIdx.x);
    } else {
      for (int64_t e = threadIdx.x; e < f1 - f0; e += blockDim.x) out[f0 + e] = value(e);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Content validation (page "loopq/packed_weight.py", validate; asymmetric extras).
// Each thread ORs the rules it saw broken into a block-shared word; one atomic per block.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) validate_kernel(const uint8_t *__restrict__ codes,
                                                            const float *__restrict__ scales,
                                                            const int8_t *__restrict__ zeros,
                                                            const int32_t *__restrict__ g_idx,
                                                            int64_t N, int64_t K, int64_t n_scale_cols,
                                                            int64_t n_groups, int check_v1,
                                                            uint32_t *__restrict__ flags) {
  __shared__ uint32_t block_flags;
  if (threadIdx.x == 0) block_flags = 0;
  __syncthreads();
  uint32_t f = 0;
  const int64_t P = (K + 1) / 2;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < N * n_scale_cols; i += step) {
    const float s = scales[i];
    if (!(isfinite(s) && s > 0.0f)) f |= FLAG_SCALE;
    if (zeros != nullptr) {
      const int z = zeros[i];
      if (z < 0 || z > 15) f |= FLAG_ZERO;
    }
  }
  if (check_v1) {
    for (int64_t i = tid; i < N * P; i += step) {
      const uint32_t b = codes[i];
      if ((b & 15u) == 8u || (b >> 4) == 8u) f |= FLAG_RESERVED;
    }
  }
  if (K & 1) {
    for (int64_t n = tid; n < N; n += step) {
      if (codes[n * P + P - 1] >> 4) f |= FLAG_HIGH_NIBBLE;
    }
  }
  if (g_idx != nullptr) {
    for (int64_t k = tid; k < K; k += step) {
      const int32_t g = g_idx[k];
      if (g < 0 || g >= n_groups) f |= FLAG_GIDX;
    }
  }
  if (f) atomicOr(&block_flags, f);
  __syncthreads();
  if (threadIdx.x == 0 && block_flags) atomicOr(flags, block_flags);
}

// Column reorder for act-order weights: column j of the output is column perm[j] of the
// input (unsigned nibbles), one thread per output byte; the pad nibble stays zero.
__global__ void __launch_bounds__(kThreads) reorder_codes_kernel(const uint8_t *__restrict__ in,
                                                                 const int32_t *__restrict__ perm,
                                                                 int64_t N, int64_t K,
                                                                 uint8_t *__restrict__ out) {
  const int64_t P = (K + 1) / 2;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N * P;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / P, j = i % P;
    const uint8_t *row = in + n * P;
    uint32_t v = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t col = 2 * j + h;
      if (col < K) {
        const int64_t src = perm[col];
        const uint32_t b = row[src >> 1];
        v |= ((src & 1) ? (b >> 4) : (b & 15u)) << (4 * h);
      }
    }
    out[i] = static_cast<uint8_t>(v);
  }
}

}  // namespace

cudaError_t launch_quantize_rtn(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                int32_t *status, cudaStream_t stream) {
  const int64_t groups = N * ((K + 31) / 32);
  const int vec_ok = (K % 4 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
  quantize_rtn_kernel<<<grid_for(groups, kThreads / 8), kThreads, 0, stream>>>(W, N, K, codes, scales,
                                                                              status, vec_ok);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t dequant_typed(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                                 void *out, cudaStream_t stream) {
  T *o = static_cast<T *>(out);
  const bool vec = (K % 8 == 0) && (reinterpret_cast<uintptr_t>(codes) % 4 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) % 16 == 0);
  if (vec) {
    dequant_vec_kernel<T><<<grid_for(N * (K / 8), kThreads), kThreads, 0, stream>>>(codes, scales, N, K, o);
  } else if (reinterpret_cast<uintptr_t>(out) % 16 == 0 && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
             (K + 1) / 2 <= kTileCodeBytes) {
    // rows per tile: at most kTileCodeBytes of codes, and few enough that the tiles fill
    // one wave of resident blocks
    const int64_t P = (K + 1) / 2, G = (K + 31) / 32;
    int64_t rows = kTileCodeBytes / P;
    const int64_t wave = static_cast<int64_t>(sm_count()) * 8;
    const int64_t spread = (N + wave - 1) / wave;
    if (spread < rows) rows = spread;
    if (rows < 1) rows = 1;
    const int64_t tiles = (N + rows - 1) / rows;
    const int blocks = static_cast<int>(tiles < wave ? tiles : wave);
    // + 16: the 8-byte code window of the last chunk may read a few bytes past the tile
    const int smem = static_cast<int>((rows * P + 31) / 16 * 16 + rows * G * 4 + 16);
    dequant_tile_kernel<T><<<blocks, kThreads, smem, stream>>>(codes, scales, N, K, static_cast<int>(rows), o);
  } else {
    dequant_generic_kernel<T><<<grid_for(N * ((K + 1) / 2), kThreads), kThreads, 0, stream>>>(codes, scales,
                                                                                           N, K, o);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                              int out_dtype, void *out, cudaStream_t stream) {
  switch (out_dtype) {
    case W4_BF16: return dequant_typed<__nv_bfloat16>(codes, scales, N, K, out, stream);
    case W4_F16: return dequant_typed<__half>(codes, scales, N, K, out, stream);
    case W4_F32: return dequant_typed<float>(codes, scales, N, K, out, stream);
    case W4_F64: return dequant_typed<double>(codes, scales, N, K, out, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_validate(const uint8_t *codes, const float *scales, const int8_t *zeros,
                            const int32_t *g_idx, int64_t N, int64_t K, int64_t n_groups,
                            int format_version, int asym, uint32_t *flags, cudaStream_t stream) {
  const int64_t scale_cols = asym ? n_groups : (K + 31) / 32;
  const int64_t work = N * ((K + 1) / 2);
  validate_kernel<<<grid_for(work, kThreads * 4), kThreads, 0, stream>>>(
      codes, scales, asym ? zeros : nullptr, asym ? g_idx : nullptr, N, K, scale_cols, n_groups,
      (!asym && format_version == 1) ? 1 : 0, flags);
  return cudaGetLastError();
}

cudaError_t launch_reorder_codes(const uint8_t *codes_in, const int32_t *perm, int64_t N, int64_t K,
                                 uint8_t *codes_out, cudaStream_t stream) {
  reorder_codes_kernel<<<grid_for(N * ((K + 1) / 2), kThreads), kThreads, 0, stream>>>(codes_in, perm, N,
                                                                                      K, codes_out);
  return cudaGetLastError();
}

}  // namespace w4i

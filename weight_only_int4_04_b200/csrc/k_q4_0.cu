// GGUF Q4_0 block format: dequantization and the linear y = x . dequant(W)^T (+ b).
//
// Page "max/python/max/graph/quantization.py" (Modular MAX), QuantizationEncoding.Q4_0 and
// its block parameters: 32 elements per block in 2 + 32/2 = 18 bytes, the scale d then the
// 4-bit codes. Readings (not on the page): d is binary16, little-endian, in the block's first
// two bytes; element j (j < 16) is the low nibble of code byte j and element j + 16 its high
// nibble; the value is d * (code - 8) (exact in fp32). A weight [N, K] (K a multiple of 32)
// is uint8 [N, K/32, 18], a row's blocks consecutive, rows consecutive.
//
// Kernels:
//   * q4_0_gemv_tma_kernel (M = 1, K a multiple of 256, 16-byte aligned blocks and x): the
//     decode GEMV. Two CTAs per SM, each a balanced run of 16-row blocks. One producer
//     thread fills a ring of 18 KB stages, each one 3-D TMA box of 8 k-tiles x 16 rows x
//     144 bytes (8 blocks per row per k-tile; row strides of K/32 * 18 bytes are multiples
//     of 16 when K is a multiple of 256), L2 evict-first (weights are read once). Eight
//     consumer warps take one k-tile each. Per block a lane reads, for rows g and g + 8, the
//     two code bytes of columns 2t, 2t + 1 and of 2t + 8, 2t + 9 (two 16-bit shared loads,
//     the 18-byte blocks are only 2-byte aligned), PRMT spreads each byte pair to the two
//     halves of a register, LOP3 drops the low / high nibbles into the mantissa of the bf16
//     128.0 and one exact bf16x2 subtract of 136 leaves c - 8: the A fragments of two
//     mma.sync m16n8k16 (low nibbles: block columns 0-15, high nibbles: 16-31), x broadcast
//     in every MMA column as the B fragment. The block's fp32 sum is scaled by its d in one
//     FFMA per accumulator. x is staged once per CTA in fragment order. Per row block the
//     warps' sums meet in shared memory in a fixed order (deterministic). Programmatic
//     dependent launch as the group-32 decode GEMV: weights may stream before the previous
//     kernel of the stream ends (w4_set_weight_prefetch), x and y are touched after it.
//     Every wait is bounded (w4_sync.cuh).
//   * q4_0_linear_plain_kernel: any M and K (a multiple of 32), one warp per (row, 4 tokens),
//     lanes striding over blocks, exact fp32 weights, fp32 accumulation: the floor.
//   * q4_0_dequant_kernel: one thread per block, 32 outputs.
//   * q4_0_to_group32_kernel: one thread per block, the block re-laid out as a group of the
//     packed group-32 format (signed codes c - 8, the scale widened to fp32), once per weight:
//     every group-32 entry point then reads the same dequantized weights.
#include <cuda.h>

#include <mutex>

#include "w4_mma.cuh"
#include "w4_tc.cuh"
#include "w4_tmap.h"

namespace w4i {

namespace {

constexpr int kQBlockBytes = 18;
constexpr int kQTileBlocks = 8;                               // blocks per row in one k-tile
constexpr int kQTileBytes = kQTileBlocks * kQBlockBytes;      // 144 bytes = 256 columns
constexpr int kQRows = 16;                                    // rows of a row block (m16 tile)
constexpr int kQWarps = 8;                                    // consumer warps = k-tiles per stage
constexpr int kQStageBytes = kQWarps * kQRows * kQTileBytes;  // 18432
constexpr int kQStages = 3;
constexpr int kQBarBytes = (2 * kQStages) * 8 + 16;
constexpr int kQAlign = 128;
constexpr int kQXBatch = 4;  // x fragment items in flight per consumer thread

struct Q40Params {
  const __nv_bfloat16 *x;
  const float *bias;
  void *y;
  int64_t N, K;
  int rb_q, rb_r;  // CTA c owns rb_q + (c < rb_r) row blocks from c * rb_q + min(c, rb_r)
  int KT;          // 256-column k-tiles per row
  int SPR;         // stages per row block
  int y_dtype;
  int prefetch;
};

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// Byte pair (b0, b1) in the low 16 bits of `p` -> bf16x2 (lo(b0) - 8, lo(b1) - 8) and, through
// `hi`, (hi(b0) - 8, hi(b1) - 8): PRMT puts b0 in byte 0 and b1 in byte 2 (zeros elsewhere).
__device__ __forceinline__ void q4_0_pair(uint32_t spread, uint32_t &lo, uint32_t &hi) {
  lo = bf16x2_sub(nib_pair_bf16(spread, 0x43004300u), 0x43084308u);
  hi = bf16x2_sub(nib_pair_bf16(spread >> 4, 0x43004300u), 0x43084308u);
}

__global__ void __launch_bounds__(32 * (kQWarps + 1), 2)
    q4_0_gemv_tma_kernel(const __grid_constant__ CUtensorMap tm_blocks, const Q40Params p, int32_t *err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + kQAlign - 1u) & ~static_cast<uint32_t>(kQAlign - 1)) - raw);
  uint8_t *xs = smem + kQStages * kQStageBytes;            // x in fragment order, K * 2 bytes
  float *red = reinterpret_cast<float *>(xs + p.K * 2);    // [2][warp][16 rows]
  uint64_t *full = reinterpret_cast<uint64_t *>(red + 2 * kQWarps * kQRows);
  uint64_t *empty = full + kQStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kQStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = static_cast<int>(blockIdx.x);
  const int64_t rb_begin = static_cast<int64_t>(cta) * p.rb_q + (cta < p.rb_r ? cta : p.rb_r);
  const int total = (p.rb_q + (cta < p.rb_r ? 1 : 0)) * p.SPR;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kQWarps);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  grid_launch_dependents();

  if (warp == kQWarps) {
    // ---- producer: one thread issues every stage box of the CTA's row blocks ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int slot = 0, kc = 0;
      uint32_t phase = 0;
      int32_t row = static_cast<int32_t>(rb_begin * kQRows);
      if (!p.prefetch) grid_dependency_wait();  // the blocks may come from the previous kernel
      int issued = 0;
      for (int i = 0; i < total; ++i) {
        if (!mbar_wait(&empty[slot], phase ^ 1u, abort_flag, err)) break;
        // whole-stage box; k-tiles past the row end read as zeros (and count as bytes)
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(kQStageBytes));
        tma_load_3d_hint(smem + slot * kQStageBytes, &tm_blocks, 0, row, kc * kQWarps, &full[slot], pol);
        issued = i + 1;
        if (++kc == p.SPR) {
          kc = 0;
          row += kQRows;
        }
        if (++slot == kQStages) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // the copies issued land before the CTA may exit (see w4_sync.cuh, abort path)
      for (int i = issued - kQStages < 0 ? 0 : issued - kQStages; i < issued; ++i)
        mbar_drain(&full[i % kQStages], static_cast<uint32_t>(i / kQStages) & 1u, err);
    }
    return;
  }

  // ---- consumers: x -> fragment order once the previous kernel has finished. Item (b, t)
  // of block b holds the column pairs t, t + 4, t + 8, t + 12 of the block (pair = 2
  // consecutive columns): b0 / b1 of the low-nibble MMA, then b0 / b1 of the high one. ----
  grid_dependency_wait();
  {
    const uint32_t *x32 = reinterpret_cast<const uint32_t *>(p.x);
    uint4 *xf = reinterpret_cast<uint4 *>(xs);
    const int items = static_cast<int>(p.K / 8);
    for (int base = static_cast<int>(threadIdx.x); base < items; base += kQXBatch * 32 * kQWarps) {
      uint4 v[kQXBatch];
#pragma unroll
      for (int k = 0; k < kQXBatch; ++k) {
        const int i = base + k * 32 * kQWarps;
        if (i < items) {
          const int64_t q = 16 * static_cast<int64_t>(i >> 2) + (i & 3);
          v[k].x = __ldcg(x32 + q);
          v[k].y = __ldcg(x32 + q + 4);
          v[k].z = __ldcg(x32 + q + 8);
          v[k].w = __ldcg(x32 + q + 12);
        }
      }
#pragma unroll
      for (int k = 0; k < kQXBatch; ++k) {
        const int i = base + k * 32 * kQWarps;
        if (i < items) xf[i] = v[k];
      }
    }
  }
  named_barrier_sync(1, 32 * kQWarps);

  const int g = lane >> 2, t = lane & 3;
  const uint32_t stages0 = smem_u32(smem);
  // this lane's offsets inside a k-tile: rows g and g + 8, code bytes 2t and 2t + 8 of a block
  const uint32_t off_g = static_cast<uint32_t>(g * kQTileBytes), off_h = off_g + 8 * kQTileBytes;
  const uint32_t cA = static_cast<uint32_t>(2 + 2 * t), cB = cA + 8;
  const uint4 *xrow = reinterpret_cast<const uint4 *>(xs) + t;

  float acc0 = 0.0f, acc2 = 0.0f;
  int buf = 0, slot = 0, kc = 0, rbl = 0;
  uint32_t phase = 0;
  int64_t row0 = rb_begin * kQRows;
  for (int i = 0; i < total; ++i) {
    mbar_wait(&full[slot], phase, abort_flag, err);
    const int kt = kc * kQWarps + warp;
    if (kt < p.KT) {
      const uint32_t tb = stages0 + static_cast<uint32_t>(slot * kQStageBytes + warp * kQRows * kQTileBytes);
#pragma unroll
      for (int b = 0; b < kQTileBlocks; ++b) {
        const uint32_t bg = tb + off_g + static_cast<uint32_t>(b * kQBlockBytes);
        const uint32_t bh = tb + off_h + static_cast<uint32_t>(b * kQBlockBytes);
        const float sg = half_bits_to_float(lds_u16(bg));
        const float sh = half_bits_to_float(lds_u16(bh));
        const uint32_t ga = lds_u16(bg + cA), gb = lds_u16(bg + cB);
        const uint32_t ha = lds_u16(bh + cA), hb = lds_u16(bh + cB);
        // A fragments: a0 / a2 = row g (columns 2t, 2t+1 / 2t+8, 2t+9), a1 / a3 = row g + 8;
        // the low nibbles feed the MMA of block columns 0-15, the high ones 16-31.
        uint32_t g0l, g0h, g2l, g2h, h0l, h0h, h2l, h2h;
        q4_0_pair(prmt(ga, 0u, 0x5140u), g0l, g0h);
        q4_0_pair(prmt(gb, 0u, 0x5140u), g2l, g2h);
        q4_0_pair(prmt(ha, 0u, 0x5140u), h0l, h0h);
        q4_0_pair(prmt(hb, 0u, 0x5140u), h2l, h2h);
        const uint4 xv = xrow[(kt * kQTileBlocks + b) * 4];
        float d[4];
        mma_first(d, g0l, h0l, g2l, h2l, xv.x, xv.y);
        mma_next(d, g0h, h0h, g2h, h2h, xv.z, xv.w);
        acc0 = fmaf(d[0], sg, acc0);
        acc2 = fmaf(d[2], sh, acc2);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == kQStages) {
      slot = 0;
      phase ^= 1u;
    }
    if (++kc == p.SPR) {
      // row block complete: the warps' sums meet in shared memory, added in a fixed order
      kc = 0;
      float *r = red + buf * kQWarps * kQRows;
      if (t == 0) {
        r[warp * kQRows + g] = acc0;
        r[warp * kQRows + g + 8] = acc2;
      }
      named_barrier_sync(1, 32 * kQWarps);
      if (warp == (rbl & (kQWarps - 1)) && lane < kQRows) {
        const int64_t n = row0 + lane;
        if (n < p.N) {
          float v = 0.0f;
#pragma unroll
          for (int w2 = 0; w2 < kQWarps; ++w2) v += r[w2 * kQRows + lane];
          if (p.bias) v += __ldcg(p.bias + n);
          if (p.y_dtype == W4_F32)
            static_cast<float *>(p.y)[n] = v;
          else
            static_cast<__nv_bfloat16 *>(p.y)[n] = __float2bfloat16_rn(v);
        }
      }
      acc0 = acc2 = 0.0f;
      buf ^= 1;  // the next block writes the other buffer; two barriers apart from this read
      row0 += kQRows;
      ++rbl;
    }
  }
}

// One warp per (row n, up to 4 tokens starting at m0); lane l takes blocks l, l + 32, ...
constexpr int kPlainTok = 4;

__global__ void __launch_bounds__(256) q4_0_linear_plain_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                const uint8_t *__restrict__ blocks,
                                                                const float *__restrict__ bias, void *y,
                                                                int64_t M, int64_t N, int64_t K, int y_dtype) {
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n = warp_id % N, m0 = (warp_id / N) * kPlainTok;
  if (m0 >= M) return;
  const int64_t G = K / 32;
  const uint8_t *rowp = blocks + n * G * kQBlockBytes;
  float acc[kPlainTok] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t gb = lane; gb < G; gb += 32) {
    const uint8_t *bp = rowp + gb * kQBlockBytes;
    const float d = half_bits_to_float(static_cast<uint32_t>(bp[0]) | (static_cast<uint32_t>(bp[1]) << 8));
    for (int j = 0; j < 16; ++j) {
      const uint32_t byte = bp[2 + j];
      const float w_lo = d * static_cast<float>(static_cast<int>(byte & 15u) - 8);  // column 32gb + j
      const float w_hi = d * static_cast<float>(static_cast<int>(byte >> 4) - 8);   // column 32gb + j + 16
#pragma unroll
      for (int mm = 0; mm < kPlainTok; ++mm) {
        const int64_t m = m0 + mm;
        if (m < M) {
          const __nv_bfloat16 *xr = x + m * K + 32 * gb;
          acc[mm] = fmaf(__bfloat162float(xr[j]), w_lo, acc[mm]);
          acc[mm] = fmaf(__bfloat162float(xr[j + 16]), w_hi, acc[mm]);
        }
      }
    }
  }
#pragma unroll
  for (int mm = 0; mm < kPlainTok; ++mm) {
    float v = acc[mm];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
    const int64_t m = m0 + mm;
    if (lane == 0 && m < M) {
      if (bias) v += bias[n];
      if (y_dtype == W4_F32)
        static_cast<float *>(y)[m * N + n] = v;
      else
        static_cast<__nv_bfloat16 *>(y)[m * N + n] = __float2bfloat16_rn(v);
    }
  }
}

template <typename T>
__device__ __forceinline__ T q4_0_convert(float v);
template <>
__device__ __forceinline__ float q4_0_convert<float>(float v) { return v; }
template <>
__device__ __forceinline__ double q4_0_convert<double>(float v) { return static_cast<double>(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 q4_0_convert<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half q4_0_convert<__half>(float v) { return __float2half_rn(v); }

// One thread per block: w = fp32(d * (c - 8)), then the output type (round to nearest even).
template <typename T>
__global__ void __launch_bounds__(256) q4_0_dequant_kernel(const uint8_t *__restrict__ blocks, int64_t nblocks,
                                                           T *__restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const uint8_t *bp = blocks + i * kQBlockBytes;
  const float d = half_bits_to_float(static_cast<uint32_t>(bp[0]) | (static_cast<uint32_t>(bp[1]) << 8));
  T *o = out + i * 32;  // block i covers columns 32 (i mod K/32) .. + 31 of its row: a contiguous run
  for (int j = 0; j < 16; ++j) {
    const uint32_t byte = bp[2 + j];
    o[j] = q4_0_convert<T>(d * static_cast<float>(static_cast<int>(byte & 15u) - 8));
    o[j + 16] = q4_0_convert<T>(d * static_cast<float>(static_cast<int>(byte >> 4) - 8));
  }
}

// One thread per block: the block's 16 code bytes become the 16 bytes of its 32-column group
// in the packed group-32 layout (column 2b in the low nibble of byte b, column 2b + 1 in the
// high one) holding the signed code c - 8 as a two's-complement nibble (c ^ 8), and the
// binary16 scale its exact fp32 value. Block i of the weight is group i % (K/32) of row
// i / (K/32), so its codes start at byte 16 i and its scale is scales[i].
__global__ void __launch_bounds__(256) q4_0_to_group32_kernel(const uint8_t *__restrict__ blocks, int64_t nblocks,
                                                              uint8_t *__restrict__ codes,
                                                              float *__restrict__ scales, bool vec) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const uint8_t *bp = blocks + i * kQBlockBytes;
  uint32_t c[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) c[j] = bp[2 + j];
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int b = 0; b < 16; ++b) {
    // columns 2b, 2b + 1: elements below 16 are low nibbles of code bytes 2b, 2b + 1; the
    // rest are high nibbles of bytes 2b - 16, 2b - 15
    const uint32_t lo = b < 8 ? (c[2 * b] & 15u) : (c[2 * b - 16] >> 4);
    const uint32_t hi = b < 8 ? (c[2 * b + 1] & 15u) : (c[2 * b - 15] >> 4);
    out[b / 4] |= ((lo | (hi << 4)) ^ 0x88u) << (8 * (b % 4));
  }
  uint8_t *o = codes + i * 16;
  if (vec) {
    *reinterpret_cast<uint4 *>(o) = make_uint4(out[0], out[1], out[2], out[3]);
  } else {
#pragma unroll
    for (int b = 0; b < 16; ++b) o[b] = static_cast<uint8_t>(out[b / 4] >> (8 * (b % 4)));
  }
  scales[i] = half_bits_to_float(static_cast<uint32_t>(bp[0]) | (static_cast<uint32_t>(bp[1]) << 8));
}

cudaError_t ensure_q4_0_smem() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(q4_0_gemv_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

int q4_0_sm_count() {
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

int64_t q4_0_tma_smem(int64_t K) {
  return kQAlign + static_cast<int64_t>(kQStages) * kQStageBytes + K * 2 + 2 * kQWarps * kQRows * 4 + kQBarBytes;
}

}  // namespace

bool q4_0_gemv_supports(const void *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K, int y_dtype) {
  if (M != 1 || K % 256 != 0 || N < 1 || N > 0x7fffffffLL) return false;
  if (y_dtype != W4_BF16 && y_dtype != W4_F32) return false;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(blocks)) % 16 != 0) return false;
  return q4_0_tma_smem(K) <= 113 * 1024 && encode_fn() != nullptr;  // two CTAs per SM
}

cudaError_t launch_q4_0_linear(const __nv_bfloat16 *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K,
                               const float *bias, void *y, int y_dtype, bool prefetch, int32_t *err,
                               cudaStream_t stream) {
  if (q4_0_gemv_supports(x, M, blocks, N, K, y_dtype)) {
    const int64_t row_bytes = K / 32 * kQBlockBytes, KT = K / 256;
    CUtensorMap tm;
    if (make_map_3d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, blocks, kQTileBytes, N, KT, row_bytes, kQTileBytes,
                    kQTileBytes, kQRows, kQWarps, CU_TENSOR_MAP_SWIZZLE_NONE)) {
      cudaError_t e = ensure_q4_0_smem();
      if (e != cudaSuccess) return e;
      Q40Params q;
      q.x = x;
      q.bias = bias;
      q.y = y;
      q.N = N;
      q.K = K;
      q.KT = static_cast<int>(KT);
      q.SPR = static_cast<int>((KT + kQWarps - 1) / kQWarps);
      q.y_dtype = y_dtype;
      q.prefetch = prefetch ? 1 : 0;
      const int64_t NB = (N + kQRows - 1) / kQRows;
      const int64_t slots = static_cast<int64_t>(q4_0_sm_count()) * 2;
      const int64_t grid = NB < slots ? NB : slots;
      q.rb_q = static_cast<int>(NB / grid);
      q.rb_r = static_cast<int>(NB % grid);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(grid));
      cfg.blockDim = dim3(32 * (kQWarps + 1));
      cfg.dynamicSmemBytes = static_cast<size_t>(q4_0_tma_smem(K));
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, q4_0_gemv_tma_kernel, tm, q, err);
    }
  }
  const int64_t warps = N * ((M + kPlainTok - 1) / kPlainTok);
  const int64_t grid = (warps * 32 + 255) / 256;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  q4_0_linear_plain_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(x, blocks, bias, y, M, N, K, y_dtype);
  return cudaGetLastError();
}

cudaError_t launch_q4_0_dequantize(const uint8_t *blocks, int64_t N, int64_t K, int out_dtype, void *out,
                                   cudaStream_t stream) {
  const int64_t nb = N * (K / 32);
  const int64_t grid = (nb + 255) / 256;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const unsigned gi = static_cast<unsigned>(grid);
  switch (out_dtype) {
    case W4_BF16: q4_0_dequant_kernel<__nv_bfloat16><<<gi, 256, 0, stream>>>(blocks, nb, static_cast<__nv_bfloat16 *>(out)); break;
    case W4_F16: q4_0_dequant_kernel<__half><<<gi, 256, 0, stream>>>(blocks, nb, static_cast<__half *>(out)); break;
    case W4_F32: q4_0_dequant_kernel<float><<<gi, 256, 0, stream>>>(blocks, nb, static_cast<float *>(out)); break;
    case W4_F64: q4_0_dequant_kernel<double><<<gi, 256, 0, stream>>>(blocks, nb, static_cast<double *>(out)); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_q4_0_to_group32(const uint8_t *blocks, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                   cudaStream_t stream) {
  const int64_t nb = N * (K / 32);
  const int64_t grid = (nb + 255) / 256;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const bool vec = reinterpret_cast<uintptr_t>(codes) % 16 == 0;
  q4_0_to_group32_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(blocks, nb, codes, scales, vec);
  return cudaGetLastError();
}

}  // namespace w4i

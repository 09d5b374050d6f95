// Device helpers of the CUDA-core decode GEMV kernels: activation chunk loading with the
// pair permutation that matches the nibble unpack order, the 32-column chunk dot product and
// the transposing warp reduction of 8 rows.
#pragma once

#include "w4_internal.cuh"

namespace w4i {

constexpr int kGemvRows = 8;  // rows reduced together by reduce_rows8

template <int MT>
__device__ __forceinline__ void pack_x_pairs(const uint32_t r[4], uint32_t *xp) {
  // r holds x[8t + 0..7] as bf16 pairs (0,1) (2,3) (4,5) (6,7); the nibble pairs of a
  // code word come out as columns (0,4) (1,5) (2,6) (3,7).
  xp[0] = prmt(r[0], r[2], 0x5410);
  xp[1] = prmt(r[0], r[2], 0x7632);
  xp[2] = prmt(r[1], r[3], 0x5410);
  xp[3] = prmt(r[1], r[3], 0x7632);
}

// Activation chunk (32 columns starting at col0) of row m, as 16 permuted bf16x2 pairs.
// Columns past K read as zero. perm != null gathers original columns (act-order).
template <int MT>
__device__ __forceinline__ void load_x_chunk(const __nv_bfloat16 *__restrict__ x, int64_t M, int64_t K,
                                             int64_t col0, bool vec, const int32_t *__restrict__ perm,
                                             uint32_t (&xp)[MT][16]) {
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
#pragma unroll
  for (int m = 0; m < MT; ++m) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t r[4] = {0u, 0u, 0u, 0u};
      const int64_t c = col0 + 8 * t;
      if (m < M) {
        if (perm == nullptr && vec && c + 7 < K) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xb + m * K + c));
          r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (c + e < K) {
              const int64_t col = perm ? static_cast<int64_t>(__ldg(perm + c + e)) : c + e;
              const uint32_t b = __ldg(xb + m * K + col);
              r[e >> 1] |= b << (16 * (e & 1));
            }
          }
        }
      }
      pack_x_pairs<MT>(r, &xp[m][4 * t]);
    }
  }
}

// sum over the chunk's 32 columns of x * (nibble value - offset), in fp32.
// magic/offset: signed codes 0x43084308 / 0x43084308 (136 + q - 136 = q);
// asymmetric 0x43004300 / (128 + z) pair (128 + u - 128 - z = u - z).
__device__ __forceinline__ float dot_chunk(const uint4 cw, const uint32_t *xp, uint32_t magic,
                                           uint32_t offset, float acc) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t w = words[t];
    const uint32_t q0 = bf16x2_sub(nib_pair_bf16(w, magic), offset);
    const uint32_t q1 = bf16x2_sub(nib_pair_bf16(w >> 4, magic), offset);
    const uint32_t q2 = bf16x2_sub(nib_pair_bf16(w >> 8, magic), offset);
    const uint32_t q3 = bf16x2_sub(nib_pair_bf16(w >> 12, magic), offset);
    acc = fma2_bf16_f32(xp[4 * t + 0], q0, acc);
    acc = fma2_bf16_f32(xp[4 * t + 1], q1, acc);
    acc = fma2_bf16_f32(xp[4 * t + 2], q2, acc);
    acc = fma2_bf16_f32(xp[4 * t + 3], q3, acc);
  }
  return acc;
}

// Same sum with four independent accumulators (one per code word) so that consecutive FMAs
// do not wait on each other; the partial sums are added at the end.
__device__ __forceinline__ float dot_chunk_ilp(const uint4 cw, const uint32_t *xp, uint32_t magic,
                                               uint32_t offset) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t w = words[t];
    acc[t] = fma2_bf16_f32(xp[4 * t + 0], bf16x2_sub(nib_pair_bf16(w, magic), offset), acc[t]);
    acc[t] = fma2_bf16_f32(xp[4 * t + 1], bf16x2_sub(nib_pair_bf16(w >> 4, magic), offset), acc[t]);
    acc[t] = fma2_bf16_f32(xp[4 * t + 2], bf16x2_sub(nib_pair_bf16(w >> 8, magic), offset), acc[t]);
    acc[t] = fma2_bf16_f32(xp[4 * t + 3], bf16x2_sub(nib_pair_bf16(w >> 12, magic), offset), acc[t]);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Transposing butterfly: lane l ends with the warp-wide sum of row (l >> 2) & 7.
__device__ __forceinline__ float reduce_rows8(float v[kGemvRows], int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 16;
    const float keep = up ? v[i + 4] : v[i];
    const float send = up ? v[i] : v[i + 4];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 8;
    const float keep = up ? v[i + 2] : v[i];
    const float send = up ? v[i] : v[i + 2];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  {
    const bool up = lane & 4;
    const float keep = up ? v[1] : v[0];
    const float send = up ? v[0] : v[1];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  return v[0];
}


// ---------------------------------------------------------------------------
// fp32-pair formulation (the streaming GEMV): exact integer code values are formed in
// fp32 and multiplied with fp32 activations two at a time (fma.rn.f32x2).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ float f32x2_sum(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v)) + __uint_as_float(static_cast<uint32_t>(v >> 32));
}

// 32 activations of one chunk as 16 fp32 pairs (x[2i], x[2i+1]), columns past K zero;
// perm != null gathers original columns (act-order). bf16 -> fp32 is exact.
__device__ __forceinline__ void load_x_chunk_f32(const __nv_bfloat16 *__restrict__ x, int64_t m, int64_t M,
                                                 int64_t K, int64_t col0, bool vec,
                                                 const int32_t *__restrict__ perm, uint64_t (&xf)[16]) {
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint32_t r[4] = {0u, 0u, 0u, 0u};
    const int64_t c = col0 + 8 * t;
    if (m < M) {
      if (perm == nullptr && vec && c + 7 < K) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xb + m * K + c));
        r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (c + e < K) {
            const int64_t col = perm ? static_cast<int64_t>(__ldg(perm + c + e)) : c + e;
            r[e >> 1] |= static_cast<uint32_t>(__ldg(xb + m * K + col)) << (16 * (e & 1));
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) xf[4 * t + i] = pack2(r[i] << 16, r[i] & 0xFFFF0000u);
  }
}

// acc += sum over the chunk's 32 columns of x * value, value = nibble - offset, as an fp32
// pair accumulator. Each nibble is dropped into the low byte of the fp32 2^23 (PRMT; the
// xor turns a signed nibble n into n + 8 in [0, 15]); an exact fp32x2 subtract of
// offset2 = (2^23 + 8) [signed] or (2^23 + z) [asymmetric, zero point z] leaves the exact
// integer, and fp32x2 FMAs accumulate (the activation x integer product is exact).
__device__ __forceinline__ uint64_t dot_chunk_f32(const uint4 cw, const uint64_t (&xf)[16], uint32_t xorc,
                                                  uint64_t neg_offset2, uint64_t acc) {
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t lo = lop3_and_xor(words[t], 0x0F0F0F0Fu, xorc);       // columns 8t+0,2,4,6
    const uint32_t hi = lop3_and_xor(words[t] >> 4, 0x0F0F0F0Fu, xorc);  // columns 8t+1,3,5,7
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t fe = prmt(lo, 0x00004B00u, 0x5440u | b);
      const uint32_t fo = prmt(hi, 0x00004B00u, 0x5440u | b);
      const uint64_t q2 = f32x2_add(pack2(fe, fo), neg_offset2);
      acc = f32x2_fma(xf[4 * t + b], q2, acc);
    }
  }
  return acc;
}

// -(2^23 + v) as an fp32 bit pattern, both halves (v in [0, 15]).
__device__ __forceinline__ uint64_t neg_magic2(uint32_t v) {
  const uint32_t f = 0xCB000000u | v;
  return pack2(f, f);
}

}  // namespace w4i

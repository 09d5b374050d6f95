// Register-fed tensor-core building blocks shared by the small-M kernels: ldmatrix of
// swizzled code words, mma.sync m16n8k16 (bf16 in, fp32 accumulate) and the exact
// nibble -> bf16x2 unpack of signed codes.
#pragma once

#include <stdint.h>

#include "w4_internal.cuh"

namespace w4i {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&d)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(addr));
}

// D = A * B (+ 0) and D = A * B + D for m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ void mma_next(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One code word (columns 8t .. 8t+7 of a group, even column in the low nibble) -> four
// bf16x2 registers holding the exact signed integers of columns (0,4) (1,5) (2,6) (3,7).
__device__ __forceinline__ void unpack_signed(uint32_t w, uint32_t (&a)[4]) {
  a[0] = bf16x2_sub(nib_pair_bf16(w, 0x43084308u), 0x43084308u);
  a[1] = bf16x2_sub(nib_pair_bf16(w >> 4, 0x43084308u), 0x43084308u);
  a[2] = bf16x2_sub(nib_pair_bf16(w >> 8, 0x43084308u), 0x43084308u);
  a[3] = bf16x2_sub(nib_pair_bf16(w >> 12, 0x43084308u), 0x43084308u);
}

}  // namespace w4i


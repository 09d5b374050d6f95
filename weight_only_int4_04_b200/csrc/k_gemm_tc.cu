// Tensor-core W4A16 GEMM for prefill-sized M on sm_100a (tcgen05 + TMA + TMEM):
//   y[m][n] = sum_k x[m][k] * bf16(fp32(q[n][k] * s[n][k/32])) + b[n]
//
// Swap-AB formulation: the dequantized weight tile is the MMA's A operand (M_mma = 128 weight
// rows) and the activation tile is B (N_mma = 256 activation rows), so D = W_tile . x_tile^T
// is a 128 x 256 fp32 tile of y^T held in tensor memory. This puts the larger MMA dimension
// on the activations and dequantizes each weight tile once per 256 activation rows.
//
// One CTA per (128-row weight tile, 256-row activation tile); 10 warps, specialised:
//   warp 0     TMA producer: per 64-column K block, the x tile (256 x 64 bf16, 128-byte
//              swizzle), the code tile (128 rows x 32 bytes) and the scale tile
//              (128 rows x 4 groups) land on one mbarrier;
//   warp 1     allocates 256 TMEM columns; one thread issues 4 tcgen05.mma (K = 16 each)
//              per K block and commits the stage back to the producer;
//   warps 2-9  dequantize (warps 2-17 for 64-row activation tiles): thread (row, part)
//              turns 16 (8) code bytes + 1 scale into 32 (16) bf16 weights with LOP3/PRMT
//              and fp32x2 arithmetic and writes them with
//              tcgen05.st into the A operand's stage in tensor memory (row = TMEM lane,
//              the warp's own lane quarter); then, after the last MMA, the same warps move
//              D out of TMEM (tcgen05.ld), add the bias in fp32, round to the output dtype
//              and store y.
// The dequantized A operand never touches shared memory (it would cost 4 B of shared-memory
// traffic per weight, written by the dequant warps and read by the MMA, against 0.5 B of
// codes): shared memory holds only the TMA stages of x, codes and scales, and TMEM holds D
// (BN columns) plus one 32-column A slice per stage. A ring of 5 (BN = 256) or 8 (BN = 64)
// stages overlaps loads, dequantization and MMA. All waits are bounded (see w4_sync.cuh).
#include <cuda.h>

#include <mutex>

#include "w4_tc.cuh"
#include "w4_tmap.h"

namespace w4i {

namespace {

constexpr int BM_W = 128;  // weight rows per tile (MMA M)
constexpr int BK = 64;     // K per stage: one 128-byte swizzle row of bf16
constexpr int kDequantWarp0 = 2;
// Dequant (and epilogue) warps: 16 for 64-row activation tiles, where dequantization is the
// whole cost of a K block and more warps hide its latency; 8 for prefill tiles.
constexpr int dequant_warps(int BN) { return BN <= 64 ? 16 : 8; }
constexpr int threads_for(int BN) { return 32 * (kDequantWarp0 + dequant_warps(BN)); }

constexpr int C_BYTES = BM_W * (BK / 2);  // 4 KB of codes
constexpr int S_BYTES = BM_W * 4 * 4;     // 2 KB: 4 scale columns per row
constexpr int Z_BYTES = BM_W * 16;        // 2 KB: 16 zero-point columns per row (asymmetric)
constexpr int A_TMEM_COLS = BK / 2;       // one stage of A in TMEM: 64 bf16 per row = 32 columns
constexpr int kMaxStagesAsym = 512;       // K <= 32768 on the asymmetric path

// Shared-memory and tensor-memory plan for BN activation rows per tile (MMA N = BN: 64 for
// the mid-M range, 256 for prefill); a narrower tile leaves room for a deeper ring.
template <bool ASYM, int BN>
struct TcLayout {
  static constexpr int STAGES = BN <= 64 ? 8 : 5;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_S = OFF_C + STAGES * C_BYTES;
  static constexpr int OFF_Z = OFF_S + STAGES * S_BYTES;
  static constexpr int OFF_G = ASYM ? OFF_Z + STAGES * Z_BYTES : OFF_Z;
  static constexpr int OFF_BAR = OFF_G + (ASYM ? 2 * kMaxStagesAsym : 0);
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers + 1 KB alignment slack
  static constexpr uint32_t TX = B_BYTES + C_BYTES + S_BYTES + (ASYM ? Z_BYTES : 0);
  // D in columns [0, BN), A stage s in [BN + 32 s, BN + 32 s + 32); allocation: power of 2
  static constexpr uint32_t TMEM_NEED = BN + STAGES * A_TMEM_COLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                        : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(TMEM_NEED <= 512, "GEMM exceeds the tensor-memory budget");
  static_assert(SMEM <= 227 * 1024, "GEMM exceeds the shared-memory budget");
};

struct TcParams {
  const float *bias;
  void *y;
  int64_t M, N, K;
  int y_dtype;
  // asymmetric act-order only: columns are sorted; the stage table maps each 64-column K
  // block to its scale column (or -1 when the block spans two groups)
  const int32_t *g_idx;
  const int32_t *perm;
  const float *scales;
  const int8_t *zeros;
  int n_groups;
};

template <bool ASYM, int BN>
__global__ void __launch_bounds__(threads_for(BN), 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                   const __grid_constant__ CUtensorMap tmap_scales, const __grid_constant__ CUtensorMap tmap_zeros,
                   const TcParams p, int32_t *err) {
  using L = TcLayout<ASYM, BN>;
  constexpr int STAGES = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base (the 128-byte swizzle atoms must start on 1024-byte boundaries)
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t *full_load = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
  int16_t *gstage = reinterpret_cast<int16_t *>(smem + L::OFF_G);
  uint64_t *full_a = full_load + STAGES;
  uint64_t *empty = full_a + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *issued_sm = const_cast<int *>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BM_W;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BN;
  const int KB = static_cast<int>((p.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_load[s], 1);
      mbar_init(&full_a[s], dequant_warps(BN));  // one arrive per dequant warp
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (ASYM) {
    // scale column of every 64-column K block of the sorted columns (-1: two groups)
    for (int kb = threadIdx.x; kb < KB; kb += blockDim.x) {
      const int64_t c0 = static_cast<int64_t>(kb) * BK;
      const int64_t last = (c0 + BK - 1 < p.K) ? c0 + BK - 1 : p.K - 1;
      const int32_t g0 = __ldg(p.g_idx + __ldg(p.perm + c0));
      gstage[kb] = static_cast<int16_t>(g0 == __ldg(p.g_idx + __ldg(p.perm + last)) ? g0 : -1);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int kb = 0;
      for (; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, err)) break;
        mbar_arrive_expect_tx(&full_load[s], L::TX);
        tma_load_2d(smem + L::OFF_B + s * L::B_BYTES, &tmap_x, kb * BK, static_cast<int32_t>(m0), &full_load[s]);
        tma_load_2d(smem + L::OFF_C + s * C_BYTES, &tmap_codes, kb * (BK / 2), static_cast<int32_t>(n0),
                    &full_load[s]);
        if (!ASYM) {
          tma_load_2d(smem + L::OFF_S + s * S_BYTES, &tmap_scales, 4 * (kb / 2), static_cast<int32_t>(n0),
                      &full_load[s]);
        } else {
          const int gs = gstage[kb] < 0 ? 0 : gstage[kb];
          tma_load_2d(smem + L::OFF_S + s * S_BYTES, &tmap_scales, gs & ~3, static_cast<int32_t>(n0), &full_load[s]);
          tma_load_2d(smem + L::OFF_Z + s * Z_BYTES, &tmap_zeros, gs & ~15, static_cast<int32_t>(n0), &full_load[s]);
        }
      }
      *issued_sm = kb;  // stages whose copies were issued (read on the abort path below)
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(BM_W, BN);
      const uint32_t b_base = smem_u32(smem + L::OFF_B);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
        mbar_wait(&full_a[s], ph, abort_flag, err);
        mbar_wait(&full_load[s], ph, abort_flag, err);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t a_tmem = tmem_d + BN + s * A_TMEM_COLS + kk * 8;  // K = 16: 8 columns
          const uint64_t bd = umma_desc_sw128(b_base + s * L::B_BYTES + kk * 32);
          umma_bf16_tmem_a(tmem_d, a_tmem, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);
    }
  } else {
    // ---- dequantize into the A stages ----
    constexpr int PARTS = dequant_warps(BN) / 4;  // warps per TMEM lane quarter
    constexpr int CP = BK / PARTS;                 // K columns of a stage per thread (32 or 16)
    constexpr int NW = CP / 8;                     // code words per thread (4 or 2)
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    const int part = (warp - kDequantWarp0) >> 2;  // which CP of the stage's 64 columns
    const int r = 32 * q + lane;                   // weight row inside the tile
    // this warp's lane quarter, columns of its part of the stage's 64 K values
    const uint32_t a_tmem0 = tmem_d + (static_cast<uint32_t>(32 * q) << 16) + BN + (CP / 2) * part;
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
      mbar_wait(&full_load[s], ph, abort_flag, err);
      uint32_t words[NW];
      const uint8_t *cp = smem + L::OFF_C + s * C_BYTES + r * 32 + (CP / 2) * part;
      if constexpr (NW == 4) {
        const uint4 cw = *reinterpret_cast<const uint4 *>(cp);
        words[0] = cw.x, words[1] = cw.y, words[2] = cw.z, words[3] = cw.w;
      } else {
        const uint2 cw = *reinterpret_cast<const uint2 *>(cp);
        words[0] = cw.x, words[1] = cw.y;
      }
      float sc;
      uint32_t xorc = 0x08080808u;
      uint64_t nb2 = neg_bias_pair(8u);
      int gs = 0;
      if (!ASYM) {
        sc = reinterpret_cast<const float *>(smem + L::OFF_S + s * S_BYTES)[r * 4 + (kb & 1) * 2 + ((CP * part) >> 5)];
      } else {
        gs = gstage[kb];
        const int gsc = gs < 0 ? 0 : gs;
        sc = reinterpret_cast<const float *>(smem + L::OFF_S + s * S_BYTES)[r * 4 + (gsc & 3)];
        const uint32_t z = static_cast<uint32_t>(
            reinterpret_cast<const uint8_t *>(smem + L::OFF_Z + s * Z_BYTES)[r * 16 + (gsc & 15)]) & 15u;
        xorc = 0u;
        nb2 = neg_bias_pair(z);
      }
      const uint64_t scale2 = (static_cast<uint64_t>(__float_as_uint(sc)) << 32) | __float_as_uint(sc);
      uint32_t av[4 * NW];  // CP bf16 of this row: K pairs (2c, 2c + 1) in column c
      if (!ASYM || gs >= 0) {
#pragma unroll
        for (int t = 0; t < NW; ++t) {
          const uint4 v = dequant_word_bf16(words[t], scale2, xorc, nb2);
          av[4 * t] = v.x;
          av[4 * t + 1] = v.y;
          av[4 * t + 2] = v.z;
          av[4 * t + 3] = v.w;
        }
      } else {
        // this K block spans two groups: per-column scale and zero from global memory
        const int64_t n = n0 + r;
#pragma unroll
        for (int t = 0; t < NW; ++t) {
          uint32_t packed[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float wv[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e2 + h2;
              const int64_t col = static_cast<int64_t>(kb) * BK + CP * part + 8 * t + e;
              wv[h2] = 0.0f;
              if (n < p.N && col < p.K) {
                const int64_t gg = __ldg(p.g_idx + __ldg(p.perm + col));
                const int u = static_cast<int>((words[t] >> (4 * e)) & 15u);
                wv[h2] = __fmul_rn(static_cast<float>(u - p.zeros[n * p.n_groups + gg]),
                                   p.scales[n * p.n_groups + gg]);
              }
            }
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed[e2]) : "f"(wv[1]), "f"(wv[0]));
          }
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) av[4 * t + e2] = packed[e2];
        }
      }
      if constexpr (NW == 4)
        tmem_st_32x32b_x16(a_tmem0 + s * A_TMEM_COLS, av);
      else
        tmem_st_32x32b_x8(a_tmem0 + s * A_TMEM_COLS, av);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full_a[s]);
    }

    // ---- epilogue: TMEM -> registers -> y ----
    mbar_wait(acc_full, 0, abort_flag, err);
    __syncwarp();  // tcgen05.ld is warp-collective; the lanes left the wait one by one
    tc_fence_after();
    const int64_t n = n0 + r;
    const float b = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN / PARTS / 16; ++c) {
      const int col0 = (BN / PARTS) * part + 16 * c;
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem_d + (static_cast<uint32_t>(32 * q) << 16) + col0, v);
      if (n < p.N) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int64_t m = m0 + col0 + j;
          if (m < p.M) {
            const float o = __uint_as_float(v[j]) + b;
            if (p.y_dtype == W4_F32) {
              static_cast<float *>(p.y)[m * p.N + n] = o;
            } else {
              static_cast<__nv_bfloat16 *>(p.y)[m * p.N + n] = __float2bfloat16_rn(o);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // abort path (see w4_sync.cuh): the consumers stopped waiting, so the copies issued must
    // land and every MMA must finish before the CTA frees its tensor memory and exits
    const int issued = *issued_sm;
    for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
      mbar_drain(&full_load[kb % STAGES], static_cast<uint32_t>(kb / STAGES) & 1u, err);
    mbar_drain(acc_full, 0u, err);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, L::TMEM_COLS);
  }
}

}  // namespace

bool gemm_tc_supports(const LinearParams &p) {
  const int64_t P = (p.K + 1) / 2, G = (p.K + 31) / 32;
  if (p.K % 8 != 0 || P % 16 != 0) return false;
  if (!p.asym && G % 4 != 0) return false;
  if (p.asym && (p.perm == nullptr || p.n_groups % 16 != 0 || (p.K + BK - 1) / BK > kMaxStagesAsym ||
                 p.n_groups > 32767))
    return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p.codes) | reinterpret_cast<uintptr_t>(p.scales) |
                      (p.asym ? reinterpret_cast<uintptr_t>(p.zeros) : 0) |
                      (p.asym ? 0 : reinterpret_cast<uintptr_t>(p.x));
  if (a % 16 != 0) return false;
  if ((p.M + 255) / 256 > 65535 || (p.N + BM_W - 1) / BM_W > 0x7fffffffLL) return false;
  return encode_fn() != nullptr;
}

// x gathered through perm (act-order): xg[m][j] = x[m][perm[j]], eight columns per thread.
__global__ void __launch_bounds__(256) gather_x_kernel(const __nv_bfloat16 *__restrict__ x,
                                                       const int32_t *__restrict__ perm, int64_t M, int64_t K,
                                                       __nv_bfloat16 *__restrict__ xg) {
  // Launched with programmatic stream serialization: the next kernel may launch at once;
  // x (written by the previous kernel) is read only after grid_dependency_wait, perm (a
  // weight) before it.
  grid_launch_dependents();
  const int64_t units = M * (K / 8);
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(x);
  bool waited = false;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = u / (K / 8), j0 = (u % (K / 8)) * 8;
    const int4 p0 = __ldg(reinterpret_cast<const int4 *>(perm + j0));
    const int4 p1 = __ldg(reinterpret_cast<const int4 *>(perm + j0) + 1);
    if (!waited) {
      grid_dependency_wait();
      waited = true;
    }
    const int32_t col[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    uint32_t v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = __ldca(xb + m * K + col[2 * i]);
      const uint32_t hi = __ldca(xb + m * K + col[2 * i + 1]);
      v[i] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(xg + m * K + j0) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

cudaError_t launch_gather_x(const __nv_bfloat16 *x, const int32_t *perm, int64_t M, int64_t K, __nv_bfloat16 *xg,
                            cudaStream_t stream) {
  if (reinterpret_cast<uintptr_t>(perm) % 16 != 0 || K % 8 != 0) return cudaErrorInvalidValue;
  int64_t blocks = (M * (K / 8) + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gather_x_kernel, x, perm, M, K, xg);
}

size_t gemm_tc_asym_workspace(int64_t M, int64_t K) {
  return static_cast<size_t>(((M * K * 2 + 255) / 256) * 256);
}

template <bool ASYM, int BN>
cudaError_t launch_typed(dim3 grid, const CUtensorMap &mx, const CUtensorMap &mc, const CUtensorMap &ms,
                         const CUtensorMap &mz, const TcParams &tp, int32_t *err, cudaStream_t stream) {
  using L = TcLayout<ASYM, BN>;
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
      e = cudaFuncSetAttribute(gemm_tc_kernel<ASYM, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
      if (e != cudaSuccess) return e;
      done[dev] = true;
    }
  }
  gemm_tc_kernel<ASYM, BN><<<grid, threads_for(BN), L::SMEM, stream>>>(mx, mc, ms, mz, tp, err);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const LinearParams &p, int32_t *err, cudaStream_t stream, void *workspace) {
  if (!gemm_tc_supports(p)) return cudaErrorNotSupported;
  const int64_t P = (p.K + 1) / 2, G = (p.K + 31) / 32;
  const __nv_bfloat16 *xsrc = p.x;
  if (p.asym) {
    // act-order: the activations are gathered once into the workspace in sorted column order
    if (workspace == nullptr || reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return cudaErrorInvalidValue;
    __nv_bfloat16 *xg = static_cast<__nv_bfloat16 *>(workspace);
    const cudaError_t e = launch_gather_x(p.x, p.perm, p.M, p.K, xg, stream);
    if (e != cudaSuccess) return e;
    xsrc = xg;
  }
  const int64_t SG = p.asym ? p.n_groups : G;
  // MMA N = activation rows per tile: 64 up to M = 64 (the mid-M range, where the weight
  // stream dominates and a wider tile would only multiply idle tensor work), else 256
  const int bn = p.M <= 64 ? 64 : 256;
  CUtensorMap mx, mc, ms, mz;
  if (!make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xsrc, p.K, p.M, p.K * 2, BK, bn,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.codes, P, p.N, P, BK / 2, BM_W, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.scales, SG, p.N, SG * 4, 4, BM_W,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (p.asym) {
    if (!make_map_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.zeros, SG, p.N, SG, 16, BM_W, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    mz = ms;  // unused by the symmetric kernel
  }
  TcParams tp{p.bias, p.y, p.M, p.N, p.K, p.y_dtype, p.g_idx, p.perm, p.scales, p.zeros, p.n_groups};
  const dim3 grid(static_cast<unsigned>((p.N + BM_W - 1) / BM_W), static_cast<unsigned>((p.M + bn - 1) / bn));
  if (p.asym) {
    if (bn == 64) return launch_typed<true, 64>(grid, mx, mc, ms, mz, tp, err, stream);
    return launch_typed<true, 256>(grid, mx, mc, ms, mz, tp, err, stream);
  }
  if (bn == 64) return launch_typed<false, 64>(grid, mx, mc, ms, mz, tp, err, stream);
  return launch_typed<false, 256>(grid, mx, mc, ms, mz, tp, err, stream);
}

}  // namespace w4i

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
//   * bwd_x_mma_kernel (2 <= M, K a multiple of 128, N a multiple of 8, 16-byte aligned codes
//     and dy, 4-byte aligned scales): tensor cores. A CTA owns 128 columns (four scale groups),
//     a slice of rows and 16 upstream rows. Per step of 32 weight rows each thread unpacks one
//     32-column group of one row (one 16-byte code load) into a bf16 tile of exact integer
//     codes in shared memory, 16-byte chunks XOR-swizzled by the row so that both the stores
//     and the transposing loads are conflict-free, and stores the row's scale; the upstream
//     rows go to a padded tile. Warp w owns columns 32w .. 32w+31, exactly scale group w: it
//     loads its A fragments (upstream rows x weight rows) with ldmatrix, multiplies each value
//     by its weight row's scale in fp32 and splits the product into a bf16 pair hi + lo
//     (within 2^-16 of it: one bf16 alone could cost 2^-8 per term, too much for the
//     tolerance once the output is rounded to bf16 as well), loads the B fragments (weight
//     rows x columns: the contraction runs over the weight's rows, which the packed codes do
//     not pair) with ldmatrix.trans, and runs two mma.sync m16n8k16 (bf16 in, fp32
//     accumulate) per fragment. Two buffers, one barrier per step; the codes, scales and
//     upstream values of the next two steps are in flight while the current step multiplies.
//     Row splits meet in bwd_x_reduce_kernel as above.
//   * bwd_x_plain_kernel: any K, one thread per (token, column), rows in order.
#include "w4_mma.cuh"
#include "w4_tc.cuh"

namespace w4i {

namespace {

constexpr int kBwdTile = 256;   // columns per CTA (32 code words)
constexpr int kBwdWarps = 8;
constexpr int kBwdTargetCtas = 592;  // four per SM on a 148-SM part; sets the row split
constexpr int kBwdStageRows = 1024;  // rows whose upstream gradient is staged in shared memory at once
constexpr int64_t kBwdMinRows = 64;  // rows per split at least
constexpr int64_t kBwdMmaMinM = 2;   // upstream rows from which the tensor-core kernel serves
constexpr int64_t kBwdMmaTargetCtas = 888;  // six 128-thread CTAs per SM of a 148-SM part

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

constexpr int kMmaCols = 128;   // columns per CTA (four warps x 32)
constexpr int kMmaRows = 32;    // weight rows per step
constexpr int kMmaTok = 16;     // upstream rows per CTA (the MMA's M)
constexpr int kMmaThreads = 128;
constexpr int kWtPitch = kMmaCols * 2;  // bytes per row of the bf16 weight tile
constexpr int kDyPitch = 80;            // 32 bf16 + 16 bytes: conflict-free ldmatrix rows

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&d)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Upstream values of one A-fragment register (two bf16, weight rows n, n + 1) times the two
// rows' scales, as a pair of bf16x2 registers hi + lo: hi = bf16(fl32(dy * s)), lo = bf16 of
// the (exact) remainder, so hi + lo is within 2^-16 of the fp32 product. (ptxas may fuse the
// packed multiply and subtract into one fma; lo is then the remainder of the exact product,
// which only tightens the bound.)
__device__ __forceinline__ void scale_split(uint32_t x2, uint64_t s2, uint32_t &hi, uint32_t &lo) {
  uint64_t v = (static_cast<uint64_t>(x2 & 0xFFFF0000u) << 32) | (x2 << 16);
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(v) : "l"(s2));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
      : "=r"(hi)
      : "f"(__uint_as_float(static_cast<uint32_t>(v >> 32))), "f"(__uint_as_float(static_cast<uint32_t>(v))));
  const uint64_t hw = (static_cast<uint64_t>(hi & 0xFFFF0000u) << 32) | (hi << 16);
  asm("sub.rn.f32x2 %0, %0, %1;" : "+l"(v) : "l"(hw));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
      : "=r"(lo)
      : "f"(__uint_as_float(static_cast<uint32_t>(v >> 32))), "f"(__uint_as_float(static_cast<uint32_t>(v))));
}

__global__ void __launch_bounds__(kMmaThreads) bwd_x_mma_kernel(const __nv_bfloat16 *__restrict__ dy,
                                                                const uint8_t *__restrict__ codes,
                                                                const float *__restrict__ scales, float *part,
                                                                void *dx, int dx_dtype, int64_t M, int64_t N,
                                                                int64_t K, int64_t rows_per_split, int splits) {
  __shared__ __align__(128) uint8_t wq[2][kMmaRows * kWtPitch];  // exact codes as bf16 [row][128 columns]
  __shared__ __align__(16) float wsc[2][4][kMmaRows];             // the step's scales [group][row]
  __shared__ __align__(128) uint8_t dys[2][kMmaTok * kDyPitch];
  const int tid = static_cast<int>(threadIdx.x), warp = tid >> 5, lane = tid & 31;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kMmaCols;
  const int split = static_cast<int>(blockIdx.y);
  const int64_t m0 = static_cast<int64_t>(blockIdx.z) * kMmaTok;
  const int64_t n_begin = static_cast<int64_t>(split) * rows_per_split;
  const int64_t n_end = (n_begin + rows_per_split < N) ? n_begin + rows_per_split : N;
  const int64_t P = K / 2, G = K / 32;
  // unpack role: row r of the step, the 32 columns of group q of the tile (four code words,
  // one 16-byte load, one scale)
  const int r = tid >> 2, q = tid & 3;
  const uint4 *cw_base = reinterpret_cast<const uint4 *>(codes + k0 / 2) + q;
  const float *sc_base = scales + k0 / 32 + q;
  // upstream role (threads 0..63): row tok of the 16, eight weight rows q8 .. q8+7 of the step
  const int tok = tid >> 2, q8 = (tid & 3) * 8;
  const bool dy_row = tid < 64 && m0 + tok < M;
  const __nv_bfloat16 *dy_base = dy + (m0 + tok) * N + q8;

  struct Step {
    uint4 cw;
    float sc;
    uint4 dv;
  };
  // rows past the slice: codes 0, scale 0, upstream 0
  auto fetch = [&](Step &st, int64_t n0) {
    const int64_t n = n0 + r;
    const bool ok = n < n_end;
    st.cw = ok ? __ldg(cw_base + n * (P / 16)) : make_uint4(0u, 0u, 0u, 0u);
    st.sc = ok ? __ldg(sc_base + n * G) : 0.0f;
    st.dv = (dy_row && n0 + q8 < n_end) ? __ldg(reinterpret_cast<const uint4 *>(dy_base + n0))
                                        : make_uint4(0u, 0u, 0u, 0u);
  };
  // The codes go to the tile as exact integers (one LOP3 and one bf16x2 FMA per column pair);
  // each 16-byte chunk holds its eight columns in the order 0 4 1 5 2 6 3 7, which the output
  // indexing undoes. The scale stays fp32 and multiplies the upstream values instead.
  auto put = [&](const Step &st, int buf) {
    const uint32_t words[4] = {st.cw.x, st.cw.y, st.cw.z, st.cw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // the four lanes of a row start at different chunks: fewer bank conflicts on the stores
      const int jj = (j + q) & 3;
      uint32_t a[4];
      unpack_signed(words[jj], a);
      const int off = r * kWtPitch + (((4 * q + jj) ^ (r & 7)) << 4);
      *reinterpret_cast<uint4 *>(&wq[buf][off]) = make_uint4(a[0], a[1], a[2], a[3]);
    }
    wsc[buf][q][r] = st.sc;
    if (tid < 64) *reinterpret_cast<uint4 *>(&dys[buf][tok * kDyPitch + (tid & 3) * 16]) = st.dv;
  };

  // per-lane ldmatrix addresses (offsets inside a buffer)
  // A (upstream rows x weight rows, row-major): matrix i = lane >> 3: rows (l & 7) + 8 (i & 1),
  // columns 8 (i >> 1) .. of the 16-row half h
  const int li = lane >> 3, lr = lane & 7;
  const uint32_t a_off = static_cast<uint32_t>((lr + 8 * (li & 1)) * kDyPitch + 16 * (li >> 1));
  // B (weight rows x columns, transposed on load): matrix i: rows (l & 7) + 8 (i & 1) of the
  // half, 16-byte chunk 4 warp + pair + (i >> 1)
  const int b_row = lr + 8 * (li & 1);
  const int g = lane >> 2, t = lane & 3;

  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;

  const int steps = n_end > n_begin ? static_cast<int>((n_end - n_begin + kMmaRows - 1) / kMmaRows) : 0;
  // warp w owns columns 32w .. 32w+31: exactly scale group w of the tile
  auto multiply = [&](int buf) {
    const uint32_t wbase = smem_u32(&wq[buf][0]);
    const uint32_t dbase = smem_u32(&dys[buf][0]);
    const float *sw = &wsc[buf][warp][0];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a[4];
      ldsm_x4(dbase + a_off + 32u * h, a);
      // the rows of this lane's A registers: 16h + 2t (+1) for a0 / a1, 16h + 2t + 8 (+1) for a2 / a3
      const uint64_t s01 = *reinterpret_cast<const uint64_t *>(sw + 16 * h + 2 * t);
      const uint64_t s89 = *reinterpret_cast<const uint64_t *>(sw + 16 * h + 2 * t + 8);
      uint32_t ah[4], al[4];
      scale_split(a[0], s01, ah[0], al[0]);
      scale_split(a[1], s01, ah[1], al[1]);
      scale_split(a[2], s89, ah[2], al[2]);
      scale_split(a[3], s89, ah[3], al[3]);
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int row = 16 * h + b_row;
        const int chunk = 4 * warp + 2 * pr + (li >> 1);
        uint32_t b[4];
        ldsm_x4_trans(wbase + static_cast<uint32_t>(row * kWtPitch + ((chunk ^ (row & 7)) << 4)), b);
        mma_acc(acc[2 * pr], ah, b[0], b[1]);
        mma_acc(acc[2 * pr], al, b[0], b[1]);
        mma_acc(acc[2 * pr + 1], ah, b[2], b[3]);
        mma_acc(acc[2 * pr + 1], al, b[2], b[3]);
      }
    }
  };
  // two steps in flight: step i's loads are issued two steps ahead of its multiply
  Step sa, sb;
  if (steps > 0) fetch(sa, n_begin);
  if (steps > 1) fetch(sb, n_begin + kMmaRows);
  if (steps > 0) put(sa, 0);
  for (int it = 0; it < steps; it += 2) {
    // even step: buffer 0 holds it; sb holds it + 1
    if (it + 2 < steps) fetch(sa, n_begin + static_cast<int64_t>(it + 2) * kMmaRows);
    __syncthreads();  // buffer 0 is written; buffer 1's readers (step it - 1) are done
    multiply(0);
    if (it + 1 >= steps) break;
    put(sb, 1);
    // odd step: buffer 1 holds it + 1; sa holds it + 2
    if (it + 3 < steps) fetch(sb, n_begin + static_cast<int64_t>(it + 3) * kMmaRows);
    __syncthreads();
    multiply(1);
    if (it + 2 < steps) put(sa, 0);
  }

  // acc[j]: upstream rows g, g + 8 x tile positions 2t, 2t + 1 of column chunk 4 warp + j,
  // which hold columns t and t + 4 of the chunk
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t kk = k0 + 32 * warp + 8 * j + t;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int64_t m = m0 + g + 8 * hf;
      if (m >= M) continue;
      const float v0 = acc[j][2 * hf], v1 = acc[j][2 * hf + 1];
      if (splits == 1) {
        store_out(dx, dx_dtype, m * K + kk, v0);
        store_out(dx, dx_dtype, m * K + kk + 4, v1);
      } else {
        float *dst = part + (static_cast<int64_t>(split) * M + m) * K + kk;
        dst[0] = v0;
        dst[4] = v1;
      }
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

// Row splits of the tensor-core kernel: about four CTAs per SM, whole 32-row steps.
bool bwd_mma_shape(int64_t M, int64_t N, int64_t K) {
  return M >= kBwdMmaMinM && K % kMmaCols == 0 && N % 8 == 0 && (M + kMmaTok - 1) / kMmaTok <= 65535;
}

int64_t bwd_mma_rows(int64_t M, int64_t N, int64_t K) {
  const int64_t ctas = (K / kMmaCols) * ((M + kMmaTok - 1) / kMmaTok);
  int64_t splits = (kBwdMmaTargetCtas + ctas - 1) / ctas;
  const int64_t max_splits = (N + kMmaRows - 1) / kMmaRows;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  const int64_t rows = (N + splits - 1) / splits;
  return (rows + kMmaRows - 1) / kMmaRows * kMmaRows;
}

int64_t bwd_mma_splits(int64_t M, int64_t N, int64_t K) {
  const int64_t rows = bwd_mma_rows(M, N, K);
  return (N + rows - 1) / rows;
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
  // the larger of the two kernels' needs: which one serves can depend on pointer alignment
  const int64_t s = bwd_splits(M, N, K);
  const int64_t s2 = bwd_mma_shape(M, N, K) ? bwd_mma_splits(M, N, K) : 1;
  const int64_t sm = s > s2 ? s : s2;
  return sm > 1 ? static_cast<size_t>(sm) * static_cast<size_t>(M) * static_cast<size_t>(K) * sizeof(float) : 0;
}

cudaError_t launch_linear_backward_x(const __nv_bfloat16 *dy, int64_t M, const uint8_t *codes, const float *scales,
                                     int64_t N, int64_t K, void *dx, int dx_dtype, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream) {
  if (bwd_mma_shape(M, N, K) && bwd_fast(codes, scales, K) &&
      (reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(codes)) % 16 == 0) {
    const int64_t rows = bwd_mma_rows(M, N, K), splits = (N + rows - 1) / rows;
    const size_t need_mma = splits > 1 ? static_cast<size_t>(splits * M * K) * sizeof(float) : 0;
    if (need_mma == 0 || (workspace != nullptr && workspace_bytes >= need_mma)) {
      const dim3 grid(static_cast<unsigned>(K / kMmaCols), static_cast<unsigned>(splits),
                      static_cast<unsigned>((M + kMmaTok - 1) / kMmaTok));
      bwd_x_mma_kernel<<<grid, kMmaThreads, 0, stream>>>(dy, codes, scales, static_cast<float *>(workspace), dx,
                                                         dx_dtype, M, N, K, rows, static_cast<int>(splits));
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess || splits == 1) return e;
      const int64_t MK = M * K;
      bwd_x_reduce_kernel<<<static_cast<unsigned>((MK + 255) / 256), 256, 0, stream>>>(
          static_cast<float *>(workspace), dx, dx_dtype, MK, static_cast<int>(splits));
      return cudaGetLastError();
    }
  }
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

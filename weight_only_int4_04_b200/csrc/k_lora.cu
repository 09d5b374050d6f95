// LoRA merge into a packed weight (Keras page, keras/src/layers/core/dense.py int4 diff,
// Dense's merged-kernel helper: dequantize, add (lora_alpha / lora_rank) * A . B in the
// float domain, re-quantize, pack). Layout [N, K]: delta[n][k] = c * sum_j b[n][j] * a[j][k]
// with b = B^T [N, r], a = A^T [r, K], c = alpha / rank. Reading of the arithmetic (fp32,
// every step rounded, in this order, so the new codes depend on the inputs alone):
//     w = fl32(q * s);  t = 0; for j: t = fl32(t + fl32(b[n][j] * a[j][k]));  w' = fl32(w + fl32(c * t))
// then the RTN group-32 rule of w4_quantize_rtn on w'. The products and sums are separately
// rounded scalar operations (__fmul_rn / __fadd_rn), j ascending. The packed f32x2 multiply
// and add are not used for the sum: ptxas fuses such a pair into one fma, which rounds once.
//   * lora_merge_kernel: the weight is cut into 32-row x 128-column tiles; a CTA keeps one
//     column tile and walks row tiles (the grid is a multiple of the column-tile count), so
//     the column tile's slice of a is staged in shared memory once when the rank fits one
//     32-step chunk. Each (tile, chunk) step's slices of a (32 x 128) and b (32 rows x 32
//     steps, transposed) are double-buffered with cp.async: the next step's copies are in
//     flight while the current one computes. A thread owns 4 rows x 4 consecutive columns
//     (the 8 lanes of a quarter warp cover one 32-column group of one row); its code bytes
//     and scales are loaded into registers one tile ahead and used by the epilogue,
//     which dequantizes, adds c * t, reduces each group's amax over its 8 lanes by shuffles
//     and writes codes and scale. A code byte belongs to one group and a tile to one CTA, so
//     the output may overwrite the input.
#include <cfloat>

#include "w4_internal.cuh"

namespace w4i {

namespace {

constexpr int kLoraThreads = 256;
constexpr int kLoraRows = 32;     // tile rows: 8 warps x 4 rows
constexpr int kLoraCols = 128;    // tile columns: 4 groups of 32
constexpr int kLoraChunk = 32;    // rank steps staged at a time
constexpr int kLoraBPitch = 36;   // b slice row pitch (floats): 16-B aligned rows for the float4 reads
constexpr int kLoraCtasPerSm = 2;

struct LoraSmem {
  float a[2][kLoraChunk][kLoraCols];    // a[j0 + jj][k0 + cc]
  float b[2][kLoraChunk][kLoraBPitch];  // b[n0 + rr][j0 + jj] at [jj][rr]
};

__device__ __forceinline__ void cp_async4(float *dst, const float *src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int Pending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(Pending) : "memory");
}

// t[i][e] = fl32(t[i][e] + fl32(b[row i][j] * a[j][column e])) for one rank step j
__device__ __forceinline__ void lora_rank_step(const float *a_row, const float *b_row, int cl, int rl,
                                               float (&t)[4][4]) {
  const float4 av = *reinterpret_cast<const float4 *>(a_row + cl);
  const float4 bv = *reinterpret_cast<const float4 *>(b_row + rl);
  const float aa[4] = {av.x, av.y, av.z, av.w};
  const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) t[i][e] = __fadd_rn(t[i][e], __fmul_rn(bb[i], aa[e]));
}

// signed value of nibble e of a code word, as an exact fp32: (u ^ 8) - 8 through the 2^23 bias
// (the bias's bits and the nibble's are disjoint, so one xor sets both)
__device__ __forceinline__ float lora_code(uint32_t word, int e) {
  return __fsub_rn(__uint_as_float(((word >> (4 * e)) & 15u) ^ 0x4B000008u), 8388616.0f);
}

// max that returns NaN when either input is NaN, so a group's amax carries a NaN merged value
__device__ __forceinline__ float lora_max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// code nibble of round-half-even(fl32(w / s2)), where |w / s2| < 8 (|w| <= amax, s2 >= amax / 7).
// With y = fl32(1 / s2), x = fl32(w * y) lies within 2^-20 of w / s2 and fl32(w / s2) within
// 2^-22 of it, so both round to the same integer unless x is within 2^-19 of a half-integer;
// `near` is raised inside a 2^-18 band around one, and the caller then forms the exact
// quotient instead (lora_rtn_nibble_exact). Adding 1.5 * 2^23 rounds to an integer, half to
// even, and leaves its two's-complement nibble in the low bits.
__device__ __forceinline__ uint32_t lora_rtn_nibble(float w, float y, bool &near) {
  const float x = __fmul_rn(w, y);
  const float xm = __fadd_rn(x, 12582912.0f);
  near |= fabsf(__fsub_rn(x, __fsub_rn(xm, 12582912.0f))) > 0.5f - 0x1p-18f;
  return __float_as_uint(xm) & 15u;
}

__device__ __forceinline__ uint32_t lora_rtn_nibble_exact(float w, float s2) {
  return __float_as_uint(__fadd_rn(__fdiv_rn(w, s2), 12582912.0f)) & 15u;
}

__global__ void __launch_bounds__(kLoraThreads, kLoraCtasPerSm)
    lora_merge_kernel(const uint8_t *codes, const float *scales, const float *__restrict__ b,
                      const float *__restrict__ a, int64_t N, int64_t K, int64_t r, float c, uint8_t *codes_out,
                      float *scales_out, int32_t *__restrict__ status) {
  __shared__ __align__(16) LoraSmem sm;
  const int64_t G = (K + 31) / 32;
  const int64_t P = (K + 1) / 2;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int cl = 32 * (lane >> 3) + 4 * (lane & 7);  // first of the thread's 4 columns in the tile
  const int rl = 4 * (tid >> 5);                     // first of the thread's 4 rows in the tile
  // the grid is (column tiles) x (row-tile walkers); a CTA keeps column tile ct and takes row
  // tiles rt0, rt0 + walkers, ...
  const int64_t col_tiles = (K + kLoraCols - 1) / kLoraCols;
  const int64_t row_tiles = (N + kLoraRows - 1) / kLoraRows;
  const int64_t walkers = gridDim.x / col_tiles;
  const int64_t ct = blockIdx.x % col_tiles, rt0 = blockIdx.x / col_tiles;
  const int64_t my_tiles = (row_tiles - rt0 + walkers - 1) / walkers;
  const int64_t k0 = ct * kLoraCols;
  const int64_t c0 = k0 + cl;  // the thread's first column; all four share one group
  const int ncols = c0 >= K ? 0 : (K - c0 >= 4 ? 4 : static_cast<int>(K - c0));
  const int64_t g = c0 / 32;
  const int64_t jb = c0 / 2;  // code bytes jb (columns c0, c0+1) and jb+1
  const bool two_bytes = jb + 1 < P;  // false: columns c0 + 2, c0 + 3 are past K
  const int nch = static_cast<int>((r + kLoraChunk - 1) / kLoraChunk);
  int a_tag0 = -1, a_tag1 = -1;  // the chunk each a buffer holds; block-uniform

  // stage (row tile it, chunk ch) into buffers buf
  auto issue = [&](int64_t it, int ch, int buf) {
    const int64_t n0 = (rt0 + it * walkers) * kLoraRows;
    const int64_t j0 = static_cast<int64_t>(ch) * kLoraChunk;
    if ((buf ? a_tag1 : a_tag0) != ch) {
      if (buf) a_tag1 = ch; else a_tag0 = ch;
      const int cc = tid % kLoraCols;
      const bool col_ok = k0 + cc < K;
#pragma unroll 4
      for (int jj = tid / kLoraCols; jj < kLoraChunk; jj += kLoraThreads / kLoraCols) {
        const bool ok = col_ok && j0 + jj < r;
        cp_async4(&sm.a[buf][jj][cc], ok ? a + (j0 + jj) * K + k0 + cc : a, ok);
      }
    }
    const int jj = tid % kLoraChunk;
#pragma unroll
    for (int rr = tid / kLoraChunk; rr < kLoraRows; rr += kLoraThreads / kLoraChunk) {
      const bool ok = j0 + jj < r && n0 + rr < N;
      cp_async4(&sm.b[buf][jj][rr], ok ? b + (n0 + rr) * r + j0 + jj : b, ok);
    }
    cp_async_commit();
  };
  // the thread's two code bytes per row and scales of row tile it. The addresses are clamped
  // into the arrays and the loads are unconditional, so nothing consumes a loaded value before
  // the epilogue of the tile (which discards rows and columns outside the weight): the loads
  // of the next tile stay in flight through this tile's rank loop.
  const int64_t jb_lo = jb < P - 1 ? jb : P - 1;
  const int64_t jb_hi = jb + 1 < P - 1 ? jb + 1 : P - 1;
  const int64_t g_in = g < G - 1 ? g : G - 1;
  auto load_tile = [&](int64_t it, uint32_t (&lo)[4], uint32_t (&hi)[4], float (&sc)[4]) {
    const int64_t n0 = (rt0 + it * walkers) * kLoraRows;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t n = n0 + rl + i < N ? n0 + rl + i : N - 1;
      const uint8_t *crow = codes + n * P;
      lo[i] = crow[jb_lo];
      hi[i] = crow[jb_hi];
      sc[i] = scales[n * G + g_in];
    }
  };

  if (my_tiles <= 0) return;
  bool bad = false;  // a non-finite merged value was seen
  uint32_t lo[4], hi[4];
  float sc[4];
  load_tile(0, lo, hi, sc);
  if (nch > 0) issue(0, 0, 0);
  int buf = 0;
  for (int64_t it = 0; it < my_tiles; ++it) {
    uint32_t lo_next[4], hi_next[4];
    float sc_next[4];
    load_tile(it + 1 < my_tiles ? it + 1 : it, lo_next, hi_next, sc_next);
    float t[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) t[i][e] = 0.0f;
    for (int ch = 0; ch < nch; ++ch) {
      const bool last_step = ch + 1 == nch && it + 1 == my_tiles;
      if (!last_step) {
        issue(ch + 1 == nch ? it + 1 : it, ch + 1 == nch ? 0 : ch + 1, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // this step's slices are in shared memory for every thread
      const int64_t left = r - static_cast<int64_t>(ch) * kLoraChunk;
      const int jn = static_cast<int>(left < kLoraChunk ? left : kLoraChunk);
      int jj = 0;
      for (; jj + 8 <= jn; jj += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) lora_rank_step(sm.a[buf][jj + u], sm.b[buf][jj + u], cl, rl, t);
      }
      for (; jj < jn; ++jj) lora_rank_step(sm.a[buf][jj], sm.b[buf][jj], cl, rl, t);
      __syncthreads();  // buffers buf are free for the step after next
      buf ^= 1;
    }
    // epilogue: w' = fl32(fl32(q * s) + fl32(c * t)), then RTN over each row's group.
    // Columns past K have zero codes (masked here) and t = 0 (zero-filled a), so w' = 0 there;
    // rows past N repeat row N - 1 (clamped loads) and are never stored.
    const int64_t n0 = (rt0 + it * walkers) * kLoraRows;
    const uint32_t colmask = ncols >= 4 ? 0xFFFFu : ((1u << (4 * ncols)) - 1u);
    float am[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t word = (lo[i] | (hi[i] << 8)) & colmask;
      am[i] = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        t[i][e] = __fadd_rn(__fmul_rn(lora_code(word, e), sc[i]), __fmul_rn(c, t[i][e]));  // t now holds w'
        am[i] = lora_max_nan(am[i], fabsf(t[i][e]));
      }
    }
    // the 8 lanes of a quarter warp hold one group of each of the 4 rows: reduce the amax
    // (NaN-propagating, so a non-finite merged value shows in its row's amax), then lane
    // (sub & 3) of the group forms row (sub & 3)'s scale and reciprocal for all
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      am[i] = lora_max_nan(am[i], __shfl_xor_sync(0xffffffffu, am[i], 1));
      am[i] = lora_max_nan(am[i], __shfl_xor_sync(0xffffffffu, am[i], 2));
      am[i] = lora_max_nan(am[i], __shfl_xor_sync(0xffffffffu, am[i], 4));
    }
    const int pick = lane & 3;
    const float mine = pick == 0 ? am[0] : (pick == 1 ? am[1] : (pick == 2 ? am[2] : am[3]));
    bad |= !(mine <= FLT_MAX);  // a NaN or infinite merged value in the row's group
    const float s2_mine = fmaxf(__fdiv_rn(mine, 7.0f), FLT_MIN);
    const float y_mine = __frcp_rn(s2_mine);
    float s2[4], y[4];
    uint32_t packed[4];
    bool near = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s2[i] = __shfl_sync(0xffffffffu, s2_mine, (lane & ~7) | i);
      y[i] = __shfl_sync(0xffffffffu, y_mine, (lane & ~7) | i);
      packed[i] = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) packed[i] |= lora_rtn_nibble(t[i][e], y[i], near) << (4 * e);
    }
    if (near) {  // rare: a value close to a half-integer takes the exact quotient
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        packed[i] = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) packed[i] |= lora_rtn_nibble_exact(t[i][e], s2[i]) << (4 * e);
      }
    }
    // columns past K keep a zero pad nibble. The output may alias the input: a lane writes
    // only the two code bytes it read itself, and the group's scale, read by its eight lanes
    // before the shuffles, is written after
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t n = n0 + rl + i;
      if (n < N && ncols > 0) {
        const uint32_t v = packed[i] & colmask;
        uint8_t *orow = codes_out + n * P;
        orow[jb] = static_cast<uint8_t>(v);
        if (two_bytes) orow[jb + 1] = static_cast<uint8_t>(v >> 8);
        if ((lane & 7) == 0) scales_out[n * G + g] = s2[i];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo[i] = lo_next[i];
      hi[i] = hi_next[i];
      sc[i] = sc_next[i];
    }
  }
  if (bad) *status = W4_ERR_NONFINITE;
}

}  // namespace

cudaError_t launch_lora_merge(const uint8_t *codes, const float *scales, const float *lora_b_t,
                              const float *lora_a_t, int64_t N, int64_t K, int64_t r, float alpha_over_rank,
                              uint8_t *codes_out, float *scales_out, int32_t *status, cudaStream_t stream) {
  // grid: every column tile times as many row-tile walkers as fill the resident slots; a CTA
  // keeps its column tile because the grid is a multiple of the column-tile count
  const int64_t col_tiles = (K + kLoraCols - 1) / kLoraCols;
  const int64_t row_tiles = (N + kLoraRows - 1) / kLoraRows;
  const int64_t slots = 148LL * kLoraCtasPerSm;
  int64_t walkers = slots / col_tiles;
  if (walkers > row_tiles) walkers = row_tiles;
  if (walkers < 1) walkers = 1;
  const int64_t blocks = col_tiles * walkers;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  lora_merge_kernel<<<static_cast<unsigned>(blocks), kLoraThreads, 0, stream>>>(
      codes, scales, lora_b_t, lora_a_t, N, K, r, alpha_over_rank, codes_out, scales_out, status);
  return cudaGetLastError();
}

}  // namespace w4i

// Decode GEMV / small-M linear (M <= 16) on register-fed tensor cores, fed by TMA:
//   y[m][n] = sum_k x[m][k] * (q[n][k] * s[n][k/32]) + b[n]
//
// The weight stream (0.625 B per weight) is the whole cost, so the design goal is to keep
// HBM busy with as few issue slots per weight as possible:
//   * one or two CTAs per SM (two when their shared memory fits), each owning a balanced
//     contiguous range of 16-row blocks; a single producer thread walks them in (row block,
//     2048-column chunk) order and fills a ring of 20 KB shared-memory stages with TMA boxes
//     of codes and scales, all with the 128-byte swizzle (conflict-free reads below). The
//     boxes carry the L2 evict-first policy: weights are read once per call, so they should
//     not push the activations (this call's x, the next call's input) out of L2 -- an x
//     that has to come back from HBM behind the weight stream costs ~1 us per launch;
//   * eight consumer warps take one 256-column k-tile of each stage. Per 32-column group a
//     lane holds one code word of row g and one of row g + 8 (ldmatrix.x4 fetches four such
//     words, two groups, in one instruction); LOP3 drops each nibble pair into the mantissa
//     of the bf16 128.0 and one exact bf16x2 FMA removes the offset, which gives the exact
//     integers q as the A fragment of mma.sync m16n8k16 (bf16 in, fp32 accumulate). The
//     activations are the B fragment: with M = 1 every MMA column carries x (broadcast),
//     otherwise column n of n-tile j carries activation row 8j + n. Two MMAs cover a group;
//     the group's fp32 scale multiplies the fp32 group sum in one FFMA per accumulator, so
//     the only rounding besides fp32 accumulation is that of the scale product -- no bf16
//     rounding of dequantized weights. At M = 1 the inner loop is about 1.75
//     thread-instructions per weight (a CUDA-core dot product needs ~4.5);
//   * x arrives by one bulk copy per activation row, issued as soon as the grid dependency
//     resolves, and is permuted in place (within each 16-byte chunk) into fragment order;
//   * per row block the warps' partial sums meet in shared memory and are added in a fixed
//     order (deterministic), the bias is added and y is written: with several activation
//     rows by a reducer warp fed through two mbarrier-guarded buffers (the consumers never
//     wait on one another), with one row by one consumer warp after a named barrier.
// Launch overlap: the kernel is launched with programmatic stream serialization and lets
// its successor launch at once. It reads x and writes y only after the grid dependency has
// resolved; when weight prefetch is enabled it streams codes and scales before that, so a
// chain of decode GEMVs (constant weights) overlaps each kernel's ramp-up with the tail of
// the previous one. Every wait is bounded (w4_sync.cuh).
#include <cuda.h>

#include <mutex>

#include "w4_mma.cuh"
#include "w4_tc.cuh"
#include "w4_tmap.h"

namespace w4i {

namespace {

constexpr int kWarps = 8;  // consumer warps for M = 1 and 9 <= M <= 16 (the producer is one more warp)
constexpr int kRowsPerBlock = 16;            // one m16 MMA tile of weight rows
constexpr int kKtileCodeBytes = 128;         // 256 columns = 8 groups per k-tile
constexpr int kCodeBox = kRowsPerBlock * kKtileCodeBytes;  // 2 KB
constexpr int kScaleBox = kRowsPerBlock * 32 * 4;          // 2 KB: 32 scales = 4 k-tiles per row
// Consumer warps per CTA: 16 for 2 <= M <= 8 (one CTA per SM: its activations take the
// shared memory a second CTA would need, so the warps come from one CTA), else 8. A stage
// holds one k-tile per consumer warp.
constexpr int warps_for(int nt) { return nt == 1 ? 16 : kWarps; }
constexpr int stage_bytes(int w, bool ch = false) { return w * kCodeBox + (ch ? 0 : (w / 4) * kScaleBox); }
// Several activation rows: a reducer warp adds the consumer warps' row-block sums, so the
// consumers never wait on each other (a row block is one or two stages there). One row: the
// consumers meet at a named barrier per row block and one of them adds (measured 1-3% faster
// than a reducer warp at M = 1, which costs a warp slot per CTA).
constexpr bool async_reduce(int nt) { return nt != 0; }
constexpr int block_threads(int nt) { return 32 * (warps_for(nt) + 1 + (async_reduce(nt) ? 1 : 0)); }
constexpr int kMaxStages = 8;
constexpr int kBarBytes = (2 * kMaxStages + 1 + 4) * 8 + 16;  // ring, x, reduction ring (2 x 2)
constexpr int kAlignSlack = 1024;
// Two CTAs per SM when each fits in this much shared memory (16 consumer warps hide more
// latency than 8); a successor launch's CTAs move in as these exit.
constexpr int kTwoPerSmSmem = 112 * 1024;
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxM = 16;
constexpr int kBarConsumers = 1;  // named barrier of the consumer warps
constexpr int kXBatch = 8;        // x chunks in flight per consumer thread (M = 1, K <= 16384 at once)
constexpr int kGatherChunks = 8;  // act-order, one row gathered in the kernel: K <= 8 * 8 * 256

struct TmaGemvParams {
  const __nv_bfloat16 *x;
  const float *bias;
  void *y;
  // asymmetric act-order only (codes sorted by group, x gathered through perm)
  const float *scales;    // [N, n_groups]
  const int8_t *zeros;    // [N, n_groups]
  const int32_t *g_idx;   // [K], group of an original column
  const int32_t *perm;    // [K], original column at each sorted position
  int n_groups;
  int asym_staged;        // 1: each stage also carries the row block's scales and zero points
  int x_sorted;           // 1: x already gathered into sorted column order (by the caller)
  int64_t N;
  int64_t K;
  int64_t NB;      // 16-row blocks
  int rb_q, rb_r;  // CTA c owns rb_q + (c < rb_r) row blocks starting at c * rb_q + min(c, rb_r)
  int M;           // activation rows
  int KT;          // 256-column k-tiles per row
  int SPR;         // stages per row block: ceil(KT / 8)
  int S;           // stages in the ring
  int x_stride;    // bytes between activation rows in shared memory: KT * 512 + 64
  int red_floats;  // one buffer of the row-block reduction
  int y_dtype;
  int prefetch;    // stream codes and scales before the grid dependency resolves
  int boxes3d;     // 1: one 3-D box per stage for the codes and one for the scales
  int channel;     // 1: one scale per row (scales [N]); applied once to the row's sum
};

__device__ __forceinline__ void store_y(const TmaGemvParams &p, int64_t m, int64_t n, float v) {
  if (p.channel) v *= __ldg(p.scales + n);  // per-channel: the row's sum of code * x, scaled once
  if (p.bias) v += __ldcg(p.bias + n);
  if (p.y_dtype == W4_F32)
    static_cast<float *>(p.y)[m * p.N + n] = v;
  else
    static_cast<__nv_bfloat16 *>(p.y)[m * p.N + n] = __float2bfloat16_rn(v);
}

// One sorted 32-column chunk whose columns belong to two or more groups (asymmetric
// act-order codes with group boundaries that are not multiples of 32): lane (g, t) takes
// its 8 columns of rows g and g + 8 on CUDA cores, exact per-column dequantization, and
// the four lanes of a row pool their sums. Returns the chunk's sum for (row, token)
// through `out[r][m]` (r = 0: row g, 1: row g + 8) in every lane of the row.
template <int MT>
__device__ void mixed_chunk(const TmaGemvParams &p, int64_t row_g, int c, int t, uint32_t w_g, uint32_t w_g8,
                            const uint8_t *xs, float (&out)[2][MT]) {
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) out[r][m] = 0.0f;
  for (int e = 0; e < 8; ++e) {
    const int64_t col = 32 * static_cast<int64_t>(c) + 8 * t + e;
    if (col >= p.K) break;
    const int gc = __ldg(p.g_idx + __ldg(p.perm + col));
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int64_t n = row_g + 8 * r;
      if (n >= p.N) continue;
      const int u = static_cast<int>(((r ? w_g8 : w_g) >> (4 * e)) & 15u);
      const float wv = __fmul_rn(static_cast<float>(u - __ldg(p.zeros + n * p.n_groups + gc)),
                                 __ldg(p.scales + n * p.n_groups + gc));
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= p.M) break;
        // x chunk (c, t) in fragment order: pairs (x0,x4) (x1,x5) (x2,x6) (x3,x7)
        const uint32_t pair = reinterpret_cast<const uint32_t *>(xs + m * p.x_stride)[(c * 4 + t) * 4 + (e & 3)];
        const float xv = __uint_as_float((e < 4 ? (pair & 0xFFFFu) : (pair >> 16)) << 16);
        out[r][m] = fmaf(wv, xv, out[r][m]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      out[r][m] += __shfl_xor_sync(0xffffffffu, out[r][m], 1);
      out[r][m] += __shfl_xor_sync(0xffffffffu, out[r][m], 2);
    }
}

// Staged act-order scales [16 rows][n_groups] and zero points [16 rows][n_groups] (one TMA box
// each per stage, n_groups 16 or 32). The boxes are swizzled so that the eight rows a warp's
// lane quads read for one group fall on distinct banks: scales with the 128-byte (32
// groups: 128-byte rows) or 64-byte (16 groups) pattern, zero points with the 32-byte
// pattern (32 groups; 16-byte rows need none). The patterns XOR the 16-byte chunk index with
// address bits 7 and up of the 1024/512/256-byte aligned box.
__device__ __forceinline__ float staged_scale(const uint8_t *sa, int n_groups, int r, int j) {
  const uint32_t off =
      n_groups == 32 ? static_cast<uint32_t>(r * 128 + ((((j >> 2) ^ (r & 7)) << 4) | ((j & 3) << 2)))
                     : static_cast<uint32_t>(r * 64 + ((((j >> 2) ^ ((r >> 1) & 3)) << 4) | ((j & 3) << 2)));
  return *reinterpret_cast<const float *>(sa + off);
}

__device__ __forceinline__ uint32_t staged_zero(const uint8_t *za, int n_groups, int r, int j) {
  const uint32_t off = n_groups == 32
                           ? static_cast<uint32_t>(r * 32 + ((((j >> 4) ^ ((r >> 2) & 1)) << 4) | (j & 15)))
                           : static_cast<uint32_t>(r * 16 + j);
  return za[off];
}

// a + c for bf16x2 pairs as one exact FMA (a * 1.0 + c).
__device__ __forceinline__ uint32_t bf16x2_add1(uint32_t a, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(0x3F803F80u), "r"(c));
  return d;
}

// One code word of unsigned nibbles -> the exact integers u - z. nzz is the bf16x2 pair
// (-(128 + z), -(128 + z)) of the row's zero point z for the chunk's group, formed once per
// group, so each nibble pair costs one LOP3 (u into the mantissa of 128.0) and one exact FMA.
__device__ __forceinline__ void unpack_asym(uint32_t w, uint32_t nzz, uint32_t (&a)[4]) {
  a[0] = bf16x2_add1(nib_pair_bf16(w, 0x43004300u), nzz);
  a[1] = bf16x2_add1(nib_pair_bf16(w >> 4, 0x43004300u), nzz);
  a[2] = bf16x2_add1(nib_pair_bf16(w >> 8, 0x43004300u), nzz);
  a[3] = bf16x2_add1(nib_pair_bf16(w >> 12, 0x43004300u), nzz);
}

// NT = 0: M = 1, x broadcast to every MMA column. NT = 1, 2: up to 8 NT activation rows,
// one per MMA column of each n-tile. ASYM: unsigned codes sorted by group (act-order),
// per-(row, group) scale and zero point read through a per-CTA group table. CH: symmetric
// codes with one scale per row (per-channel): the stages carry codes only, the group sums
// are added unscaled and the row's scale multiplies its final sum.
template <int NT, bool ASYM, bool CH>
__global__ void __launch_bounds__(block_threads(NT), NT == 0 ? 2 : 1)
    gemv_tma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
                    const __grid_constant__ CUtensorMap tm_zeros, const TmaGemvParams p, int32_t *err) {
  constexpr int W = warps_for(NT);            // consumer warps = k-tiles per stage
  constexpr int SB = stage_bytes(W, CH);      // bytes per stage
  constexpr int kTok = NT == 0 ? 1 : 8 * NT;  // token slots of the reduction buffer
  constexpr int kAcc = NT == 0 ? 1 : NT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // 1024-byte swizzle atoms
  uint8_t *xs = smem + p.S * SB;
  float *red = reinterpret_cast<float *>(xs + p.M * p.x_stride);
  int32_t *gtab = reinterpret_cast<int32_t *>(red + 2 * p.red_floats);  // ASYM: group of each chunk
  int32_t *gtab4 = gtab + p.KT * 8;  // ASYM: group of each 128-column half k-tile (-1: several)
  uint64_t *full = reinterpret_cast<uint64_t *>(gtab + (ASYM ? p.KT * 10 : 0));
  uint64_t *empty = full + kMaxStages;
  uint64_t *x_full = empty + kMaxStages;
  uint64_t *red_full = x_full + 1;  // two reduction buffers: the consumer warps' sums written
  uint64_t *red_empty = red_full + 2;  // ... and read by the reducer warp
  volatile int *abort_flag = reinterpret_cast<volatile int *>(red_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = static_cast<int>(blockIdx.x);
  const int64_t rb_begin = static_cast<int64_t>(cta) * p.rb_q + (cta < p.rb_r ? cta : p.rb_r);
  const int nrb = p.rb_q + (cta < p.rb_r ? 1 : 0);  // row blocks of this CTA
  const int total = nrb * p.SPR;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], W);
    }
    mbar_init(x_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&red_full[i], W);
      mbar_init(&red_empty[i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  grid_launch_dependents();

  if (warp == W) {
    // ---- producer: one thread issues every TMA box of the CTA's row blocks ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int slot = 0, kc = 0;
      uint32_t phase = 0;
      int32_t row = static_cast<int32_t>(rb_begin * kRowsPerBlock);
      // weights first when they may be prefetched (they do not depend on the previous kernel)
      const int early = p.prefetch ? (total < p.S ? total : p.S) : 0;
      int issued = 0;        // stages whose copies were issued
      bool x_issued = false;  // the activation copies (several rows)
      for (int i = 0; i <= total; ++i) {
        if (NT != 0 && (!ASYM || p.x_sorted) && i == early) {
          x_issued = true;
          // x is written by the previous kernel: copy it only once that kernel has finished.
          // (M = 1: the consumers load it themselves, in one round trip.)
          grid_dependency_wait();
          mbar_arrive_expect_tx(x_full, static_cast<uint32_t>(p.M * p.K * 2));
          for (int m = 0; m < p.M; ++m)
            bulk_copy_g2s(xs + m * p.x_stride, p.x + m * p.K, static_cast<uint32_t>(p.K * 2), x_full);
        }
        if (i == total) break;
        if ((NT == 0 || (ASYM && !p.x_sorted)) && i == early && !p.prefetch) grid_dependency_wait();
        if (!mbar_wait(&empty[slot], phase ^ 1u, abort_flag, err)) break;
        const int kt0 = kc * W;
        const int nkt = (p.KT - kt0) < W ? (p.KT - kt0) : W;
        const int nsb = (nkt + 3) / 4;
        uint8_t *st = smem + slot * SB;
        if (ASYM) {
          // codes, and (staged layout) the row block's scales and zero points of every group
          const uint32_t sz = p.asym_staged ? static_cast<uint32_t>(kRowsPerBlock * p.n_groups * 5) : 0u;
          if (p.boxes3d) {
            mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(W * kCodeBox) + sz);
            tma_load_3d_hint(st, &tm_codes, 0, row, kt0, &full[slot], pol);
          } else {
            mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nkt * kCodeBox) + sz);
            for (int j = 0; j < nkt; ++j)
              tma_load_2d_hint(st + j * kCodeBox, &tm_codes, (kt0 + j) * kKtileCodeBytes, row, &full[slot], pol);
          }
          if (p.asym_staged) {
            uint8_t *sa = st + W * kCodeBox;
            tma_load_2d_hint(sa, &tm_scales, 0, row, &full[slot], pol);
            tma_load_2d_hint(sa + kRowsPerBlock * p.n_groups * 4, &tm_zeros, 0, row, &full[slot], pol);
          }
        } else if (p.boxes3d) {
          // whole-stage boxes; k-tiles past the row end read as zeros (and count as bytes)
          mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(SB));
          tma_load_3d_hint(st, &tm_codes, 0, row, kt0, &full[slot], pol);
          if (!CH) tma_load_3d_hint(st + W * kCodeBox, &tm_scales, 0, row, kt0 / 4, &full[slot], pol);
        } else {
          mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nkt * kCodeBox + (CH ? 0 : nsb * kScaleBox)));
          for (int j = 0; j < nkt; ++j)
            tma_load_2d_hint(st + j * kCodeBox, &tm_codes, (kt0 + j) * kKtileCodeBytes, row, &full[slot], pol);
          if (!CH)
            for (int b = 0; b < nsb; ++b)
              tma_load_2d_hint(st + W * kCodeBox + b * kScaleBox, &tm_scales, (kt0 + 4 * b) * 8, row,
                               &full[slot], pol);
        }
        issued = i + 1;
        if (++kc == p.SPR) {
          kc = 0;
          row += kRowsPerBlock;
        }
        if (++slot == p.S) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // every copy issued must land before the CTA may exit (the consumers stop waiting on
      // an abort): the last S stages hold distinct slots, each at its latest phase
      for (int i = issued - p.S < 0 ? 0 : issued - p.S; i < issued; ++i)
        mbar_drain(&full[i % p.S], static_cast<uint32_t>(i / p.S) & 1u, err);
      if (x_issued) mbar_drain(x_full, 0u, err);
    }
    return;
  }

  if (async_reduce(NT) && warp == W + 1) {
    // ---- reducer: per row block, the W consumer warps' sums (buffer [warp][token][16 rows])
    // are added in warp order (deterministic), the bias added and y written; the buffer is
    // then handed back. The consumers never wait on each other. ----
    grid_dependency_wait();  // y may be read by the previous kernel
    const int64_t rows0 = rb_begin * kRowsPerBlock;
    for (int b = 0; b < nrb; ++b) {
      const int rbuf = b & 1;
      mbar_wait(&red_full[rbuf], static_cast<uint32_t>(b >> 1) & 1u, abort_flag, err);
      const float *r = red + rbuf * p.red_floats;
      for (int e = lane; e < p.M * kRowsPerBlock; e += 32) {
        const int m = e / kRowsPerBlock, rr = e % kRowsPerBlock;
        const int64_t n = rows0 + static_cast<int64_t>(b) * kRowsPerBlock + rr;
        if (n < p.N) {
          float v = 0.0f;
#pragma unroll
          for (int w2 = 0; w2 < W; ++w2) v += r[(w2 * kTok + m) * kRowsPerBlock + rr];
          store_y(p, m, n, v);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_empty[rbuf]);
    }
    return;
  }

  // ---- consumers: x -> B-fragment order; the tail past K (up to a whole k-tile) is
  // cleared. Chunk c of a row holds columns (8c + e, 8c + e + 4) for e = 0..3. ----
  if (ASYM) {
    // act-order: the group of every sorted 32-column chunk (-1: the chunk straddles groups;
    // -2: past K). perm and g_idx are weights (constant).
    for (int c = threadIdx.x; c < p.KT * 8; c += 32 * W) {
      int gv = -2;
      if (32 * static_cast<int64_t>(c) < p.K) {
        const int64_t c0 = 32 * static_cast<int64_t>(c);
        const int64_t c1 = (c0 + 31 < p.K) ? c0 + 31 : p.K - 1;
        const int g0 = __ldg(p.g_idx + __ldg(p.perm + c0));
        gv = g0 == __ldg(p.g_idx + __ldg(p.perm + c1)) ? g0 : -1;
      }
      gtab[c] = gv;
    }
    for (int h = threadIdx.x; h < p.KT * 2; h += 32 * W) {
      int gv = -1;
      const int64_t c0 = 128 * static_cast<int64_t>(h), c1 = c0 + 127;
      if (c1 < p.K) {
        // sorted by group: the first and last column decide whether one group spans the block
        const int g0 = __ldg(p.g_idx + __ldg(p.perm + c0));
        if (g0 == __ldg(p.g_idx + __ldg(p.perm + c1))) gv = g0;
      }
      gtab4[h] = gv;
    }
  }
  if (ASYM && !p.x_sorted) {
    // one activation row gathered through perm by every CTA (host: M = 1, at most
    // kGatherChunks chunks per thread): x is copied in coalesced 16-byte pieces into the
    // activation buffer, each thread gathers its chunks from there into registers (perm, a
    // weight, is read before the grid dependency), then writes them back in fragment order.
    const int per_row = p.KT * 32, valid = static_cast<int>(p.K / 8);
    uint4 *xr = reinterpret_cast<uint4 *>(xs);
    const uint16_t *xh = reinterpret_cast<const uint16_t *>(xs);
    // this thread's column indices (a weight: the first kHoist chunks' are read before the
    // wait, which covers K <= 4096; longer rows read the rest after it)
    constexpr int kHoist = 2;
    int4 pc[kHoist][2];
#pragma unroll
    for (int k = 0; k < kHoist; ++k) {
      const int c = static_cast<int>(threadIdx.x) + k * 32 * W;
      if (c < valid) {
        pc[k][0] = __ldg(reinterpret_cast<const int4 *>(p.perm) + 2 * c);
        pc[k][1] = __ldg(reinterpret_cast<const int4 *>(p.perm) + 2 * c + 1);
      } else {
        pc[k][0] = pc[k][1] = make_int4(0, 0, 0, 0);
      }
    }
    grid_dependency_wait();
    for (int c = threadIdx.x; c < valid; c += 32 * W) xr[c] = __ldcg(reinterpret_cast<const uint4 *>(p.x) + c);
    named_barrier_sync(kBarConsumers, 32 * W);
    uint4 v[kGatherChunks];
#pragma unroll
    for (int k = 0; k < kGatherChunks; ++k) {
      const int c = static_cast<int>(threadIdx.x) + k * 32 * W;
      v[k] = make_uint4(0u, 0u, 0u, 0u);
      if (c < valid) {
        int4 p0, p1;
        if (k < kHoist) {
          p0 = pc[k < kHoist ? k : 0][0];
          p1 = pc[k < kHoist ? k : 0][1];
        } else {
          p0 = __ldg(reinterpret_cast<const int4 *>(p.perm) + 2 * c);
          p1 = __ldg(reinterpret_cast<const int4 *>(p.perm) + 2 * c + 1);
        }
        const uint32_t r0 = xh[p0.x] | (static_cast<uint32_t>(xh[p0.y]) << 16);
        const uint32_t r1 = xh[p0.z] | (static_cast<uint32_t>(xh[p0.w]) << 16);
        const uint32_t r2 = xh[p1.x] | (static_cast<uint32_t>(xh[p1.y]) << 16);
        const uint32_t r3 = xh[p1.z] | (static_cast<uint32_t>(xh[p1.w]) << 16);
        v[k].x = prmt(r0, r2, 0x5410);
        v[k].y = prmt(r0, r2, 0x7632);
        v[k].z = prmt(r1, r3, 0x5410);
        v[k].w = prmt(r1, r3, 0x7632);
      }
    }
    named_barrier_sync(kBarConsumers, 32 * W);
#pragma unroll
    for (int k = 0; k < kGatherChunks; ++k) {
      const int c = static_cast<int>(threadIdx.x) + k * 32 * W;
      if (c < per_row) xr[c] = v[k];
    }
  } else if (NT == 0) {
    // one activation row (already in sorted order for act-order codes): every thread issues
    // all its loads before using any (one memory
    // round trip), straight from global memory once the previous kernel has finished
    grid_dependency_wait();
    const int per_row = p.KT * 32, valid = static_cast<int>(p.K / 8);
    const uint4 *x4 = reinterpret_cast<const uint4 *>(p.x);
    uint4 *xr = reinterpret_cast<uint4 *>(xs);
    for (int base = static_cast<int>(threadIdx.x); base < per_row; base += kXBatch * 32 * W) {
      uint4 r4[kXBatch];
#pragma unroll
      for (int k = 0; k < kXBatch; ++k) {
        const int c = base + k * 32 * W;
        r4[k] = (c < valid) ? __ldcg(x4 + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < kXBatch; ++k) {
        const int c = base + k * 32 * W;
        if (c < per_row) {
          uint4 v;
          v.x = prmt(r4[k].x, r4[k].z, 0x5410);
          v.y = prmt(r4[k].x, r4[k].z, 0x7632);
          v.z = prmt(r4[k].y, r4[k].w, 0x5410);
          v.w = prmt(r4[k].y, r4[k].w, 0x7632);
          xr[c] = v;
        }
      }
    }
  } else {
    // several rows: one bulk copy per row (issued by the producer), permuted in place, eight
    // chunks per thread loaded before any is stored (a chunk-by-chunk pass took 2.4 us for
    // sixteen rows of 4096 columns: each load waited on the previous store)
    mbar_wait(x_full, 0, abort_flag, err);
    const int per_row = p.KT * 32, valid = static_cast<int>(p.K / 8);
    const int chunks = p.M * per_row;
    constexpr int kPerm = 8;
    for (int base = static_cast<int>(threadIdx.x); base < chunks; base += kPerm * 32 * W) {
      uint4 v[kPerm];
#pragma unroll
      for (int k = 0; k < kPerm; ++k) {
        const int i = base + k * 32 * W;
        const int m = i / per_row, c = i - m * per_row;
        v[k] = (i < chunks && c < valid) ? reinterpret_cast<const uint4 *>(xs + m * p.x_stride)[c]
                                         : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < kPerm; ++k) {
        const int i = base + k * 32 * W;
        if (i < chunks) {
          const int m = i / per_row, c = i - m * per_row;
          uint4 o;
          o.x = prmt(v[k].x, v[k].z, 0x5410);
          o.y = prmt(v[k].x, v[k].z, 0x7632);
          o.z = prmt(v[k].y, v[k].w, 0x5410);
          o.w = prmt(v[k].y, v[k].w, 0x7632);
          reinterpret_cast<uint4 *>(xs + m * p.x_stride)[c] = o;
        }
      }
    }
  }
  named_barrier_sync(kBarConsumers, 32 * W);

  const int g = lane >> 2, t = lane & 3;
  const uint32_t stages0 = smem_u32(smem);
  // ldmatrix.x4: lanes 8i .. 8i+7 address the rows of matrix i = (rows 0-7 | rows 8-15) x
  // (group 2p | group 2p+1); the 128-byte swizzle puts 16-byte chunk c of row r at c ^ (r & 7).
  const uint32_t ld_row = static_cast<uint32_t>(((lane & 7) + ((lane >> 3) & 1) * 8) * kKtileCodeBytes);
  const uint32_t ld_xor = static_cast<uint32_t>(lane & 7), ld_hi = static_cast<uint32_t>(lane >> 4);
  // this warp's 8 scales per row: chunks 2(w%4), 2(w%4)+1 of scale box w/4
  const uint32_t sbox = static_cast<uint32_t>(W * kCodeBox + (warp >> 2) * kScaleBox);
  const uint32_t sch = static_cast<uint32_t>(2 * (warp & 3));
  const uint32_t s_lo = static_cast<uint32_t>(g * 128) + ((sch ^ g) << 4);
  const uint32_t s_hi = static_cast<uint32_t>(g * 128) + (((sch + 1) ^ g) << 4);

  uint32_t ld_off[4];  // this lane's four swizzled ldmatrix offsets (q: groups 2q, 2q + 1)
#pragma unroll
  for (int q = 0; q < 4; ++q) ld_off[q] = ld_row + ((((2u * q) + ld_hi) ^ ld_xor) << 4);

  // this lane's activation rows (one per n-tile; NT = 0: row 0 for every lane)
  const uint4 *xrow[kAcc];
  bool xok[kAcc];
#pragma unroll
  for (int j = 0; j < kAcc; ++j) {
    const int m = NT == 0 ? 0 : 8 * j + g;
    xok[j] = m < p.M;
    xrow[j] = reinterpret_cast<const uint4 *>(xs + (xok[j] ? m : 0) * p.x_stride) + t;
  }

  float acc[kAcc][4];
#pragma unroll
  for (int j = 0; j < kAcc; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
  int buf = 0, slot = 0, kc = 0, rbl = 0;
  uint32_t phase = 0;
  int64_t row0 = rb_begin * kRowsPerBlock;
  for (int i = 0; i < total; ++i) {
    mbar_wait(&full[slot], phase, abort_flag, err);
    const int kt = kc * W + warp;
    if (kt < p.KT) {
      const uint32_t st = stages0 + static_cast<uint32_t>(slot * SB);
      const uint32_t cb = st + static_cast<uint32_t>(warp * kCodeBox);
      uint32_t w[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q) ldsm_x4(cb + ld_off[q], w[q]);
      if (!ASYM && CH) {
        // per-channel: the k-tile's group sums added unscaled (the row's scale comes last)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          uint32_t a[4], b[4];
          unpack_signed(w[jj >> 1][(jj & 1) * 2], a);      // row g
          unpack_signed(w[jj >> 1][(jj & 1) * 2 + 1], b);  // row g + 8
#pragma unroll
          for (int j = 0; j < kAcc; ++j) {
            const uint4 xf = (NT == 0 || xok[j]) ? xrow[j][kt * 32 + 4 * jj] : make_uint4(0u, 0u, 0u, 0u);
            float d[4];
            mma_first(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
            mma_next(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
            acc[j][0] += d[0];
            acc[j][2] += d[2];
            if (NT != 0) {
              acc[j][1] += d[1];
              acc[j][3] += d[3];
            }
          }
        }
      } else if (!ASYM) {
        const uint8_t *sp = smem + slot * SB + sbox;
        const uint4 sg0 = *reinterpret_cast<const uint4 *>(sp + s_lo);
        const uint4 sg1 = *reinterpret_cast<const uint4 *>(sp + s_hi);
        const uint4 sh0 = *reinterpret_cast<const uint4 *>(sp + 1024 + s_lo);
        const uint4 sh1 = *reinterpret_cast<const uint4 *>(sp + 1024 + s_hi);
        const float s0[8] = {__uint_as_float(sg0.x), __uint_as_float(sg0.y), __uint_as_float(sg0.z),
                             __uint_as_float(sg0.w), __uint_as_float(sg1.x), __uint_as_float(sg1.y),
                             __uint_as_float(sg1.z), __uint_as_float(sg1.w)};
        const float s1[8] = {__uint_as_float(sh0.x), __uint_as_float(sh0.y), __uint_as_float(sh0.z),
                             __uint_as_float(sh0.w), __uint_as_float(sh1.x), __uint_as_float(sh1.y),
                             __uint_as_float(sh1.z), __uint_as_float(sh1.w)};
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          uint32_t a[4], b[4];
          unpack_signed(w[jj >> 1][(jj & 1) * 2], a);      // row g
          unpack_signed(w[jj >> 1][(jj & 1) * 2 + 1], b);  // row g + 8
#pragma unroll
          for (int j = 0; j < kAcc; ++j) {
            const uint4 xf = (NT == 0 || xok[j]) ? xrow[j][kt * 32 + 4 * jj] : make_uint4(0u, 0u, 0u, 0u);
            float d[4];
            mma_first(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
            mma_next(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
            acc[j][0] = fmaf(d[0], s0[jj], acc[j][0]);
            acc[j][2] = fmaf(d[2], s1[jj], acc[j][2]);
            if (NT != 0) {
              acc[j][1] = fmaf(d[1], s0[jj], acc[j][1]);
              acc[j][3] = fmaf(d[3], s1[jj], acc[j][3]);
            }
          }
        }
      } else if (gtab4[2 * kt] >= 0 && gtab4[2 * kt + 1] >= 0) {
        // act-order, each 128-column half of the k-tile within one group (e.g. groups of
        // 128 or 256 columns): one (scale, zero point) per half and row, no per-chunk branch
        const int64_t row_g = row0 + g;
        float sv[2][2];
        uint32_t zv[2][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int grp = gtab4[2 * kt + h];
          uint32_t z0 = 0u, z1 = 0u;
          if (p.asym_staged) {
            const uint8_t *sa = smem + slot * SB + W * kCodeBox;
            const uint8_t *zr = sa + kRowsPerBlock * p.n_groups * 4;
            sv[h][0] = staged_scale(sa, p.n_groups, g, grp);
            sv[h][1] = staged_scale(sa, p.n_groups, g + 8, grp);
            z0 = staged_zero(zr, p.n_groups, g, grp) & 15u;
            z1 = staged_zero(zr, p.n_groups, g + 8, grp) & 15u;
          } else {
            sv[h][0] = sv[h][1] = 0.0f;
            if (row_g < p.N) {
              sv[h][0] = __ldg(p.scales + row_g * p.n_groups + grp);
              z0 = static_cast<uint32_t>(__ldg(p.zeros + row_g * p.n_groups + grp)) & 15u;
            }
            if (row_g + 8 < p.N) {
              sv[h][1] = __ldg(p.scales + (row_g + 8) * p.n_groups + grp);
              z1 = static_cast<uint32_t>(__ldg(p.zeros + (row_g + 8) * p.n_groups + grp)) & 15u;
            }
          }
          zv[h][0] = ((0x4300u | z0) * 0x00010001u) ^ 0x80008000u;  // -(128 + z) pairs
          zv[h][1] = ((0x4300u | z1) * 0x00010001u) ^ 0x80008000u;
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int h = jj >> 2;
          uint32_t a[4], b[4];
          unpack_asym(w[jj >> 1][(jj & 1) * 2], zv[h][0], a);
          unpack_asym(w[jj >> 1][(jj & 1) * 2 + 1], zv[h][1], b);
#pragma unroll
          for (int j = 0; j < kAcc; ++j) {
            const uint4 xf = (NT == 0 || xok[j]) ? xrow[j][kt * 32 + 4 * jj] : make_uint4(0u, 0u, 0u, 0u);
            float d[4];
            mma_first(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
            mma_next(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
            acc[j][0] = fmaf(d[0], sv[h][0], acc[j][0]);
            acc[j][2] = fmaf(d[2], sv[h][1], acc[j][2]);
            if (NT != 0) {
              acc[j][1] = fmaf(d[1], sv[h][0], acc[j][1]);
              acc[j][3] = fmaf(d[3], sv[h][1], acc[j][3]);
            }
          }
        }
      } else {
        // act-order: each chunk's group from the table; (scale, zero) of rows g and g + 8
        // re-read only when the group changes (consecutive chunks usually share it)
        const int64_t row_g = row0 + g;
        int cur = -3;
        float s0 = 0.0f, s1 = 0.0f;
        uint32_t zz0 = 0xC300C300u, zz1 = 0xC300C300u;  // -(128 + z) pairs
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int c = kt * 8 + jj;
          const int grp = gtab[c];
          if (grp == -2) continue;  // past K
          const uint32_t wg = w[jj >> 1][(jj & 1) * 2], wg8 = w[jj >> 1][(jj & 1) * 2 + 1];
          if (grp >= 0) {
            if (grp != cur) {
              cur = grp;
              uint32_t z0 = 0u, z1 = 0u;
              if (p.asym_staged) {
                // this stage's copy of the row block's scales [16][n_groups] and zeros [16][n_groups]
                const uint8_t *sa = smem + slot * SB + W * kCodeBox;
                const uint8_t *zr = sa + kRowsPerBlock * p.n_groups * 4;
                s0 = staged_scale(sa, p.n_groups, g, grp);
                s1 = staged_scale(sa, p.n_groups, g + 8, grp);
                z0 = staged_zero(zr, p.n_groups, g, grp) & 15u;
                z1 = staged_zero(zr, p.n_groups, g + 8, grp) & 15u;
              } else {
                s0 = s1 = 0.0f;
                if (row_g < p.N) {
                  s0 = __ldg(p.scales + row_g * p.n_groups + grp);
                  z0 = static_cast<uint32_t>(__ldg(p.zeros + row_g * p.n_groups + grp)) & 15u;
                }
                if (row_g + 8 < p.N) {
                  s1 = __ldg(p.scales + (row_g + 8) * p.n_groups + grp);
                  z1 = static_cast<uint32_t>(__ldg(p.zeros + (row_g + 8) * p.n_groups + grp)) & 15u;
                }
              }
              zz0 = ((0x4300u | z0) * 0x00010001u) ^ 0x80008000u;
              zz1 = ((0x4300u | z1) * 0x00010001u) ^ 0x80008000u;
            }
            uint32_t a[4], b[4];
            unpack_asym(wg, zz0, a);
            unpack_asym(wg8, zz1, b);
#pragma unroll
            for (int j = 0; j < kAcc; ++j) {
              const uint4 xf = (NT == 0 || xok[j]) ? xrow[j][c * 4] : make_uint4(0u, 0u, 0u, 0u);
              float d[4];
              mma_first(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
              mma_next(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
              acc[j][0] = fmaf(d[0], s0, acc[j][0]);
              acc[j][2] = fmaf(d[2], s1, acc[j][2]);
              if (NT != 0) {
                acc[j][1] = fmaf(d[1], s0, acc[j][1]);
                acc[j][3] = fmaf(d[3], s1, acc[j][3]);
              }
            }
          } else {
            // the chunk straddles groups: exact per-column path, pooled over the row's lanes
            constexpr int MT = NT == 0 ? 1 : 8 * NT;
            float part[2][MT];
            mixed_chunk<MT>(p, row_g, c, t, wg, wg8, xs, part);
            if (NT == 0) {
              acc[0][0] += part[0][0];
              acc[0][2] += part[1][0];
            } else {
#pragma unroll
              for (int j = 0; j < kAcc; ++j) {
                acc[j][0] += part[0][8 * j + 2 * t];
                acc[j][1] += part[0][8 * j + 2 * t + 1];
                acc[j][2] += part[1][8 * j + 2 * t];
                acc[j][3] += part[1][8 * j + 2 * t + 1];
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == p.S) {
      slot = 0;
      phase ^= 1u;
    }

    if (++kc == p.SPR) {
      // row block complete: this warp's sums go to the reducer through buffer rbl & 1
      // (layout [warp][token][16 rows]) once the reducer has read that buffer's last use
      kc = 0;
      if (async_reduce(NT) && rbl >= 2)
        mbar_wait(&red_empty[buf], static_cast<uint32_t>((rbl >> 1) - 1) & 1u, abort_flag, err);
      float *r = red + buf * p.red_floats;
      if (NT == 0) {
        if (t == 0) {
          r[warp * kRowsPerBlock + g] = acc[0][0];
          r[warp * kRowsPerBlock + g + 8] = acc[0][2];
        }
      } else {
#pragma unroll
        for (int j = 0; j < kAcc; ++j) {
          float *rw = r + (warp * kTok + 8 * j + 2 * t) * kRowsPerBlock;
          rw[g] = acc[j][0];
          rw[kRowsPerBlock + g] = acc[j][1];
          rw[g + 8] = acc[j][2];
          rw[kRowsPerBlock + g + 8] = acc[j][3];
        }
      }
      if (async_reduce(NT)) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[buf]);
      } else {
        named_barrier_sync(kBarConsumers, 32 * W);
        if (warp == (rbl & (W - 1))) {
          for (int e = lane; e < kRowsPerBlock; e += 32) {
            const int64_t n = row0 + e;
            if (n < p.N) {
              float v = 0.0f;
#pragma unroll
              for (int w2 = 0; w2 < W; ++w2) v += r[w2 * kRowsPerBlock + e];
              store_y(p, 0, n, v);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kAcc; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
      buf ^= 1;  // one row: the next block writes the other buffer, two barriers apart from this read
      row0 += kRowsPerBlock;
      ++rbl;
    }
  }
}

int sm_count_current() {
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

// Shapes, alignment and the shared-memory plan; *ctas_per_sm is 1 or 2.
bool make_params(const LinearParams &lp, TmaGemvParams *q, int *smem, int *ctas_per_sm) {
  if (lp.M < 1 || lp.M > kMaxM) return false;
  if (lp.asym && (lp.perm == nullptr || reinterpret_cast<uintptr_t>(lp.perm) % 16 != 0 || lp.n_groups < 1))
    return false;  // act-order codes must be sorted by group (w4_asym_prepare)
  if (lp.K % 128 != 0 || lp.N > 0x7fffffffLL) return false;  // TMA: 16-byte row strides, int32 rows
  if (lp.y_dtype != W4_BF16 && lp.y_dtype != W4_F32) return false;
  if (lp.channel && lp.asym) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(lp.codes) | reinterpret_cast<uintptr_t>(lp.x) |
                      ((lp.asym || lp.channel) ? 0 : reinterpret_cast<uintptr_t>(lp.scales));
  if (a % 16 != 0) return false;
  const int64_t KT = (lp.K + 255) / 256;
  const int64_t x_stride = KT * 512 + 64;  // the 64 bytes keep two rows of a lane quad on distinct banks
  const int64_t tok = lp.M == 1 ? 1 : (lp.M <= 8 ? 8 : 16);
  const int W = warps_for(lp.M == 1 ? 0 : (lp.M <= 8 ? 1 : 2));
  const int64_t SB = stage_bytes(W, lp.channel != 0);
  const int64_t red_floats = W * tok * kRowsPerBlock;
  const int64_t gtab_bytes = lp.asym ? KT * 10 * 4 : 0;
  const int64_t fixed = kAlignSlack + lp.M * x_stride + 2 * red_floats * 4 + gtab_bytes + kBarBytes;
  int64_t S = (kTwoPerSmSmem - fixed) / SB;
  int per_sm = 2;
  if (S < 4) {  // long rows or many activation rows: one CTA per SM, a deeper ring
    S = (kMaxSmem - fixed) / SB;
    per_sm = 1;
  }
  if (S > kMaxStages) S = kMaxStages;
  // One activation row, symmetric codes: at most 3 stages in flight per CTA. With the deeper
  // ring a CTA of several row blocks requests most of its rows at once; every CTA's first
  // stage then lands late and compute overlaps the stream worse ((14336,4096): 8.6 us with
  // 3 stages, 9.7 us with 5; the other shapes unchanged).
  // Per-channel stages carry codes only (16 KB): five of them in flight measured best for
  // the decode step (23.2 us with three or four, 21.8 with five, 22.0 with six).
  const int64_t s_cap = lp.channel ? 5 : 3;
  if (lp.M == 1 && !lp.asym && S > s_cap) S = s_cap;
  if (S < 2) return false;
  q->x = lp.x;
  q->bias = lp.bias;
  q->y = lp.y;
  q->scales = lp.scales;
  q->zeros = lp.zeros;
  q->g_idx = lp.g_idx;
  q->perm = lp.perm;
  q->n_groups = lp.n_groups;
  q->N = lp.N;
  q->K = lp.K;
  q->NB = (lp.N + kRowsPerBlock - 1) / kRowsPerBlock;
  if (q->NB >= (int64_t(1) << 31) / 64) return false;
  q->M = static_cast<int>(lp.M);
  q->KT = static_cast<int>(KT);
  q->SPR = static_cast<int>((KT + W - 1) / W);
  q->S = static_cast<int>(S);
  q->x_stride = static_cast<int>(x_stride);
  q->red_floats = static_cast<int>(red_floats);
  q->y_dtype = lp.y_dtype;
  q->prefetch = 0;
  q->boxes3d = 0;
  q->channel = lp.channel;
  q->asym_staged = 0;
  q->x_sorted = 0;
  *smem = static_cast<int>(fixed + S * SB);
  *ctas_per_sm = per_sm;
  return true;
}

template <int NT, bool ASYM, bool CH>
cudaError_t ensure_smem_attr() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(gemv_tma_kernel<NT, ASYM, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

template <int NT, bool ASYM, bool CH = false>
cudaError_t launch_typed(const CUtensorMap &mc, const CUtensorMap &ms, const CUtensorMap &mz, const TmaGemvParams &q,
                         int smem, int grid, int32_t *err, cudaStream_t stream) {
  cudaError_t e = ensure_smem_attr<NT, ASYM, CH>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(block_threads(NT));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_tma_kernel<NT, ASYM, CH>, mc, ms, mz, q, err);
}

}  // namespace

bool gemv_tma_supports(const LinearParams &p) {
  TmaGemvParams q;
  int smem, per_sm;
  return make_params(p, &q, &smem, &per_sm) && encode_fn() != nullptr;
}

bool gemv_tma_gathers_x(const LinearParams &p) {
  return p.asym && p.M == 1 && (p.K + 255) / 256 * 32 <= static_cast<int64_t>(kGatherChunks) * 32 * kWarps;
}

cudaError_t launch_gemv_tma(const LinearParams &lp, bool prefetch, const __nv_bfloat16 *x_sorted, int32_t *err,
                            cudaStream_t stream) {
  TmaGemvParams q;
  int smem = 0, per_sm = 1;
  if (!make_params(lp, &q, &smem, &per_sm)) return cudaErrorNotSupported;
  q.prefetch = prefetch ? 1 : 0;
  if (lp.asym && x_sorted != nullptr) {
    if (reinterpret_cast<uintptr_t>(x_sorted) % 16 != 0) return cudaErrorInvalidValue;
    q.x = x_sorted;
    q.x_sorted = 1;
  } else if (lp.asym && !gemv_tma_gathers_x(lp)) {
    return cudaErrorInvalidValue;  // several rows (or a long row): x must come gathered
  }
  const int64_t P = lp.K / 2, G = lp.K / 32;
  const int W = warps_for(lp.M == 1 ? 0 : (lp.M <= 8 ? 1 : 2));  // k-tiles per stage
  CUtensorMap mc, ms;
  CUtensorMap mz;
  if (lp.asym) {
    // codes; with at most 32 groups per row (multiple of 16: 16-byte zero rows) each stage
    // also carries the row block's scales and zero points, else the kernel reads them per group
    q.asym_staged = (lp.n_groups == 16 || lp.n_groups == 32) &&
                    reinterpret_cast<uintptr_t>(lp.scales) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(lp.zeros) % 16 == 0 &&
                    make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lp.scales, lp.n_groups, lp.N,
                                lp.n_groups * 4, lp.n_groups, kRowsPerBlock,
                                lp.n_groups == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) &&
                    make_map_2d(&mz, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.zeros, lp.n_groups, lp.N, lp.n_groups,
                                lp.n_groups, kRowsPerBlock,
                                lp.n_groups == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE);
    q.boxes3d = lp.K % 256 == 0 &&
                make_map_3d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, kKtileCodeBytes, lp.N, P / kKtileCodeBytes,
                            P, kKtileCodeBytes, kKtileCodeBytes, kRowsPerBlock, W,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (!q.boxes3d && !make_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, P, lp.N, P, kKtileCodeBytes,
                                   kRowsPerBlock, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (!q.asym_staged) ms = mz = mc;  // unused
  } else if (lp.channel) {
    // per-channel: codes only (one 3-D box per stage when the rows hold whole stages of k-tiles)
    q.boxes3d = lp.K % 1024 == 0 &&
                make_map_3d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, kKtileCodeBytes, lp.N, P / kKtileCodeBytes,
                            P, kKtileCodeBytes, kKtileCodeBytes, kRowsPerBlock, W, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!q.boxes3d && !make_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, P, lp.N, P, kKtileCodeBytes,
                                   kRowsPerBlock, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    ms = mz = mc;  // unused
  } else {
    // 3-D boxes need whole 256-column tiles of codes and whole 1024-column quads of scales in
    // every row (a box never reaches past a row's end into the next row)
    q.boxes3d = lp.K % 1024 == 0 &&
                make_map_3d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, kKtileCodeBytes, lp.N, P / kKtileCodeBytes,
                            P, kKtileCodeBytes, kKtileCodeBytes, kRowsPerBlock, W,
                            CU_TENSOR_MAP_SWIZZLE_128B) &&
                make_map_3d(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lp.scales, 32, lp.N, G / 32, G * 4, 128, 32,
                            kRowsPerBlock, W / 4, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!q.boxes3d &&
        (!make_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, lp.codes, P, lp.N, P, kKtileCodeBytes, kRowsPerBlock,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
         !make_map_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lp.scales, G, lp.N, G * 4, 32, kRowsPerBlock,
                      CU_TENSOR_MAP_SWIZZLE_128B)))
      return cudaErrorInvalidValue;
    mz = ms;  // unused
  }
  const int64_t slots = static_cast<int64_t>(sm_count_current()) * per_sm;
  const int64_t grid = q.NB < slots ? q.NB : slots;
  q.rb_q = static_cast<int>(q.NB / grid);
  q.rb_r = static_cast<int>(q.NB % grid);
  const int gi = static_cast<int>(grid);
  if (lp.asym) {
    if (lp.M == 1) return launch_typed<0, true>(mc, ms, mz, q, smem, gi, err, stream);
    if (lp.M <= 8) return launch_typed<1, true>(mc, ms, mz, q, smem, gi, err, stream);
    return launch_typed<2, true>(mc, ms, mz, q, smem, gi, err, stream);
  }
  if (lp.channel) {
    if (lp.M == 1) return launch_typed<0, false, true>(mc, ms, mz, q, smem, gi, err, stream);
    if (lp.M <= 8) return launch_typed<1, false, true>(mc, ms, mz, q, smem, gi, err, stream);
    return launch_typed<2, false, true>(mc, ms, mz, q, smem, gi, err, stream);
  }
  if (lp.M == 1) return launch_typed<0, false>(mc, ms, mz, q, smem, gi, err, stream);
  if (lp.M <= 8) return launch_typed<1, false>(mc, ms, mz, q, smem, gi, err, stream);
  return launch_typed<2, false>(mc, ms, mz, q, smem, gi, err, stream);
}

}  // namespace w4i

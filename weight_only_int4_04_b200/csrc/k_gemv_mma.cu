// Decode / small-M linear (M <= 16) with register-fed tensor cores:
//   y[m][n] = sum_k x[m][k] * (v[n][k] * s[n][k/32]) + b[n]
//
// Why tensor cores here: the weight stream is HBM-bound (0.625 B per weight), but at the
// B200's bandwidth the SMs can issue only ~3.5 thread-instructions per streamed weight. A
// CUDA-core inner product needs >= 2.4 (exact fp32 products) and left no room for the rest,
// so the multiply-accumulate goes to mma.sync m16n8k16 (bf16 in, fp32 accumulate): the
// nibbles are unpacked by LOP3 + one exact bf16x2 subtract straight into the A-fragment
// registers (weights = A, swap-AB) and a single MMA consumes 8 weights per lane for up to
// 8 activation rows. tcgen05 cannot take register operands; staging the unpacked weights
// through shared memory would cost more issue slots than it saves.
//
// Structure (one CTA per SM, balanced contiguous row ranges):
//   * a producer thread copies each row of codes / scales (/ zeros) of a slot of RS rows with
//     cp.async.bulk into a ring of shared-memory slots. Rows land at a pitch padded by 16
//     bytes, which makes the per-lane fragment loads bank-conflict free;
//   * the activations are staged once per CTA into shared memory already permuted into
//     B-fragment order (16 bytes per lane per 32-column group);
//   * 16 consumer warps split the groups of each slot; per group a lane loads one code word
//     per row (rows g and g+8 of the 16-row A tile), unpacks it to four exact bf16x2
//     integers, runs two MMAs per 8 activation rows and folds the group's scale into its
//     fp32 accumulators (one FFMA per accumulator);
//   * per slot, the warps' accumulators are summed in shared memory in a fixed order
//     (deterministic), the bias is added and y is written; the slot is released.
// Asymmetric act-order weights (codes sorted by w4_asym_prepare) run the same kernel with
// unsigned nibbles minus a per-row zero point and x gathered through perm.
#include "w4_dot.cuh"
#include "w4_sync.cuh"

namespace w4i {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxSlots = 8;
constexpr int kSmemBudget = 220 * 1024;
constexpr int kBarAll = 1;     // named barrier of all consumer warps
constexpr int kBarGroup0 = 2;  // warp group i uses barrier 2 + i (i < 8)

struct MmaGeom {
  int64_t P;         // code bytes per row
  int64_t SG;        // scale (and zero) columns per row
  int64_t G;         // 32-column groups per row
  int rs;            // rows per slot: 8 or 16
  int code_pitch;    // P + 16
  int scale_pitch;   // 4 * SG + 16
  int zero_pitch;    // SG + 16 (asymmetric)
  int slot_bytes;
  int scales_off;
  int zeros_off;
  int nslots;
  int x_bytes;       // G * M * 64
  int red_off;       // reduction buffer (after x)
  int gcol_off;      // asym: per-group scale column table
  int zero_off;      // zeroed floats (at least one per group) read for rows that do not exist
  int bar_off;
  int x_vec;
  int wg;            // warps per group
  int ngroups;       // warp groups (each owns whole slots)
  int spg;           // slots per warp group (each group walks its own ring)
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float ldsf(uint32_t addr) { return __uint_as_float(lds32(addr)); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// One code word (8 columns of one row) -> four exact bf16x2 pairs (columns (0,4) (1,5)
// (2,6) (3,7) of the word). magic/offset as in nib_pair_bf16: signed codes give q, unsigned
// codes minus the zero point give u - z.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t magic, uint32_t offset, uint32_t (&u)[4]) {
  u[0] = bf16x2_sub(nib_pair_bf16(w, magic), offset);
  u[1] = bf16x2_sub(nib_pair_bf16(w >> 4, magic), offset);
  u[2] = bf16x2_sub(nib_pair_bf16(w >> 8, magic), offset);
  u[3] = bf16x2_sub(nib_pair_bf16(w >> 12, magic), offset);
}

// First MMA of a group with a zero accumulator input (no register zeroing needed).
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

template <int NT, int RS, bool ASYM>
__global__ void __launch_bounds__(kThreads, 1) gemv_mma_kernel(const LinearParams p, const MmaGeom g, int32_t *err) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *xs = smem + static_cast<size_t>(g.nslots) * g.slot_bytes;
  float *red = reinterpret_cast<float *>(smem + g.red_off);
  int32_t *gcol = reinterpret_cast<int32_t *>(smem + g.gcol_off);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + g.bar_off);
  uint64_t *empty = full + kMaxSlots;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kMaxSlots);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = p.N, K = p.K;
  const int M = static_cast<int>(p.M);
  const int G = static_cast<int>(g.G);
  const int64_t row_begin = static_cast<int64_t>(blockIdx.x) * N / gridDim.x;
  const int64_t row_end = static_cast<int64_t>(blockIdx.x + 1) * N / gridDim.x;
  const int nstages = static_cast<int>((row_end - row_begin + RS - 1) / RS);

  if (threadIdx.x == 0) {
    for (int i = 0; i < g.nslots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---- producer: per row one bulk copy per array into the padded slot layout ----
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < nstages; ++s) {
        // stage s belongs to warp group s % ngroups, which walks its own ring of spg slots
        const int kq = s / g.ngroups;
        const int slot = (s % g.ngroups) * g.spg + kq % g.spg;
        const uint32_t ph = static_cast<uint32_t>(kq / g.spg) & 1u;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag, err)) break;
        const int64_t r0 = row_begin + static_cast<int64_t>(s) * RS;
        const int nr = static_cast<int>((row_end - r0) < RS ? (row_end - r0) : RS);
        uint8_t *base = smem + static_cast<size_t>(slot) * g.slot_bytes;
        const uint32_t cb = static_cast<uint32_t>(g.P), sb = static_cast<uint32_t>(4 * g.SG);
        const uint32_t zb = ASYM ? static_cast<uint32_t>(g.SG) : 0u;
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nr) * (cb + sb + zb));
        for (int r = 0; r < nr; ++r) {
          bulk_copy_g2s(base + r * g.code_pitch, p.codes + (r0 + r) * g.P, cb, &full[slot]);
          bulk_copy_g2s(base + g.scales_off + r * g.scale_pitch, p.scales + (r0 + r) * g.SG, sb, &full[slot]);
          if (ASYM)
            bulk_copy_g2s(base + g.zeros_off + r * g.zero_pitch, p.zeros + (r0 + r) * g.SG, zb, &full[slot]);
        }
        issued = s + 1;
      }
      // the copies issued land before the CTA may exit (see w4_sync.cuh, abort path); each
      // slot's latest phase lies in the last ngroups * spg stages, one stage per slot
      const int ring = g.ngroups * g.spg;
      for (int s = issued - ring < 0 ? 0 : issued - ring; s < issued; ++s) {
        const int kq = s / g.ngroups;
        mbar_drain(&full[(s % g.ngroups) * g.spg + kq % g.spg], static_cast<uint32_t>(kq / g.spg) & 1u, err);
      }
    }
    return;
  }

  // ---- consumers: stage x once, in B-fragment order ----
  const int tid = threadIdx.x;
  {
    const uint16_t *xb = reinterpret_cast<const uint16_t *>(p.x);
    const int chunks = G * M * 4;  // (group, m, t) -> 16 bytes
    for (int c = tid; c < chunks; c += kConsumers) {
      const int t = c & 3;
      const int gm = c >> 2;
      const int m = gm % M, grp = gm / M;
      const int64_t col0 = 32 * static_cast<int64_t>(grp) + 8 * t;
      uint32_t r[4] = {0u, 0u, 0u, 0u};
      if (!ASYM && g.x_vec && col0 + 7 < K) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xb + m * K + col0));
        r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (col0 + e < K) {
            const int64_t col = ASYM ? static_cast<int64_t>(__ldg(p.perm + col0 + e)) : col0 + e;
            r[e >> 1] |= static_cast<uint32_t>(__ldg(xb + m * K + col)) << (16 * (e & 1));
          }
        }
      }
      uint4 v;
      v.x = prmt(r[0], r[2], 0x5410);
      v.y = prmt(r[0], r[2], 0x7632);
      v.z = prmt(r[1], r[3], 0x5410);
      v.w = prmt(r[1], r[3], 0x7632);
      *reinterpret_cast<uint4 *>(xs + ((grp * M + m) * 4 + t) * 16) = v;
    }
    if (ASYM) {
      // scale column of each 32-column sorted group, or -1 when it straddles two groups
      for (int grp = tid; grp < G; grp += kConsumers) {
        const int64_t c0 = 32 * static_cast<int64_t>(grp);
        const int64_t last = (c0 + 31 < K) ? c0 + 31 : K - 1;
        const int32_t first = __ldg(p.g_idx + __ldg(p.perm + c0));
        gcol[grp] = (first == __ldg(p.g_idx + __ldg(p.perm + last))) ? first : -1;
      }
      // zero the per-group fallback deposit areas
      float *dep0 = red + g.ngroups * (g.wg * NT * 128);
      for (int i = tid; i < g.ngroups * 256; i += kConsumers) dep0[i] = 0.0f;
    }
  }
  {
    float *zf = reinterpret_cast<float *>(smem + g.zero_off);
    for (int i = tid; i < G + 4; i += kConsumers) zf[i] = 0.0f;
  }
  named_barrier_sync(kBarAll, kConsumers);

  // ---- warp groups: group `grp_id` (wg warps) owns slots grp_id, grp_id + ngroups, ... ----
  const int grp_id = warp / g.wg, wig = warp % g.wg;
  if (grp_id >= g.ngroups) return;
  const int bar_id = kBarGroup0 + grp_id;
  const int bar_threads = 32 * g.wg;
  const int gid = lane >> 2, tig = lane & 3;
  const uint32_t xs_lane = smem_u32(xs) + static_cast<uint32_t>(tig * 16);
  const uint32_t x_gstride = static_cast<uint32_t>(M * 64);  // bytes per group in xs
  const uint32_t magic = ASYM ? 0x43004300u : 0x43084308u;
  float *fr = red + grp_id * (g.wg * NT * 128);   // [warp in group][nt][lane][4]
  float *dep = red + g.ngroups * (g.wg * NT * 128) + grp_id * 256;  // asym fallback [m][row]

  for (int s = grp_id; s < nstages; s += g.ngroups) {
    const int kq = s / g.ngroups;
    const int slot = grp_id * g.spg + kq % g.spg;
    const uint32_t ph = static_cast<uint32_t>(kq / g.spg) & 1u;
    mbar_wait(&full[slot], ph, abort_flag, err);
    const int64_t r0 = row_begin + static_cast<int64_t>(s) * RS;
    const int nr = static_cast<int>((row_end - r0) < RS ? (row_end - r0) : RS);
    const uint32_t base = smem_u32(smem + static_cast<size_t>(slot) * g.slot_bytes);
    const bool row0_ok = gid < nr;
    const bool row1_ok = (RS == 16) && (gid + 8 < nr);
    const uint32_t code0 = base + gid * g.code_pitch + 4 * tig;
    const uint32_t code1 = code0 + 8 * g.code_pitch;
    const uint32_t sc0 = base + g.scales_off + gid * g.scale_pitch;
    const uint32_t sc1 = sc0 + 8 * g.scale_pitch;
    const uint32_t zr0 = base + g.zeros_off + gid * g.zero_pitch;
    const uint32_t zr1 = zr0 + 8 * g.zero_pitch;

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;

    if (!ASYM) {
      // Symmetric fast path: this warp takes a contiguous range of groups so that every
      // address advances by a constant; rows past the slot's end read the slot's stale (but
      // finite) codes with a scale of 0 taken from a zeroed area, and activation rows past M
      // read zeros -- no predicates in the loop.
      const int per = (G + g.wg - 1) / g.wg;
      const int g_lo = wig * per;
      const int g_hi = (g_lo + per < G) ? g_lo + per : G;
      const uint32_t zero = smem_u32(smem + g.zero_off);
      uint32_t cp0 = code0 + 16 * g_lo;
      uint32_t cp1 = code1 + 16 * g_lo;
      uint32_t sp0 = (row0_ok ? sc0 : zero) + 4 * g_lo;
      uint32_t sp1 = (row1_ok ? sc1 : zero) + 4 * g_lo;
      uint32_t xpp[NT], xst[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = 8 * nt + gid;
        xst[nt] = m < M ? x_gstride : 0u;
        xpp[nt] = m < M ? xs_lane + g_lo * x_gstride + m * 64 : zero;
      }
      auto one_group = [&](uint32_t c0a, uint32_t c1a, uint32_t s0a, uint32_t s1a) {
        const uint32_t w0 = lds32(c0a);
        const uint32_t w1 = RS == 16 ? lds32(c1a) : 0u;
        const float s0 = ldsf(s0a);
        const float s1 = RS == 16 ? ldsf(s1a) : 0.0f;
        uint32_t a[4], b[4];
        unpack_word(w0, 0x43084308u, 0x43084308u, a);
        if (RS == 16) {
          unpack_word(w1, 0x43084308u, 0x43084308u, b);
        } else {
          b[0] = b[1] = b[2] = b[3] = 0u;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 xf = lds128(xpp[nt]);
          xpp[nt] += xst[nt];
          float d[4];
          mma_16816_z(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
          mma_16816(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
          acc[nt][0] = fmaf(d[0], s0, acc[nt][0]);
          acc[nt][1] = fmaf(d[1], s0, acc[nt][1]);
          acc[nt][2] = fmaf(d[2], s1, acc[nt][2]);
          acc[nt][3] = fmaf(d[3], s1, acc[nt][3]);
        }
      };
      int grp = g_lo;
      for (; grp + 4 <= g_hi; grp += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) one_group(cp0 + 16 * u, cp1 + 16 * u, sp0 + 4 * u, sp1 + 4 * u);
        cp0 += 64;
        cp1 += 64;
        sp0 += 16;
        sp1 += 16;
      }
      for (; grp < g_hi; ++grp) {
        one_group(cp0, cp1, sp0, sp1);
        cp0 += 16;
        cp1 += 16;
        sp0 += 4;
        sp1 += 4;
      }
    } else {
    for (int grp = wig; grp < G; grp += g.wg) {
        int sgc = grp;  // scale column of this group
        uint32_t off0 = 0x43084308u, off1 = 0x43084308u;
        if (ASYM) {
          sgc = gcol[grp];
          if (sgc < 0) {
            // two groups inside these 32 sorted columns: exact per-column fallback, deposited
            // per (m, row) through shared-memory atomics
            const int64_t c0 = 32 * static_cast<int64_t>(grp);
  #pragma unroll
            for (int half = 0; half < (RS == 16 ? 2 : 1); ++half) {
              const int rr = gid + 8 * half;
              if (rr >= nr) continue;
              const uint32_t w = lds32(base + rr * g.code_pitch + 16 * grp + 4 * tig);
              const uint32_t sca = base + g.scales_off + rr * g.scale_pitch;
              const uint32_t zra = base + g.zeros_off + rr * g.zero_pitch;
              for (int e = 0; e < 8; ++e) {
                const int64_t col = c0 + 8 * tig + e;
                if (col >= K) continue;
                const int gg = __ldg(p.g_idx + __ldg(p.perm + col));
                const int u = static_cast<int>((w >> (4 * e)) & 15u);
                const int z = static_cast<int>((lds32((zra + gg) & ~3u) >> (8 * ((zra + gg) & 3))) & 15u);
                const float wv = __fmul_rn(static_cast<float>(u - z), ldsf(sca + 4 * gg));
                for (int m = 0; m < M; ++m) {
                  const uint32_t xw = lds32(xs_lane + grp * x_gstride + m * 64 + 4 * (e & 3));
                  const float xv = __uint_as_float((e < 4 ? (xw & 0xFFFFu) : (xw >> 16)) << 16);
                  atomicAdd(dep + m * 16 + rr, xv * wv);
                }
              }
            }
            continue;
          }
          const uint32_t z0 = row0_ok ? ((lds32((zr0 + sgc) & ~3u) >> (8 * ((zr0 + sgc) & 3))) & 15u) : 0u;
          const uint32_t z1 = row1_ok ? ((lds32((zr1 + sgc) & ~3u) >> (8 * ((zr1 + sgc) & 3))) & 15u) : 0u;
          off0 = (0x4300u | z0) * 0x00010001u;
          off1 = (0x4300u | z1) * 0x00010001u;
        }
        const uint32_t w0 = row0_ok ? lds32(code0 + 16 * grp) : 0u;  // nibble 0 decodes to 0
        const uint32_t w1 = row1_ok ? lds32(code1 + 16 * grp) : 0u;
        const float s0 = row0_ok ? ldsf(sc0 + 4 * sgc) : 0.0f;
        const float s1 = row1_ok ? ldsf(sc1 + 4 * sgc) : 0.0f;
        uint32_t a[4], b[4];
        unpack_word(w0, magic, off0, a);
        if (RS == 16) {
          unpack_word(w1, magic, off1, b);
        } else {
          b[0] = b[1] = b[2] = b[3] = 0u;
        }
        const uint32_t xa = xs_lane + grp * x_gstride;
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int m = 8 * nt + gid;
          uint4 xf = make_uint4(0u, 0u, 0u, 0u);
          if (m < M) xf = lds128(xa + m * 64);
          float d[4];
          mma_16816_z(d, a[0], b[0], a[1], b[1], xf.x, xf.y);
          mma_16816(d, a[2], b[2], a[3], b[3], xf.z, xf.w);
          acc[nt][0] = fmaf(d[0], s0, acc[nt][0]);
          acc[nt][1] = fmaf(d[1], s0, acc[nt][1]);
          acc[nt][2] = fmaf(d[2], s1, acc[nt][2]);
          acc[nt][3] = fmaf(d[3], s1, acc[nt][3]);
        }
      }
    }

    // ---- reduction over the group's warps (fixed order) and output ----
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<float4 *>(fr + ((wig * NT + nt) * 32 + lane) * 4) =
          make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
    named_barrier_sync(bar_id, bar_threads);
    const int gt = wig * 32 + lane;
    if (gt == 0) mbar_arrive(&empty[slot]);  // the group is done reading this slot
    for (int o = gt; o < RS * M; o += bar_threads) {
      const int r = o / M, m = o % M;
      if (r < nr) {
        const int nt = m >> 3, mm = m & 7;
        const int ln = 4 * (r & 7) + (mm >> 1);
        const int idx = ((r >= 8) ? 2 : 0) + (mm & 1);
        float v = 0.0f;
        for (int w = 0; w < g.wg; ++w) v += fr[((w * NT + nt) * 32 + ln) * 4 + idx];
        if (ASYM) {
          v += dep[m * 16 + r];
          dep[m * 16 + r] = 0.0f;
        }
        const int64_t n = r0 + r;
        if (p.bias) v += __ldg(p.bias + n);
        if (p.y_dtype == W4_F32) {
          static_cast<float *>(p.y)[m * N + n] = v;
        } else {
          static_cast<__nv_bfloat16 *>(p.y)[m * N + n] = __float2bfloat16_rn(v);
        }
      }
    }
    named_barrier_sync(bar_id, bar_threads);
  }
}

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      count = n;
    else
      return 148;
  }
  return count;
}

bool make_geom(const LinearParams &p, MmaGeom *g) {
  if (p.M < 1 || p.M > 16) return false;
  const int64_t K = p.K;
  g->P = (K + 1) / 2;
  g->G = (K + 31) / 32;
  g->SG = p.asym ? p.n_groups : g->G;
  if (g->P % 16 != 0) return false;
  if (p.asym && (p.perm == nullptr || g->SG % 16 != 0)) return false;
  if (!p.asym && g->SG % 4 != 0) return false;
  const uintptr_t align = reinterpret_cast<uintptr_t>(p.codes) | reinterpret_cast<uintptr_t>(p.scales) |
                          (p.asym ? reinterpret_cast<uintptr_t>(p.zeros) : 0);
  if (align % 16 != 0) return false;
  g->code_pitch = static_cast<int>(g->P + 16);
  g->scale_pitch = static_cast<int>(4 * g->SG + 16);
  g->zero_pitch = p.asym ? static_cast<int>(((g->SG + 15) / 16) * 16 + 16) : 0;
  g->x_bytes = static_cast<int>(g->G * p.M * 64);
  // at least ~32 groups per warp-group pass; at most 8 warp groups (named barriers 2..9)
  const int64_t wg_min = (g->G + 31) / 32 < kConsumerWarps ? ((g->G + 31) / 32 < 1 ? 1 : (g->G + 31) / 32)
                                                          : kConsumerWarps;
  const int64_t ngroups = kConsumerWarps / wg_min < 8 ? kConsumerWarps / wg_min : 8;
  const int nt = p.M > 8 ? 2 : 1;
  // fragment sums [16 warps][nt][lane][4] + asym fallback deposits [group][16 m][16 rows]
  const int red_bytes = static_cast<int>((kConsumerWarps * nt * 128 + 8 * 256) * 4);
  const int gcol_bytes = p.asym ? static_cast<int>(((4 * g->G + 15) / 16) * 16) : 0;
  const int zero_bytes = static_cast<int>(((4 * g->G + 16 + 15) / 16) * 16);
  const int tail = red_bytes + gcol_bytes + zero_bytes + 2 * kMaxSlots * 8 + 16;
  for (int rs : {16, 8}) {
    const int64_t slot = static_cast<int64_t>(rs) * (g->code_pitch + g->scale_pitch + g->zero_pitch);
    const int64_t room = kSmemBudget - tail - g->x_bytes;
    if (room < 2 * slot) continue;
    int64_t nslots = room / slot < kMaxSlots ? room / slot : kMaxSlots;
    // every warp group gets its own ring of at least two slots (double buffering)
    const int64_t groups = ngroups < nslots / 2 ? ngroups : (nslots / 2 > 0 ? nslots / 2 : 1);
    const int64_t spg = nslots / groups;
    nslots = groups * spg;
    g->rs = rs;
    g->slot_bytes = static_cast<int>(slot);
    g->scales_off = rs * g->code_pitch;
    g->zeros_off = rs * (g->code_pitch + g->scale_pitch);
    g->nslots = static_cast<int>(nslots);
    g->red_off = static_cast<int>(nslots * slot + g->x_bytes);
    g->gcol_off = g->red_off + red_bytes;
    g->zero_off = g->gcol_off + gcol_bytes;
    g->bar_off = g->zero_off + zero_bytes;
    g->x_vec = (K % 8 == 0) && (reinterpret_cast<uintptr_t>(p.x) % 16 == 0);
    g->wg = static_cast<int>(kConsumerWarps / groups);  // the surviving groups share all warps
    g->ngroups = static_cast<int>(groups);
    g->spg = static_cast<int>(spg);
    return true;
  }
  return false;
}

template <int NT, int RS, bool ASYM>
cudaError_t launch_typed(const LinearParams &p, const MmaGeom &g, int32_t *err, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(g.bar_off) + 2 * kMaxSlots * 8 + 16;
  auto kern = gemv_mma_kernel<NT, RS, ASYM>;
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int64_t grid = (p.N + RS - 1) / RS;
  if (grid > sm_count()) grid = sm_count();
  kern<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(p, g, err);
  return cudaGetLastError();
}

template <int NT, int RS>
cudaError_t launch_rs(const LinearParams &p, const MmaGeom &g, int32_t *err, cudaStream_t stream) {
  return p.asym ? launch_typed<NT, RS, true>(p, g, err, stream) : launch_typed<NT, RS, false>(p, g, err, stream);
}

}  // namespace

bool gemv_mma_supports(const LinearParams &p) {
  MmaGeom g;
  return make_geom(p, &g);
}

cudaError_t launch_gemv_mma(const LinearParams &p, int32_t *err, cudaStream_t stream) {
  MmaGeom g;
  if (!make_geom(p, &g)) return cudaErrorNotSupported;
  if (p.M <= 8) return g.rs == 16 ? launch_rs<1, 16>(p, g, err, stream) : launch_rs<1, 8>(p, g, err, stream);
  return g.rs == 16 ? launch_rs<2, 16>(p, g, err, stream) : launch_rs<2, 8>(p, g, err, stream);
}

}  // namespace w4i
